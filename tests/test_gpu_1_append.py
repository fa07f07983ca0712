"""GPU parity of nomas_kv_append (bit-exact INT8 codes, scales and ring placement) and nomas_kv_dequant."""
import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, small_config
from tests.helpers import f32, gpu_cache, oracle_cache

pytestmark = pytest.mark.gpu


def _compare_cache(gc, oc):
    st = gc.state()
    assert st["frames_appended"] == oc.frames_appended
    assert st["head_tokens"] == oc.head_used
    assert st["history_tokens"] == oc.history_tokens()
    T = oc.T
    k8, v8 = gc.ring_k8().cpu().numpy(), gc.ring_v8().cpu().numpy()
    ks, vs = gc.ring_ks().cpu().numpy(), gc.ring_vs().cpu().numpy()
    for g in oc.retained_frames():
        s = slice((g % oc.C) * T, (g % oc.C + 1) * T)
        assert np.array_equal(k8[:, s], oc.k8[:, s]), f"K codes of frame {g}"
        assert np.array_equal(v8[:, s], oc.v8[:, s]), f"V codes of frame {g}"
        assert np.array_equal(ks[:, s].view(np.uint32), oc.ks[:, s].view(np.uint32)), f"K scales of frame {g}"
        assert np.array_equal(vs[:, s].view(np.uint32), oc.vs[:, s].view(np.uint32)), f"V scales of frame {g}"
    u = oc.head_used
    if u:
        assert np.array_equal(gc.head_k8()[:, :u].cpu().numpy(), oc.hk8[:, :u])
        assert np.array_equal(gc.head_v8()[:, :u].cpu().numpy(), oc.hv8[:, :u])
        assert np.array_equal(gc.head_ks()[:, :u].cpu().numpy().view(np.uint32), oc.hks[:, :u].view(np.uint32))
        assert np.array_equal(gc.head_vs()[:, :u].cpu().numpy().view(np.uint32), oc.hvs[:, :u].view(np.uint32))


SMALL = [CONFIGS["C0"], CONFIGS["C0w3"], small_config(),
         small_config(window=0, prior_frames=(2, 1, 3), head_dim=64, heads=3),
         small_config(window=3, prior_frames=(5, 1, 4), tokens_per_frame=37)]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name + f"_w{c.window_frames}_d{c.head_dim}")
def test_append_bit_exact_after_every_segment(cfg):
    from int8_kv_cache_action_b200.runtime import KVCache
    from oracle.ring import OracleCache
    inp = make_inputs(cfg)
    gc = KVCache.for_config(cfg)
    oc = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                     cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        gc.append(kv.k.cuda(), kv.v.cuda(), seg.n_frames,
                  None if kv.head_k is None else kv.head_k.cuda(), None if kv.head_v is None else kv.head_v.cuda())
        oc.append(f32(kv.k), f32(kv.v), seg.n_frames, f32(kv.head_k), f32(kv.head_v))
        _compare_cache(gc, oc)
    # and the current segment, as the step after its generation would append it
    if cfg.window_frames or oc.frames_appended + cfg.current.n_frames <= cfg.capacity_frames:
        hl = cfg.current.head_len
        if oc.head_used + hl <= cfg.head_store_tokens:
            hk, hv = inp.k_txt[:hl], inp.v_txt[:hl]
            gc.append(inp.k_cur.cuda(), inp.v_cur.cuda(), cfg.current.n_frames,
                      hk.cuda() if hl else None, hv.cuda() if hl else None)
            oc.append(f32(inp.k_cur), f32(inp.v_cur), cfg.current.n_frames, f32(hk) if hl else None,
                      f32(hv) if hl else None)
            _compare_cache(gc, oc)
    assert gc.status() == 0


@pytest.mark.parametrize("name", ["C1", "C2", "C4"])
def test_append_full_size(name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    _compare_cache(gc, oc)
    assert gc.status() == 0


def test_strided_head_major_input_and_dequant():
    cfg = small_config(window=4, prior_frames=(3, 3))
    inp = make_inputs(cfg)
    from int8_kv_cache_action_b200.runtime import KVCache
    gc = KVCache.for_config(cfg)
    for seg, kv in zip(cfg.prior, inp.prior):
        # [H, S, D] storage viewed as [S, H, D]: token stride D, head stride S*D (one stride pair for all)
        n, hl = kv.k.shape[0], kv.head_k.shape[0]
        bufs = torch.zeros(4, cfg.heads, n, cfg.head_dim, dtype=torch.bfloat16)
        bufs[0], bufs[1] = kv.k.transpose(0, 1), kv.v.transpose(0, 1)
        bufs[2, :, :hl], bufs[3, :, :hl] = kv.head_k.transpose(0, 1), kv.head_v.transpose(0, 1)
        g = bufs.cuda().transpose(1, 2)                                   # [4, S, H, D] views
        gc.append(g[0], g[1], seg.n_frames, g[2][:hl], g[3][:hl])
    oc = oracle_cache(cfg, inp)
    _compare_cache(gc, oc)
    kd, vd = gc.dequant()
    hk8, hks, hv8, hvs = oc.history()
    want_k = (hk8.astype(np.float32) * hks[..., None]).transpose(1, 0, 2)
    want_v = (hv8.astype(np.float32) * hvs[..., None]).transpose(1, 0, 2)
    assert np.array_equal(kd.cpu().numpy(), want_k) and np.array_equal(vd.cpu().numpy(), want_v)


def test_capacity_and_argument_errors_leave_cache_unchanged():
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import KVCache
    gc = KVCache(2, 128, 10, 0, 3, 8)
    k = torch.randn(20, 2, 128, device="cuda").bfloat16()
    gc.append(k, k, 2)
    with pytest.raises(N.NomasError) as e:
        gc.append(k, k, 2)
    assert e.value.status == N.NOMAS_ECAPACITY
    h = torch.randn(9, 2, 128, device="cuda").bfloat16()
    with pytest.raises(N.NomasError) as e:
        gc.append(k[:10], k[:10], 1, h, h)
    assert e.value.status == N.NOMAS_ECAPACITY
    rc = N.nomas_kv_append(gc.handle, k.data_ptr() + 2, k.data_ptr(), 256, 128, 1, 0, 0, 0)
    assert rc == N.NOMAS_EINVAL
    st = gc.state()
    assert st["frames_appended"] == 2 and st["head_tokens"] == 0 and st["segments"] == 1


def _adversarial_rows(D, seed=5):
    """bf16 rows (float32 values) whose absmax runs over every positive finite bf16 value, each with
    random other channels below it, plus rows of zeros, single subnormals, exact half-integer ties at a
    power-of-two scale and values at the bf16 maximum."""
    rng = np.random.default_rng(seed)
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint32)                 # subnormals and normals
    a = (bits << 16).view(np.float32)
    n = a.shape[0]
    frac = rng.uniform(-1.0, 1.0, size=(n, D)).astype(np.float32)
    rows = (frac * a[:, None]).astype(np.float32)
    rows[np.arange(n), rng.integers(0, D, n)] = a * rng.choice([-1.0, 1.0], n).astype(np.float32)
    extra = []
    extra.append(np.zeros(D, np.float32))
    z = np.zeros(D, np.float32)
    z[3] = np.float32(2.0 ** -133)
    extra.append(z)
    for k in (-100, -20, 0, 3, 50, 120):                           # s = 2^k, x = (j + 1/2) 2^k: ties
        j = rng.integers(-127, 127, D).astype(np.float32)
        x = ((j + np.float32(0.5)) * np.float32(2.0 ** k)).astype(np.float32)
        x[0] = np.float32(127 * 2.0 ** k)
        extra.append(x)
    big = np.float32((np.uint32(0x7F7F) << 16).view(np.float32))
    extra.append(rng.choice([-1.0, 1.0], D).astype(np.float32) * big)
    rows = np.concatenate([rows, np.stack(extra)])
    # round to bf16 (the half-integer ties and the powers of two above are exact in bf16)
    rows = torch.from_numpy(rows).bfloat16()
    return rows


@pytest.mark.parametrize("D", [128, 64])
def test_append_every_bf16_absmax(D):
    """Codes and scales bit-exact for groups whose absmax is each positive bf16 value in turn."""
    from int8_kv_cache_action_b200.runtime import KVCache
    from oracle.ring import OracleCache
    rows = _adversarial_rows(D)
    H, T = 4, 64
    n_tok = (rows.shape[0] + H * T - 1) // (H * T) * T
    pad = torch.zeros(n_tok * H - rows.shape[0], D, dtype=torch.bfloat16)
    k = torch.cat([rows, pad]).reshape(n_tok, H, D)
    v = torch.flip(k, dims=[0])                                      # a different row order for V
    frames = n_tok // T
    gc = KVCache(H, D, T, 0, frames, 8)
    oc = OracleCache(H, D, T, 0, frames, 8)
    gc.append(k.cuda(), v.cuda(), frames)
    oc.append(f32(k), f32(v), frames, None, None)
    _compare_cache(gc, oc)
    assert gc.status() == 0
