"""Pins for the oracle's fp64 masked attention: reduction to torch SDPA, closed cases, invariants."""
import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, SegmentText, Tail, make_inputs, small_config
from oracle import attention as att
from oracle import select as sel
from oracle.quant import dequantize
from oracle.ring import OracleCache
from tests.test_oracle_visibility import _brute_rollout


def _f32(t):
    return t.float().numpy()


def _build(cfg, inp=None):
    inp = inp or make_inputs(cfg)
    c = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames,
                    cfg.capacity_frames, cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        c.append(_f32(kv.k), _f32(kv.v), seg.n_frames,
                 None if kv.head_k is None else _f32(kv.head_k), None if kv.head_v is None else _f32(kv.head_v))
    return c, inp


@pytest.mark.parametrize("cfg", [CONFIGS["C0"], CONFIGS["C0w3"], small_config(),
                                 small_config(window=0, prior_frames=(2, 1), tails=((10, 0, 2),))])
def test_reduces_to_torch_sdpa_with_brute_force_mask(cfg):
    cache, inp = _build(cfg)
    scale = 1.0 / np.sqrt(cfg.head_dim)
    out, lse = att.attention(cache, _f32(inp.q), _f32(inp.k_cur), _f32(inp.v_cur),
                             _f32(inp.k_txt), _f32(inp.v_txt), cfg.current, scale)
    segs = list(cfg.prior) + [cfg.current]
    mask, lh = _brute_rollout(cfg.tokens_per_frame, cfg.window_frames, segs)
    hk8, hks, hv8, hvs = cache.history()
    pk8, pks, pv8, pvs = cache.prior_heads()
    for h in range(cfg.heads):
        K = torch.cat([torch.from_numpy(dequantize(hk8[h], hks[h])), torch.from_numpy(dequantize(pk8[h], pks[h])),
                       inp.k_cur[:, h].double(), inp.k_txt[:, h].double()])
        V = torch.cat([torch.from_numpy(dequantize(hv8[h], hvs[h])), torch.from_numpy(dequantize(pv8[h], pvs[h])),
                       inp.v_cur[:, h].double(), inp.v_txt[:, h].double()])
        Q = inp.q[:, h].double()
        m = torch.from_numpy(mask)
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=m[None], scale=scale)[0]
        assert np.allclose(out[:, h], ref.numpy(), rtol=0, atol=1e-12)
        s = (Q @ K.T) * scale
        ref_lse = torch.logsumexp(s.masked_fill(~m, -float("inf")), dim=1)
        assert np.allclose(lse[h], ref_lse.numpy(), rtol=0, atol=1e-12)


def test_weights_sum_to_one_via_constant_values():
    cfg = small_config()
    cache, inp = _build(cfg)
    # V = 1 in every uncached source; cached V of 1 dequantises to 127 * fp32(1/127)
    ones = torch.ones_like(inp.v_cur)
    inp2 = type(inp)(cfg, inp.q, inp.k_cur, ones, inp.k_txt, torch.ones_like(inp.v_txt), inp.prior)
    c2 = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                     cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        o = np.ones(tuple(kv.v.shape), np.float32)
        oh = None if kv.head_v is None else np.ones(tuple(kv.head_v.shape), np.float32)
        c2.append(_f32(kv.k), o, seg.n_frames, None if kv.head_k is None else _f32(kv.head_k), oh)
    out, _ = att.attention(c2, _f32(inp2.q), _f32(inp2.k_cur), _f32(inp2.v_cur), _f32(inp2.k_txt),
                           _f32(inp2.v_txt), cfg.current, 0.1)
    assert np.all(np.abs(out - 1.0) < 1e-6)


def test_single_visible_key_returns_its_value():
    cfg = small_config(tokens_per_frame=1, n_frames=1, prior_frames=(), prior_head=0, head_len=0, tails=(),
                       window=0, heads=3)
    cache, inp = _build(cfg)
    out, lse = att.attention(cache, _f32(inp.q), _f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt),
                             _f32(inp.v_txt), cfg.current, 0.125)
    assert np.array_equal(out[0], _f32(inp.v_cur)[0].astype(np.float64))
    s = (_f32(inp.q)[0].astype(np.float64) * _f32(inp.k_cur)[0]).sum(-1) * 0.125
    assert np.allclose(lse[:, 0], s, atol=1e-12)


def test_physical_ring_rotation_does_not_change_output():
    cfg = small_config(window=3, prior_frames=(2, 2, 2))
    inp = make_inputs(cfg)
    a, _ = _build(cfg, inp)
    cfg_b = small_config(window=3, prior_frames=(2, 2, 2))
    b = OracleCache(cfg_b.heads, cfg_b.head_dim, cfg_b.tokens_per_frame, 3, 8, cfg_b.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        b.append(_f32(kv.k), _f32(kv.v), seg.n_frames, _f32(kv.head_k), _f32(kv.head_v))
    args = (_f32(inp.q), _f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt), _f32(inp.v_txt), cfg.current, 0.09)
    oa, la = att.attention(a, *args)
    ob, lb = att.attention(b, *args)
    assert np.abs(oa - ob).max() < 1e-12 and np.abs(la - lb).max() < 1e-12


def test_earlier_tails_never_influence_later_segments_and_heads_do():
    cfg = small_config(window=0, prior_frames=(2, 2))
    cache, inp = _build(cfg)
    args = (_f32(inp.q), _f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt), _f32(inp.v_txt), cfg.current, 0.09)
    base, _ = att.attention(cache, *args)
    # an earlier segment's action tails are not part of what it appends: the cache has no place for them
    assert cache.head_used == sum(p.head_len for p in cfg.prior)
    # zeroing one prior description head's V changes the output
    cache.hv8[:, :5] = 0
    changed, _ = att.attention(cache, *args)
    assert np.abs(changed - base).max() > 1e-6


def test_sparse_full_keep_equals_dense_and_quarter_keep_drops_blocks():
    cfg = small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4)
    cache, inp = _build(cfg)
    q, kc = _f32(inp.q), _f32(inp.k_cur)
    hk8, hks, _, _ = cache.history()
    args = (q, kc, _f32(inp.v_cur), _f32(inp.k_txt), _f32(inp.v_txt), cfg.current, 0.09)
    dense, dl = att.attention(cache, *args)
    s_all, _ = sel.select(q, hk8, hks, kc, 1.0)
    full, fl = att.attention(cache, *args, sel=s_all)
    assert np.array_equal(dense, full) and np.array_equal(dl, fl)
    s_q, _ = sel.select(q, hk8, hks, kc, 0.25)
    part, pl = att.attention(cache, *args, sel=s_q)
    assert np.all(pl <= dl + 1e-12) and np.abs(part - dense).max() > 1e-3
