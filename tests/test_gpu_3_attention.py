"""GPU parity of nomas_attn_fwd against the fp64 oracle: max-abs 1e-2 and mean-relative 2e-3 on the
output, plus invariants the visibility rule implies (masked keys contribute exactly nothing)."""
import math

import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, small_config
from tests.helpers import (TOL_MAX_ABS, TOL_MEAN_REL, attention_errors, f32, gpu_cache, oracle_cache,
                           sample_rows, to_device)

pytestmark = pytest.mark.gpu

LSE_TOL = 2e-3


def _run(cfg, inp, gc, mode=0, keep=None):
    from int8_kv_cache_action_b200.runtime import segment_text_of
    seg = segment_text_of(cfg.current)
    d = to_device(inp)
    keep = cfg.keep_frac if keep is None else keep
    buf, lay = gc.build_mask(seg, mode, keep, d["q"], d["k_cur"])
    out, lse = gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"],
                            mode=mode, keep_frac=keep, want_lse=True)
    torch.cuda.synchronize()
    return out, lse, buf, lay


def _oracle(cfg, inp, oc, rows, mode=0, keep=None):
    from oracle import attention as att
    from oracle import select as sel
    s = None
    if mode:
        hk8, hks, _, _ = oc.history()
        s, _ = sel.select(f32(inp.q), hk8, hks, f32(inp.k_cur), cfg.keep_frac if keep is None else keep)
    return att.attention(oc, f32(inp.q), f32(inp.k_cur), f32(inp.v_cur), f32(inp.k_txt), f32(inp.v_txt),
                         cfg.current, 1.0 / math.sqrt(cfg.head_dim), rows=rows, sel=s)


def _check(cfg, mode=0, rows=None, keep=None):
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    out, lse, _, _ = _run(cfg, inp, gc, mode, keep)
    assert gc.status() == 0
    rows = np.arange(cfg.n_query) if rows is None else rows
    ref, ref_lse = _oracle(cfg, inp, oc, rows, mode, keep)
    got = out.cpu().numpy()[rows]
    mx, mr = attention_errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= TOL_MAX_ABS and mr <= TOL_MEAN_REL, (mx, mr)
    gl = lse.cpu().numpy()[:, rows]
    assert np.abs(gl - ref_lse).max() <= LSE_TOL
    return mx, mr


SMALL_DENSE = [
    CONFIGS["C0"], CONFIGS["C0w3"],
    small_config(),                                                    # 2 heads x 128, ragged everywhere
    small_config(heads=3, head_dim=64, tokens_per_frame=57, n_frames=4, window=3, prior_frames=(2, 2, 2)),
    small_config(tokens_per_frame=33, n_frames=7, window=0, prior_frames=(2, 5), tails=()),   # no text tails
    small_config(tokens_per_frame=70, n_frames=5, tails=((64, 0, 1), (100, 1, 4), (5, 4, 5), (130, 2, 3))),
    small_config(prior_frames=(), prior_head=0, head_len=0, tails=(), window=0, n_frames=2),   # no history, no text
    small_config(tokens_per_frame=128, n_frames=2, prior_frames=(1,), tails=((128, 0, 1), (128, 1, 2))),  # aligned
]


@pytest.mark.parametrize("cfg", SMALL_DENSE, ids=lambda c: f"{c.name}_d{c.head_dim}_T{c.tokens_per_frame}_F{c.current.n_frames}")
def test_dense_small_all_rows(cfg, attn_kernel):
    _check(cfg)


SMALL_SPARSE = [small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4),
                small_config(tokens_per_frame=97, n_frames=5, prior_frames=(4, 4), window=5, head_dim=64)]


@pytest.mark.parametrize("cfg", SMALL_SPARSE, ids=lambda c: f"{c.name}_d{c.head_dim}_T{c.tokens_per_frame}")
def test_sparse_small_all_rows(cfg, attn_kernel):
    _check(cfg, mode=1)


def test_sparse_full_keep_equals_dense_bitwise(attn_kernel):
    cfg = small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4)
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    dense, dl, _, _ = _run(cfg, inp, gc, 0)
    full, fl, _, _ = _run(cfg, inp, gc, 1, keep=1.0)
    assert torch.equal(dense, full) and torch.equal(dl, fl)


def test_masked_tail_keys_contribute_exactly_nothing(attn_kernel):
    # rows outside a tail's window must not change at all when that tail's K/V change
    cfg = small_config(tokens_per_frame=70, n_frames=5, tails=((64, 0, 1), (100, 1, 4), (5, 4, 5), (130, 2, 3)))
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    base, _, _, _ = _run(cfg, inp, gc)
    a0 = cfg.current.head_len + 64          # tail 1 covers frames [1, 4)
    inp.k_txt[a0:a0 + 100] *= -3
    inp.v_txt[a0:a0 + 100] += 5
    pert, _, _, _ = _run(cfg, inp, gc)
    frames = torch.arange(cfg.n_query, device="cuda") // cfg.tokens_per_frame
    outside = (frames < 1) | (frames >= 4)
    assert torch.equal(base[outside], pert[outside])
    assert (base[~outside] - pert[~outside]).abs().max() > 1e-3


def test_deterministic(attn_kernel):
    cfg = small_config()
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    a, la, _, _ = _run(cfg, inp, gc)
    b, lb, _, _ = _run(cfg, inp, gc)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_stale_mask_is_reported():
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import segment_text_of
    cfg = small_config()
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    d = to_device(inp)
    seg = segment_text_of(cfg.current)
    buf, _ = gc.build_mask(seg)
    gc.append(d["k_cur"][:cfg.tokens_per_frame], d["v_cur"][:cfg.tokens_per_frame], 1)
    gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"])
    assert gc.status() == N.NOMAS_EDEVICE
    assert gc.status() == 0   # the error word is cleared by the read


@pytest.mark.parametrize("name,mode,n_random", [("C1", 0, 300), ("C3r", 1, 300), ("C2", 0, 120), ("C3", 1, 120),
                                                ("C4", 0, 40)])
def test_full_size_sampled_rows(name, mode, n_random):
    cfg = CONFIGS[name]
    rows = sample_rows(cfg, n_random=n_random)
    if name == "C4":
        rows = rows[::3]
    _check(cfg, mode=mode, rows=rows)


def test_prepare_then_run_equals_fwd_and_a_stale_workspace_is_reported():
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import segment_text_of
    cfg = small_config()
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    d = to_device(inp)
    seg = segment_text_of(cfg.current)
    buf, _ = gc.build_mask(seg)
    ref, _ = gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"])
    q, kc, vc, kt, vt = d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"]
    ts, hs = q.stride(0), q.stride(1)
    s = torch.cuda.current_stream().cuda_stream
    scale = 1.0 / math.sqrt(cfg.head_dim)
    ws = gc.workspace(seg)

    def run(workspace, mask):
        out = torch.full_like(ref, -7.0)
        assert N.nomas_attn_run(gc.handle, seg, 0, 0.25, mask.data_ptr(), q.data_ptr(), ts, hs, scale,
                                out.data_ptr(), 0, workspace.data_ptr(), s) == 0
        torch.cuda.synchronize()
        return out

    assert N.nomas_attn_prepare(gc.handle, seg, kc.data_ptr(), vc.data_ptr(), kt.data_ptr(), vt.data_ptr(), ts, hs,
                                ws.data_ptr(), s) == 0
    assert torch.equal(run(ws, buf), ref) and gc.status() == 0
    assert torch.equal(run(ws, buf), ref) and gc.status() == 0      # a prepared workspace serves again
    never = torch.zeros_like(ws)
    out = run(never, buf)                                           # never prepared
    assert gc.status() == N.NOMAS_EDEVICE and bool((out == -7.0).all())
    gc.append(kc[:cfg.tokens_per_frame], vc[:cfg.tokens_per_frame], 1)
    fresh, _ = gc.build_mask(seg)
    out = run(ws, fresh)                                            # prepared before the append
    assert gc.status() == N.NOMAS_EDEVICE and bool((out == -7.0).all())


@pytest.mark.parametrize("name,mode", [("C1", 0), ("C3r", 1), ("C2", 0)])
def test_pair_and_block_kernels_agree(name, mode):
    # the two head_dim-128 kernels compute the same function: same fp16 operands and softmax arithmetic.
    # The order of the row sum's fp32 additions differs (one rounding per tile and partial sum: a few
    # hundred tiles x 2^-24 relative bounds the difference of ln l near 1e-4), and rows of units that
    # the pair kernel runs as list shares (the split last wave) round P to fp16 relative to another
    # running offset: each kernel's P carries at most 2^-11 relative rounding, so their outputs differ by
    # at most 2 x 2^-11 x max |v| (max |out| stands in for max |v|)
    from int8_kv_cache_action_b200 import _nomas as N
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    prev = N.nomas_set_attn_kernel(2)
    try:
        a, la, _, _ = _run(cfg, inp, gc, mode)
        N.nomas_set_attn_kernel(1)
        b, lb, _, _ = _run(cfg, inp, gc, mode)
    finally:
        N.nomas_set_attn_kernel(prev)
    assert gc.status() == 0
    assert (a - b).abs().max().item() <= 2.0 ** -10 * max(1.0, b.abs().max().item())
    assert (la - lb).abs().max().item() <= 1e-4


def test_pair_kernel_split_last_wave_all_rows():
    # 480 x 832 with the pair kernel forced: 13 pairs x 16 heads = 208 units on 148 SMs, so the last 60
    # units (heads 11-15) each run as two list shares merged by the tail kernel; every row and head
    # against the oracle
    from int8_kv_cache_action_b200 import _nomas as N
    prev = N.nomas_set_attn_kernel(2)
    try:
        _check(CONFIGS["C1"], mode=0)
    finally:
        N.nomas_set_attn_kernel(prev)
