"""Pins for the oracle's text query rows (the text stream of the double-stream joint attention; the
reading is stated in oracle/visibility.py): a token-level brute force of who sees whom, the reduction
of the attention to torch fp64 SDPA under that mask, and the invariances the rule implies."""
import math

import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import make_inputs, small_config
from oracle import attention as att
from oracle import visibility as vis
from oracle.quant import dequantize
from oracle.ring import OracleCache


def _f32(t):
    return t.float().numpy()


def _cache(cfg, inp):
    c = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                    cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        c.append(_f32(kv.k), _f32(kv.v), seg.n_frames, None if kv.head_k is None else _f32(kv.head_k),
                 None if kv.head_v is None else _f32(kv.head_v))
    return c


def _brute(cfg, lh, lp):
    """Every key token labelled by what it is; every text row decided by the rule in words."""
    T, seg = cfg.tokens_per_frame, cfg.current
    keys = [("history",)] * lh + [("earlier head",)] * lp
    keys += [("video", i // T) for i in range(cfg.n_query)]
    keys += [("head",)] * seg.head_len
    for a, tail in enumerate(seg.tails):
        keys += [("tail", a, tail.f0, tail.f1)] * tail.len
    rows = [("head",)] * seg.head_len
    for a, tail in enumerate(seg.tails):
        rows += [("tail", a, tail.f0, tail.f1)] * tail.len
    m = np.zeros((len(rows), len(keys)), bool)
    for i, r in enumerate(rows):
        for j, k in enumerate(keys):
            if k[0] in ("history", "earlier head", "head"):
                m[i, j] = True                                   # context every row of the segment sees
            elif k[0] == "video":
                m[i, j] = r[0] == "head" or r[2] <= k[1] < r[3]  # a tail row: only frames in its window
            else:                                                # an action tail key
                m[i, j] = r[0] == "tail" and max(r[2], k[2]) < min(r[3], k[3])   # windows share a frame
    return m


CFGS = [
    small_config(tokens_per_frame=10, n_frames=4, tails=((3, 0, 1), (2, 1, 3), (2, 3, 4))),
    small_config(tokens_per_frame=33, n_frames=5, window=0, prior_frames=(2, 3),
                 tails=((20, 0, 2), (7, 2, 2), (30, 1, 5), (9, 4, 5))),          # an empty window too
    small_config(tokens_per_frame=25, n_frames=3, head_len=0, tails=((11, 0, 3),)),  # no head
]


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: f"T{c.tokens_per_frame}_F{c.current.n_frames}")
def test_text_row_mask_against_brute_force(cfg):
    inp = make_inputs(cfg)
    c = _cache(cfg, inp)
    got = vis.text_query_mask(c.history_tokens(), c.head_used, cfg.n_query, cfg.tokens_per_frame, cfg.current)
    assert np.array_equal(got, _brute(cfg, c.history_tokens(), c.head_used))


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: f"T{c.tokens_per_frame}_F{c.current.n_frames}")
def test_text_rows_reduce_to_torch_sdpa(cfg):
    g = torch.Generator().manual_seed(3)
    inp = make_inputs(cfg)
    q_txt = torch.randn(inp.k_txt.shape, generator=g).bfloat16()
    c = _cache(cfg, inp)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    out, lse = att.attention_text(c, _f32(q_txt), _f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt),
                                  _f32(inp.v_txt), cfg.current, scale)
    mask = torch.from_numpy(_brute(cfg, c.history_tokens(), c.head_used))
    hk8, hks, hv8, hvs = c.history()
    pk8, pks, pv8, pvs = c.prior_heads()
    for h in range(cfg.heads):
        K = torch.cat([torch.from_numpy(dequantize(hk8[h], hks[h])), torch.from_numpy(dequantize(pk8[h], pks[h])),
                       inp.k_cur[:, h].double(), inp.k_txt[:, h].double()])
        V = torch.cat([torch.from_numpy(dequantize(hv8[h], hvs[h])), torch.from_numpy(dequantize(pv8[h], pvs[h])),
                       inp.v_cur[:, h].double(), inp.v_txt[:, h].double()])
        Q = q_txt[:, h].double()
        live = mask.any(dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(Q[live][None], K[None], V[None],
                                                               attn_mask=mask[live][None], scale=scale)[0]
        assert np.allclose(out[live.numpy(), h], ref.numpy(), rtol=0, atol=1e-12)
        ref_lse = torch.logsumexp((Q @ K.T * scale).masked_fill(~mask, -float("inf")), dim=1)
        assert np.allclose(lse[h, live.numpy()], ref_lse[live].numpy(), rtol=0, atol=1e-12)
        assert np.all(out[~live.numpy(), h] == 0) and np.all(lse[h, ~live.numpy()] == -np.inf)


def test_head_rows_never_see_tails_and_tail_rows_stay_in_their_window():
    cfg = CFGS[1]
    g = torch.Generator().manual_seed(4)
    inp = make_inputs(cfg)
    q_txt = _f32(torch.randn(inp.k_txt.shape, generator=g).bfloat16())
    c = _cache(cfg, inp)
    args = lambda kc, vc, kt, vt: (c, q_txt, kc, vc, kt, vt, cfg.current, 0.1)
    base, _ = att.attention_text(*args(_f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt), _f32(inp.v_txt)))
    hl, T = cfg.current.head_len, cfg.tokens_per_frame
    # change every action tail's K and V: head rows are bitwise unchanged, tail rows change
    kt, vt = _f32(inp.k_txt).copy(), _f32(inp.v_txt).copy()
    kt[hl:] *= -2.0
    vt[hl:] += 3.0
    pert, _ = att.attention_text(*args(_f32(inp.k_cur), _f32(inp.v_cur), kt, vt))
    assert np.array_equal(pert[:hl], base[:hl]) and np.abs(pert[hl:] - base[hl:]).max() > 1e-3
    # change the video of frames 0 and 1: rows of the tail with window [4, 5) are bitwise unchanged
    kc, vc = _f32(inp.k_cur).copy(), _f32(inp.v_cur).copy()
    vc[:2 * T] += 5.0
    kc[:2 * T] *= 3.0
    pert, _ = att.attention_text(*args(kc, vc, _f32(inp.k_txt), _f32(inp.v_txt)))
    last = slice(hl + 20 + 7 + 30, hl + 20 + 7 + 30 + 9)
    assert np.array_equal(pert[last], base[last]) and np.abs(pert[:hl] - base[:hl]).max() > 1e-3
