"""The attention's supported input range, through the C ABI.

The tensor-core operands are fp16 (fluxbbs.com "单卡 4090 怎么做到的": cached K/V are dequantised for
bf16-class compute; this library feeds the MMAs fp16, which holds every bf16 value of magnitude in
[2^-14, 65504] exactly).  Inside that range the output must meet the usual tolerance against the fp64
oracle, also with extreme magnitudes mixed in; outside it (a value that rounds to an fp16 infinity, a
NaN, or a cached value scale too large for P * scale to stay in fp16) the call must record
NOMAS_ERANGE in the device error word without faulting, and the next call on the same context must be
exact again.  A query holding an infinity also passes through the sparse selection, whose ranking
puts the resulting NaN scores last, bit for bit as the oracle does.
"""
import math

import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200 import _nomas as N
from int8_kv_cache_action_b200.runtime import mask_views, segment_text_of
from int8_kv_cache_action_b200.workloads import make_inputs, small_config
from tests.helpers import (TOL_MAX_ABS, TOL_MEAN_REL, attention_errors, f32, gpu_cache, oracle_cache,
                           to_device)

pytestmark = pytest.mark.gpu

BF16_MAX_IN_RANGE = 65280.0      # largest bf16 below 65504
BF16_OUT_OF_RANGE = 65536.0      # smallest bf16 above 65504: rounds to an fp16 infinity


def _cfg():
    return small_config(tokens_per_frame=100, n_frames=3, prior_frames=(3, 3), window=4)


def _attend(gc, cfg, inp, mode=0):
    seg = segment_text_of(cfg.current)
    d = to_device(inp)
    buf, _ = gc.build_mask(seg, mode, cfg.keep_frac, d["q"], d["k_cur"])
    out, _ = gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"], mode=mode,
                          keep_frac=cfg.keep_frac)
    torch.cuda.synchronize()
    return out


def _oracle(cfg, inp, oc):
    from oracle import attention as att
    return att.attention(oc, f32(inp.q), f32(inp.k_cur), f32(inp.v_cur), f32(inp.k_txt), f32(inp.v_txt),
                         cfg.current, 1.0 / math.sqrt(cfg.head_dim))[0]


def _extreme_inputs(cfg):
    inp = make_inputs(cfg)
    # keys with one channel at the largest in-range magnitude: one-hot scores for the rows whose query
    # channel has the matching sign, no effect on the others
    for t, c, sgn in ((3, 5, 1.0), (150, 77, -1.0), (299, 5, 1.0)):
        inp.k_cur[t, 0, c] = sgn * BF16_MAX_IN_RANGE
    inp.k_txt[45, 1, 9] = -BF16_MAX_IN_RANGE           # a key of an action tail
    inp.q[10, 1, 40] = BF16_MAX_IN_RANGE               # one query row with a huge channel
    # tiny magnitudes 2^-14 .. 2^-20 on whole tokens of q, v and the history source
    for i, e in enumerate(range(14, 21)):
        s = 2.0 ** -e
        inp.q[20 + i] = (inp.q[20 + i].float() * s).bfloat16()
        inp.v_cur[30 + 7 * i] = (inp.v_cur[30 + 7 * i].float() * s).bfloat16()
        inp.v_txt[i] = (inp.v_txt[i].float() * s).bfloat16()
        inp.prior[1].v[11 * i] = (inp.prior[1].v[11 * i].float() * s).bfloat16()
        inp.prior[1].k[13 * i] = (inp.prior[1].k[13 * i].float() * s).bfloat16()
    return inp


def test_extreme_in_range_magnitudes_match_oracle():
    cfg = _cfg()
    inp = _extreme_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    out = _attend(gc, cfg, inp)
    assert gc.status() == N.NOMAS_OK
    ref = _oracle(cfg, inp, oracle_cache(cfg, inp))
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    mx, mr = attention_errors(got, ref)
    assert mx <= TOL_MAX_ABS and mr <= TOL_MEAN_REL, (mx, mr)


def test_large_cached_values_within_the_scale_limit():
    # a history value of 1.0e5 gives a value scale of 787 (<= 65504 / 64): supported.  The absolute
    # bound is stated for unit-scale outputs, so it is applied relative to each row's output scale.
    cfg = _cfg()
    inp = make_inputs(cfg)
    inp.prior[1].v[40, 1, 3] = 1.0e5
    gc = gpu_cache(cfg, inp)
    out = _attend(gc, cfg, inp)
    assert gc.status() == N.NOMAS_OK
    ref = _oracle(cfg, inp, oracle_cache(cfg, inp))
    got = out.cpu().numpy().astype(np.float64)
    row_scale = np.maximum(1.0, np.abs(ref).max(axis=2, keepdims=True))
    assert (np.abs(got - ref) / row_scale).max() <= TOL_MAX_ABS
    assert np.abs(got - ref).sum() / np.abs(ref).sum() <= TOL_MEAN_REL


@pytest.mark.parametrize("where,value", [("q", BF16_OUT_OF_RANGE), ("k_cur", -BF16_OUT_OF_RANGE),
                                         ("v_cur", BF16_OUT_OF_RANGE), ("k_txt", float("inf")),
                                         ("v_txt", float("nan")), ("hist_v", 2.0e5)])
def test_out_of_range_input_reports_erange_and_context_stays_usable(where, value):
    cfg = _cfg()
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    clean = _attend(gc, cfg, inp)
    assert gc.status() == N.NOMAS_OK
    if where == "hist_v":
        # appended after the clean run: a (token, head) absmax of 2e5 gives a value scale above 1023.5
        bad_k = inp.k_cur[:cfg.tokens_per_frame].clone()
        bad_v = inp.v_cur[:cfg.tokens_per_frame].clone()
        bad_v[7, 0, 0] = value
        gc.append(bad_k.cuda(), bad_v.cuda(), 1)
        _attend(gc, cfg, inp)
        assert gc.status() == N.NOMAS_ERANGE
        return
    t = getattr(inp, where)
    saved = t[5, 1, 17].clone()
    t[5, 1, 17] = value
    _attend(gc, cfg, inp)
    assert gc.status() == N.NOMAS_ERANGE
    assert gc.status() == N.NOMAS_OK           # read-and-clear
    t[5, 1, 17] = saved
    again = _attend(gc, cfg, inp)
    assert gc.status() == N.NOMAS_OK
    assert torch.equal(again, clean)


def test_inf_query_sparse_selection_matches_oracle_and_attention_reports_range():
    from oracle import select as sel
    cfg = small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4, keep_frac=0.25)
    inp = make_inputs(cfg)
    # query block 1 of head 0: channel means +inf and -inf, so each score is +-inf or, where the two
    # candidate channels have the same sign, inf - inf = NaN
    inp.q[130, 0, 3] = float("inf")
    inp.q[131, 0, 4] = float("-inf")
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    q, kc = inp.q.cuda(), inp.k_cur.cuda()
    buf, lay = gc.build_mask(segment_text_of(cfg.current), N.NOMAS_MODE_SPARSE, cfg.keep_frac, q, kc)
    mv = mask_views(buf, lay)
    hk8, hks, _, _ = oc.history()
    want_sel, want_score = sel.select(f32(inp.q), hk8, hks, f32(inp.k_cur), cfg.keep_frac)
    got_score = mv["score"].cpu().numpy()
    nan = np.isnan(want_score)
    assert nan.any() and np.array_equal(np.isnan(got_score), nan)
    assert np.array_equal(got_score[~nan].view(np.uint32), want_score[~nan].view(np.uint32))
    assert np.array_equal(mv["sel"].cpu().numpy(), want_sel)
    assert gc.status() == N.NOMAS_OK               # the selection itself has nothing to report
    _attend(gc, cfg, inp, mode=N.NOMAS_MODE_SPARSE)
    assert gc.status() == N.NOMAS_ERANGE
