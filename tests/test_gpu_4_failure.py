"""Failure detection on the GPU without a fault: with the attention kernel's wait limit forced to 0,
a wait that its first poll does not satisfy gives up at once, the kernel records NOMAS_ETIMEOUT in the
device error word and every role unwinds (in-flight copies and MMAs complete, TMEM is released).
The host reads the status, the limit is restored, and the next call on the same context is correct."""
import pytest
import torch

from int8_kv_cache_action_b200 import _nomas as N
from int8_kv_cache_action_b200.workloads import make_inputs, small_config
from tests.helpers import gpu_cache, to_device

pytestmark = pytest.mark.gpu


def _attention(gc, cfg, d, seg):
    buf, _ = gc.build_mask(seg)
    out, _ = gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"])
    return out


def test_forced_wait_limit_reports_timeout_and_context_stays_usable(attn_kernel):
    from int8_kv_cache_action_b200.runtime import segment_text_of
    cfg = small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4)
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    d = to_device(inp)
    seg = segment_text_of(cfg.current)
    ref = _attention(gc, cfg, d, seg)
    assert gc.status() == N.NOMAS_OK
    prev = N.nomas_set_wait_limit_ns(0)
    try:
        _attention(gc, cfg, d, seg)
        torch.cuda.synchronize()
        st = gc.status()
    finally:
        N.nomas_set_wait_limit_ns(prev)
    assert st == N.NOMAS_ETIMEOUT
    assert gc.status() == N.NOMAS_OK          # read-and-clear
    again = _attention(gc, cfg, d, seg)
    torch.cuda.synchronize()
    assert gc.status() == N.NOMAS_OK
    assert torch.equal(again, ref)


def test_forced_wait_limit_in_append_reports_timeout_and_the_next_append_is_exact():
    # The append kernel's consumers wait for each chunk's TMA copy with the same bounded wait: with the
    # limit at 0 the first wait that is not yet satisfied gives up, the kernel records NOMAS_ETIMEOUT
    # and unwinds (the producer lets its copies land).  The ring contents of that call are undefined;
    # a fresh cache on the same context then appends bit for bit as the oracle does.
    import numpy as np
    from int8_kv_cache_action_b200.runtime import KVCache
    from tests.helpers import f32, oracle_cache
    cfg = small_config(tokens_per_frame=880, n_frames=2, prior_frames=(6,), window=4, heads=16)
    inp = make_inputs(cfg)
    kv = inp.prior[0]
    gc = KVCache.for_config(cfg)
    prev = N.nomas_set_wait_limit_ns(0)
    try:
        gc.append(kv.k.cuda(), kv.v.cuda(), 6, kv.head_k.cuda(), kv.head_v.cuda())
        torch.cuda.synchronize()
        st = gc.status()
    finally:
        N.nomas_set_wait_limit_ns(prev)
    assert st == N.NOMAS_ETIMEOUT
    fresh = gpu_cache(cfg, inp)
    assert fresh.status() == N.NOMAS_OK
    oc = oracle_cache(cfg, inp)
    T = cfg.tokens_per_frame
    for g in oc.retained_frames():
        s = slice((g % oc.C) * T, (g % oc.C + 1) * T)
        assert np.array_equal(fresh.ring_k8().cpu().numpy()[:, s], oc.k8[:, s])
        assert np.array_equal(fresh.ring_vs().cpu().numpy()[:, s].view(np.uint32), oc.vs[:, s].view(np.uint32))


def test_forced_wait_limit_in_sparse_pooling_reports_timeout_and_the_next_build_is_exact():
    # The sparse selection's pooling kernel waits for its TMA and bulk copies with the same bounded
    # wait; with the limit at 0 the build records NOMAS_ETIMEOUT, its producer lets the copies land,
    # and a rebuild on the same context reproduces the first build's selection and lists bit for bit.
    from int8_kv_cache_action_b200.runtime import mask_views, segment_text_of
    cfg = small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4)
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    d = to_device(inp)
    seg = segment_text_of(cfg.current)
    buf, lay = gc.build_mask(seg, N.NOMAS_MODE_SPARSE, 0.25, d["q"], d["k_cur"])
    torch.cuda.synchronize()
    assert gc.status() == N.NOMAS_OK
    ref = {k: v.clone() for k, v in mask_views(buf, lay).items() if k in ("sel", "score", "count", "list")}
    prev = N.nomas_set_wait_limit_ns(0)
    try:
        gc.build_mask(seg, N.NOMAS_MODE_SPARSE, 0.25, d["q"], d["k_cur"])
        torch.cuda.synchronize()
        st = gc.status()
    finally:
        N.nomas_set_wait_limit_ns(prev)
    assert st == N.NOMAS_ETIMEOUT
    buf2, lay2 = gc.build_mask(seg, N.NOMAS_MODE_SPARSE, 0.25, d["q"], d["k_cur"])
    torch.cuda.synchronize()
    assert gc.status() == N.NOMAS_OK
    mv = mask_views(buf2, lay2)
    for k in ("sel", "score", "count"):
        assert torch.equal(mv[k], ref[k]), k
    for i, n in enumerate(ref["count"].tolist()):     # list entries past a list's count are unused
        assert torch.equal(mv["list"][i, :n], ref["list"][i, :n])
