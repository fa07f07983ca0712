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


def test_forced_wait_limit_reports_timeout_and_context_stays_usable():
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
