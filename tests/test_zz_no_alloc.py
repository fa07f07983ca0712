"""nomas_mask_build_static -- the mask/selection build for callers that cannot allocate device memory
(a host framework that owns the device pool and exposes no allocator to plugins, or a serving loop
where a cudaMalloc could synchronise the device).  Its pooled-mean scratch lives in a fixed device
array inside the library; this checks, through the C ABI, that two calls in a row give exactly what
nomas_mask_build gives (selection and scores bit for bit, the same attention output), and that a
request beyond the array's size is refused before anything runs.  Runs alone or after the other tests."""
import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, small_config
from tests.helpers import gpu_cache, to_device

pytestmark = pytest.mark.gpu


def _build(N, gc, seg, d, keep, static):
    lay = gc.mask_layout(seg, N.NOMAS_MODE_SPARSE, keep)
    buf = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    fn = N.nomas_mask_build_static if static else N.nomas_mask_build
    q, kc = d["q"], d["k_cur"]
    rc = fn(gc.handle, seg, N.NOMAS_MODE_SPARSE, keep, q.data_ptr(), kc.data_ptr(), q.stride(0), q.stride(1),
            buf.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, N.nomas_status_string(rc)
    return buf, lay


def test_static_scratch_matches_allocating_build_on_two_calls():
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import mask_views, segment_text_of
    cfgs = [CONFIGS["C3r"], small_config(tokens_per_frame=97, n_frames=5, prior_frames=(4, 4), window=5,
                                         head_dim=64)]
    for cfg in cfgs:                       # two calls in a row, different shapes: no state carries over
        inp = make_inputs(cfg)
        gc = gpu_cache(cfg, inp)
        d = to_device(inp)
        seg = segment_text_of(cfg.current)
        ref_buf, lay = _build(N, gc, seg, d, cfg.keep_frac, static=False)
        got_buf, _ = _build(N, gc, seg, d, cfg.keep_frac, static=True)
        torch.cuda.synchronize()
        a, b = mask_views(ref_buf, lay), mask_views(got_buf, lay)
        for key in ("class", "sel", "count"):
            assert torch.equal(a[key], b[key]), key
        assert np.array_equal(a["score"].cpu().numpy().view(np.uint32), b["score"].cpu().numpy().view(np.uint32))
        for li in range(lay["n_lists"]):
            n = int(a["count"][li])
            assert torch.equal(a["list"][li, :n], b["list"][li, :n])
        outs = []
        for buf in (ref_buf, got_buf):
            o, _ = gc.attention(seg, buf, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"],
                                mode=N.NOMAS_MODE_SPARSE, keep_frac=cfg.keep_frac)
            outs.append(o)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1])
        assert gc.status() == 0


def test_request_beyond_the_static_array_is_refused():
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import KVCache, segment_text
    # 16 heads x 128, 130 retained frames of 1024 tokens: 1040 + 8 candidates, 8 query blocks
    gc = KVCache(16, 128, 1024, 0, 131, 0)
    z = torch.zeros(130 * 1024, 16, 128, dtype=torch.bfloat16, device="cuda")
    gc.append(z, z, 130)
    q = torch.zeros(1024, 16, 128, dtype=torch.bfloat16, device="cuda")
    seg = segment_text(1, 0)
    lay = gc.mask_layout(seg, N.NOMAS_MODE_SPARSE, 0.25)
    assert 16 * (lay["n_qblocks"] + lay["n_cand"]) * 128 > N.NOMAS_STATIC_POOL_FLOATS
    buf = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    rc = N.nomas_mask_build_static(gc.handle, seg, N.NOMAS_MODE_SPARSE, 0.25, q.data_ptr(), q.data_ptr(),
                                   q.stride(0), q.stride(1), buf.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == N.NOMAS_ECAPACITY
    torch.cuda.synchronize()
    assert not buf.any()                   # refused before anything was enqueued
    assert gc.status() == 0
