"""CPU checks of the C ABI library: it loads, exports every declared entry point, and its host-only
logic (sizes, argument validation, status strings) behaves as documented.  No kernel is launched."""
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nomas.h")


@pytest.fixture(scope="module")
def N():
    from int8_kv_cache_action_b200 import build
    build.build()
    from int8_kv_cache_action_b200 import _nomas
    return _nomas


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(nomas_[a-z_0-9]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    d = _declared()
    for name in ["nomas_kv_append", "nomas_mask_build", "nomas_attn_fwd", "nomas_kv_cache_bytes",
                 "nomas_kv_cache_init", "nomas_kv_dequant", "nomas_device_status", "nomas_status_string"]:
        assert name in d


def test_library_exports_every_declared_symbol(N):
    for name in _declared():
        assert hasattr(N.lib, name), name
    assert sorted(N.EXPORTED) == _declared()


def test_exports_only_the_abi():
    import subprocess
    from int8_kv_cache_action_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True).stdout
    names = sorted(l.split()[-1] for l in out.splitlines() if l.strip())
    assert names == _declared()


def test_cache_sizes(N):
    d = N.make_dims(16, 128, 880, 18, 18, 768)
    total, sizes = N.nomas_kv_cache_bytes(d)
    rows = 18 * 880
    assert sizes[N.NOMAS_BUF_K8] == 16 * rows * 128 and sizes[N.NOMAS_BUF_KS] == 16 * rows * 4
    assert sizes[N.NOMAS_BUF_HK8] == 16 * 768 * 128 and sizes[N.NOMAS_BUF_ERR] == 16
    assert total == sum(sizes)
    for bad in [N.make_dims(16, 96, 880, 18, 18, 0), N.make_dims(0, 128, 880, 18, 18, 0),
                N.make_dims(16, 128, 880, 18, 17, 0), N.make_dims(16, 128, 0, 18, 18, 0)]:
        assert N.nomas_kv_cache_bytes(bad)[0] == 0


def test_invalid_arguments_fail_before_any_cuda_call(N):
    import ctypes
    d = N.make_dims(2, 64, 24, 4, 4, 48)
    h = ctypes.c_void_p()
    assert N.lib.nomas_kv_cache_init(ctypes.byref(h), ctypes.byref(d), None, None) == N.NOMAS_EINVAL
    arr = (ctypes.c_void_p * N.NOMAS_NBUF)()
    assert N.lib.nomas_kv_cache_init(ctypes.byref(h), ctypes.byref(d), arr, None) == N.NOMAS_EINVAL
    assert N.nomas_kv_append(None, 0, 0, 128, 64, 1, 0, 0, 0) == N.NOMAS_EINVAL
    seg = N.make_segment_text(2, 16, [(8, 0, 1)])
    assert N.nomas_mask_bytes(None, seg, 0, 0.25) == 0
    assert N.nomas_device_status(None) == N.NOMAS_EINVAL


def test_status_strings(N):
    assert N.nomas_status_string(0) == "ok"
    assert N.nomas_status_string(N.NOMAS_ETIMEOUT) == "device wait timed out"
    assert N.nomas_status_string(12345) == "unknown status"


def test_prompt_times_to_latent_windows():
    from int8_kv_cache_action_b200.text_layout import action_windows, segment_frames
    with open(os.path.join(ROOT, "tests", "golden", "prompt_two_segments.json")) as f:
        g = json.load(f)
    assert [segment_frames(s) for s in g["segments"]] == g["_expected_n_frames"]
    assert [[list(w) for w in action_windows(s)] for s in g["segments"]] == g["_expected_windows"]


def test_frame_record_bytes(N):
    # one archived frame: K and V codes (H*T*D int8 each) then K and V scales (H*T fp32 each)
    d = N.make_dims(16, 128, 880, 18, 18, 768)
    assert N.nomas_kv_frame_record_bytes(d) == 2 * 16 * 880 * 128 + 2 * 16 * 880 * 4
    assert N.nomas_kv_frame_record_bytes(N.make_dims(16, 96, 880, 18, 18, 768)) == 0   # invalid head_dim


def test_linear_host_checks_without_a_device(N):
    # every rejected argument returns before any CUDA call, so this runs without a GPU
    assert N.nomas_w8a16_workspace_bytes(2048, 6144) == 2048 * 6144 * 2
    assert N.nomas_w8a16_workspace_bytes(0, 8) == 0
    a = 0x10000                                          # 16-byte aligned stand-in addresses (never read)
    ok = dict(x=a, m=4, k_in=32, ldx=32, codes=a, scales=a, n_out=16, y=a, ldy=16, y_dtype=N.NOMAS_DTYPE_F32,
              workspace=a, status=a)

    def call(**kw):
        v = dict(ok, **kw)
        return N.nomas_w8a16_linear(v["x"], v["m"], v["k_in"], v["ldx"], v["codes"], v["scales"], v["n_out"],
                                    v["y"], v["ldy"], v["y_dtype"], v["workspace"], v["status"])
    for bad in (dict(k_in=30, ldx=30), dict(ldx=16), dict(m=0), dict(n_out=0), dict(x=a + 4), dict(y=0),
                dict(y_dtype=2), dict(status=0), dict(ldy=12), dict(codes=0), dict(workspace=a + 8)):
        assert call(**bad) == N.NOMAS_EINVAL, bad
    assert N.nomas_linear_bf16(a, 4, 32, 32, a, 16, 24, a, 16, 0, a) == N.NOMAS_EINVAL   # W pitch not a multiple of 8
    assert N.nomas_w8_dequant(a, a, 16, 12, a) == N.NOMAS_EINVAL                         # K not a multiple of 8
    assert N.nomas_w8_quantize(0, 16, 32, 32, a, a) == N.NOMAS_EINVAL
    assert N.nomas_status_read(0) == N.NOMAS_EINVAL


def test_text_split_setting_round_trips(N):
    # host-side setting only: 0 = chosen per call, 1..16 forced, anything else back to 0
    prev = N.nomas_set_text_split(3)
    try:
        assert N.nomas_set_text_split(17) == 3
        assert N.nomas_set_text_split(16) == 0
        assert N.nomas_set_text_split(-1) == 16
    finally:
        N.nomas_set_text_split(prev)


def test_attn_kernel_setting_round_trips(N):
    # host-only setter: no GPU needed
    prev = N.nomas_set_attn_kernel(1)
    try:
        assert N.nomas_set_attn_kernel(2) == 1
        assert N.nomas_set_attn_kernel(7) == 2
        assert N.nomas_set_attn_kernel(0) == 0
        assert N.nomas_set_attn_kernel(-3) == 0
    finally:
        N.nomas_set_attn_kernel(prev)
