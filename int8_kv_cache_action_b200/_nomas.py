"""ctypes binding of libnomas (include/nomas.h).  Argument marshalling only: every step of the path
runs in the library's CUDA kernels.  Functions keep the C names; device buffers are passed as
integer addresses (e.g. ``tensor.data_ptr()``) and streams as ``torch.cuda.Stream.cuda_stream``.

There is no fallback: if libnomas.so has not been built, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnomas.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libnomas.so is not built ({_LIB_PATH}); run `python -m int8_kv_cache_action_b200.build` "
                      "or __graft_entry__.build()")
lib = ctypes.CDLL(_LIB_PATH)

NOMAS_OK, NOMAS_EINVAL, NOMAS_ECAPACITY, NOMAS_ECUDA, NOMAS_ETIMEOUT, NOMAS_EDEVICE, NOMAS_EUNSUPPORTED, \
    NOMAS_ESTATE, NOMAS_ERANGE = 0, -1, -2, -3, -4, -5, -6, -7, -8
NOMAS_BUF_K8, NOMAS_BUF_V8, NOMAS_BUF_KS, NOMAS_BUF_VS, NOMAS_BUF_HK8, NOMAS_BUF_HV8, NOMAS_BUF_HKS, \
    NOMAS_BUF_HVS, NOMAS_BUF_ERR, NOMAS_NBUF = range(10)
NOMAS_MODE_DENSE, NOMAS_MODE_SPARSE, NOMAS_MODE_TEXT = 0, 1, 2
NOMAS_MAX_TAILS = 64
NOMAS_STATIC_POOL_FLOATS = 2 << 20
NOMAS_MAX_SPARSE_CANDIDATES = 8192
NOMAS_MAX_SELECT_FRAMES = 64
NOMAS_DTYPE_F32, NOMAS_DTYPE_BF16 = 0, 1

EXPORTED = ["nomas_kv_cache_bytes", "nomas_kv_cache_init", "nomas_kv_cache_destroy", "nomas_kv_cache_state",
            "nomas_kv_append", "nomas_mask_layout_query", "nomas_mask_bytes", "nomas_mask_build",
            "nomas_attn_fwd", "nomas_kv_dequant", "nomas_device_status", "nomas_status_string",
            "nomas_last_error", "nomas_mask_build_static", "nomas_attn_workspace_bytes",
            "nomas_set_wait_limit_ns", "nomas_set_text_split", "nomas_set_attn_kernel", "nomas_attn_prepare", "nomas_attn_run", "nomas_kv_frame_record_bytes",
            "nomas_kv_retained", "nomas_kv_evicted_by", "nomas_kv_archive", "nomas_kv_select",
            "nomas_w8_quantize", "nomas_w8_dequant", "nomas_linear_bf16", "nomas_w8a16_workspace_bytes",
            "nomas_w8a16_linear", "nomas_status_read"]


class nomas_cache_dims(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("window_frames", ctypes.c_int32), ("capacity_frames", ctypes.c_int32),
                ("head_store_tokens", ctypes.c_int32)]


class nomas_tail(ctypes.Structure):
    _fields_ = [("len", ctypes.c_int32), ("f0", ctypes.c_int32), ("f1", ctypes.c_int32)]


class nomas_segment_text(ctypes.Structure):
    _fields_ = [("n_frames", ctypes.c_int32), ("head_len", ctypes.c_int32), ("n_tails", ctypes.c_int32),
                ("tails", ctypes.POINTER(nomas_tail))]


class nomas_cache_state(ctypes.Structure):
    _fields_ = [("frames_appended", ctypes.c_int64), ("retained_frames", ctypes.c_int32),
                ("first_slot", ctypes.c_int32), ("history_tokens", ctypes.c_int64),
                ("head_tokens", ctypes.c_int64), ("segments", ctypes.c_int32), ("_pad", ctypes.c_int32)]


class nomas_mask_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ["mode", "head_dim", "heads", "n_qblocks", "n_tiles", "n_hist_tiles",
                                               "n_head_tiles", "n_cur_tiles", "n_text_tiles", "n_cand", "keep",
                                               "n_lists", "list_cap", "_pad"]] + \
               [(n, ctypes.c_int64) for n in ["history_tokens", "head_tokens", "n_query", "text_tokens"]] + \
               [(n, ctypes.c_size_t) for n in ["off_class", "off_sel", "off_score", "off_qmean", "off_kmean",
                                                "off_txtwin", "off_count", "off_list", "total_bytes"]]


_p = ctypes.c_void_p
_i32, _i64, _f32, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_sigs = {
    "nomas_kv_cache_bytes": (_sz, [ctypes.POINTER(nomas_cache_dims), ctypes.POINTER(_sz)]),
    "nomas_kv_cache_init": (ctypes.c_int, [ctypes.POINTER(_p), ctypes.POINTER(nomas_cache_dims),
                                           ctypes.POINTER(_p), _p]),
    "nomas_kv_cache_destroy": (ctypes.c_int, [_p]),
    "nomas_kv_cache_state": (ctypes.c_int, [_p, ctypes.POINTER(nomas_cache_state)]),
    "nomas_kv_append": (ctypes.c_int, [_p, _p, _p, _i64, _i64, _i32, _p, _p, _i32, _p]),
    "nomas_mask_layout_query": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32,
                                               ctypes.POINTER(nomas_mask_layout)]),
    "nomas_mask_bytes": (_sz, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32]),
    "nomas_mask_build": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32, _p, _p,
                                        _i64, _i64, _p, _p]),
    "nomas_mask_build_static": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32, _p,
                                               _p, _i64, _i64, _p, _p]),
    "nomas_attn_workspace_bytes": (_sz, [_p, ctypes.POINTER(nomas_segment_text)]),
    "nomas_attn_fwd": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32, _p, _p, _p,
                                      _p, _p, _p, _i64, _i64, _f32, _p, _p, _p, _p]),
    "nomas_attn_prepare": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), _p, _p, _p, _p, _i64, _i64,
                                          _p, _p]),
    "nomas_attn_run": (ctypes.c_int, [_p, ctypes.POINTER(nomas_segment_text), ctypes.c_int, _f32, _p, _p, _i64,
                                      _i64, _f32, _p, _p, _p, _p]),
    "nomas_kv_frame_record_bytes": (_sz, [ctypes.POINTER(nomas_cache_dims)]),
    "nomas_kv_retained": (ctypes.c_int, [_p, ctypes.POINTER(_i64), _i32, ctypes.POINTER(_i32)]),
    "nomas_kv_evicted_by": (ctypes.c_int, [_p, _i32, ctypes.POINTER(_i64), _i32, ctypes.POINTER(_i32)]),
    "nomas_kv_archive": (ctypes.c_int, [_p, _i64, _p, _p]),
    "nomas_kv_select": (ctypes.c_int, [_p, ctypes.POINTER(_i64), _i32, ctypes.POINTER(_p), _p]),
    "nomas_kv_dequant": (ctypes.c_int, [_p, _p, _p, _p]),
    "nomas_device_status": (ctypes.c_int, [_p, _p]),
    "nomas_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nomas_last_error": (ctypes.c_char_p, []),
    "nomas_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "nomas_set_text_split": (ctypes.c_int, [ctypes.c_int]),
    "nomas_set_attn_kernel": (ctypes.c_int, [ctypes.c_int]),
    "nomas_w8_quantize": (ctypes.c_int, [_p, _i64, _i64, _i64, _p, _p, _p]),
    "nomas_w8_dequant": (ctypes.c_int, [_p, _p, _i64, _i64, _p, _p]),
    "nomas_linear_bf16": (ctypes.c_int, [_p, _i64, _i64, _i64, _p, _i64, _i64, _p, _i64, ctypes.c_int, _p, _p]),
    "nomas_w8a16_workspace_bytes": (_sz, [_i64, _i64]),
    "nomas_w8a16_linear": (ctypes.c_int, [_p, _i64, _i64, _i64, _p, _p, _i64, _p, _i64, ctypes.c_int, _p, _p,
                                          _p]),
    "nomas_status_read": (ctypes.c_int, [_p, _p]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class NomasError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        extra = f" [{nomas_last_error()}]" if status == NOMAS_ECUDA else ""
        super().__init__(f"{what}: {nomas_status_string(status)} ({status}){extra}")


def _check(rc: int, what: str) -> None:
    if rc != NOMAS_OK:
        raise NomasError(rc, what)


def nomas_status_string(status: int) -> str:
    return lib.nomas_status_string(status).decode()


def nomas_last_error() -> str:
    return lib.nomas_last_error().decode()


def nomas_set_wait_limit_ns(limit_ns: int) -> int:
    """Set the attention kernel's bounded-wait limit (ns); returns the previous one."""
    return int(lib.nomas_set_wait_limit_ns(int(limit_ns)))


def nomas_set_text_split(shares: int) -> int:
    """Set the share count of text-row calls (0 = chosen per call, 1..16 forced); returns the previous one."""
    return int(lib.nomas_set_text_split(int(shares)))


def nomas_set_attn_kernel(which: int) -> int:
    """Choose the head_dim-128 attention kernel (0 = per call: block pairs for dense video rows, 1 = one
    block per CTA, 2 = block pairs); returns the previous choice."""
    return int(lib.nomas_set_attn_kernel(int(which)))


def make_dims(heads, head_dim, tokens_per_frame, window_frames, capacity_frames, head_store_tokens):
    return nomas_cache_dims(heads, head_dim, tokens_per_frame, window_frames, capacity_frames, head_store_tokens)


def make_segment_text(n_frames, head_len, tails=()):
    """tails: iterable of (len, f0, f1).  The returned structure keeps its tail array alive."""
    arr = (nomas_tail * max(1, len(tails)))(*[nomas_tail(*t) for t in tails])
    seg = nomas_segment_text(n_frames, head_len, len(tails), arr)
    seg._keep = arr
    return seg


def nomas_kv_cache_bytes(dims):
    sizes = (_sz * NOMAS_NBUF)()
    total = lib.nomas_kv_cache_bytes(ctypes.byref(dims), sizes)
    return total, list(sizes)


def nomas_kv_cache_init(dims, bufs, stream=0):
    h = _p()
    arr = (_p * NOMAS_NBUF)(*[b or None for b in bufs])
    _check(lib.nomas_kv_cache_init(ctypes.byref(h), ctypes.byref(dims), arr, stream or None), "nomas_kv_cache_init")
    return h.value


def nomas_kv_cache_destroy(handle):
    return lib.nomas_kv_cache_destroy(handle)


def nomas_kv_cache_state(handle):
    st = nomas_cache_state()
    _check(lib.nomas_kv_cache_state(handle, ctypes.byref(st)), "nomas_kv_cache_state")
    return {f: getattr(st, f) for f, _ in nomas_cache_state._fields_ if not f.startswith("_")}


def nomas_kv_append(handle, k, v, tok_stride, head_stride, n_frames, head_k, head_v, head_len, stream=0):
    return lib.nomas_kv_append(handle, k or None, v or None, tok_stride, head_stride, n_frames, head_k or None,
                               head_v or None, head_len, stream or None)


def nomas_mask_layout_query(handle, seg, mode, keep_frac=0.25):
    lay = nomas_mask_layout()
    _check(lib.nomas_mask_layout_query(handle, ctypes.byref(seg), mode, keep_frac, ctypes.byref(lay)),
           "nomas_mask_layout_query")
    return {f: getattr(lay, f) for f, _ in nomas_mask_layout._fields_ if not f.startswith("_")}


def nomas_mask_bytes(handle, seg, mode, keep_frac=0.25):
    return lib.nomas_mask_bytes(handle, ctypes.byref(seg), mode, keep_frac)


def nomas_mask_build(handle, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, stream=0):
    return lib.nomas_mask_build(handle, ctypes.byref(seg), mode, keep_frac, q or None, kcur or None, tok_stride,
                                head_stride, mask_buf, stream or None)


def nomas_mask_build_static(handle, seg, mode, keep_frac, q, kcur, tok_stride, head_stride, mask_buf, stream=0):
    return lib.nomas_mask_build_static(handle, ctypes.byref(seg), mode, keep_frac, q or None, kcur or None,
                                       tok_stride, head_stride, mask_buf, stream or None)


def nomas_attn_workspace_bytes(handle, seg):
    return lib.nomas_attn_workspace_bytes(handle, ctypes.byref(seg))


def nomas_attn_fwd(handle, seg, mode, keep_frac, mask_buf, q, kcur, vcur, ktxt, vtxt, tok_stride, head_stride,
                   softmax_scale, out, lse=0, workspace=0, stream=0):
    return lib.nomas_attn_fwd(handle, ctypes.byref(seg), mode, keep_frac, mask_buf, q, kcur, vcur, ktxt or None,
                              vtxt or None, tok_stride, head_stride, softmax_scale, out, lse or None,
                              workspace or None, stream or None)


def nomas_attn_prepare(handle, seg, kcur, vcur, ktxt, vtxt, tok_stride, head_stride, workspace, stream=0):
    return lib.nomas_attn_prepare(handle, ctypes.byref(seg), kcur, vcur, ktxt or None, vtxt or None, tok_stride,
                                  head_stride, workspace or None, stream or None)


def nomas_attn_run(handle, seg, mode, keep_frac, mask_buf, q, tok_stride, head_stride, softmax_scale, out, lse=0,
                   workspace=0, stream=0):
    return lib.nomas_attn_run(handle, ctypes.byref(seg), mode, keep_frac, mask_buf, q, tok_stride, head_stride,
                              softmax_scale, out, lse or None, workspace or None, stream or None)


def nomas_kv_frame_record_bytes(dims):
    return lib.nomas_kv_frame_record_bytes(ctypes.byref(dims))


def _frame_list(fn, handle, *args):
    cap = 4096
    buf = (_i64 * cap)()
    n = _i32()
    _check(fn(handle, *args, buf, cap, ctypes.byref(n)), fn.__name__)
    return [int(buf[i]) for i in range(n.value)]


def nomas_kv_retained(handle):
    """Retained history frames (global indices), age order."""
    return _frame_list(lib.nomas_kv_retained, handle)


def nomas_kv_evicted_by(handle, n_frames):
    """Retained frames an append of n_frames would drop, oldest first."""
    return _frame_list(lib.nomas_kv_evicted_by, handle, n_frames)


def nomas_kv_archive(handle, frame, record, stream=0):
    return lib.nomas_kv_archive(handle, frame, record, stream or None)


def nomas_kv_select(handle, frames, records=None, stream=0):
    """frames: global indices in age order; records: host addresses (0 for retained frames) or None."""
    n = len(frames)
    fr = (_i64 * max(1, n))(*frames)
    rec = None if records is None else (_p * max(1, n))(*[r or None for r in records])
    return lib.nomas_kv_select(handle, fr, n, rec, stream or None)


def nomas_kv_dequant(handle, k_out, v_out, stream=0):
    return lib.nomas_kv_dequant(handle, k_out, v_out, stream or None)


def nomas_device_status(handle, stream=0):
    return lib.nomas_device_status(handle, stream or None)


# ------------------------------------------------------------------------------------------------
# INT8-weight / BF16-compute linear layer
# ------------------------------------------------------------------------------------------------

def nomas_w8_quantize(w, n_out, k_in, ldw, codes, scales, stream=0):
    return lib.nomas_w8_quantize(w, n_out, k_in, ldw, codes, scales, stream or None)


def nomas_w8_dequant(codes, scales, n_out, k_in, w, stream=0):
    return lib.nomas_w8_dequant(codes, scales, n_out, k_in, w, stream or None)


def nomas_linear_bf16(x, m, k_in, ldx, w, n_out, ldw, y, ldy, y_dtype, status, stream=0):
    return lib.nomas_linear_bf16(x, m, k_in, ldx, w, n_out, ldw, y, ldy, y_dtype, status, stream or None)


def nomas_w8a16_workspace_bytes(n_out, k_in):
    return lib.nomas_w8a16_workspace_bytes(n_out, k_in)


def nomas_w8a16_linear(x, m, k_in, ldx, codes, scales, n_out, y, ldy, y_dtype, workspace, status, stream=0):
    return lib.nomas_w8a16_linear(x, m, k_in, ldx, codes, scales, n_out, y, ldy, y_dtype, workspace, status,
                                  stream or None)


def nomas_status_read(status, stream=0):
    return lib.nomas_status_read(status, stream or None)
