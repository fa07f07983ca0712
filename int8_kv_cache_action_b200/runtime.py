"""Convenience wrapper over the C ABI: a KV cache whose device buffers are torch allocations.

Only allocation (torch), stream selection and argument marshalling happen here; the quantise-append,
mask build and attention all run in libnomas's kernels.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import torch

from . import _nomas as N


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _bf16_strides(t: torch.Tensor) -> Tuple[int, int]:
    if t.dtype != torch.bfloat16 or t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("expected a bf16 [tokens, heads, head_dim] tensor with contiguous head_dim")
    return t.stride(0), t.stride(1)


def segment_text(n_frames: int, head_len: int, tails: Sequence[Tuple[int, int, int]] = ()):
    return N.make_segment_text(n_frames, head_len, [tuple(t) for t in tails])


def segment_text_of(seg) -> "N.nomas_segment_text":
    """From a workloads.SegmentText."""
    return segment_text(seg.n_frames, seg.head_len, [(t.len, t.f0, t.f1) for t in seg.tails])


class KVCache:
    """INT8 history ring + description-head store on one device (see include/nomas.h)."""

    def __init__(self, heads: int, head_dim: int, tokens_per_frame: int, window_frames: int,
                 capacity_frames: int, head_store_tokens: int, device="cuda", stream=None):
        self.dims = N.make_dims(heads, head_dim, tokens_per_frame, window_frames, capacity_frames,
                                head_store_tokens)
        total, sizes = N.nomas_kv_cache_bytes(self.dims)
        if total == 0:
            raise ValueError("invalid cache dimensions")
        self.device = torch.device(device)
        self.sizes = sizes
        self.bufs = [torch.empty(max(s, 16), dtype=torch.uint8, device=self.device) for s in sizes]
        self.handle = N.nomas_kv_cache_init(self.dims, [b.data_ptr() for b in self.bufs], _stream_handle(stream))
        self.H, self.D, self.T = heads, head_dim, tokens_per_frame
        self.C, self.HS = capacity_frames, head_store_tokens

    @classmethod
    def for_config(cls, cfg, device="cuda"):
        return cls(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                   cfg.head_store_tokens, device)

    def __del__(self, _destroy=N.nomas_kv_cache_destroy):
        # the destroy function is bound at definition time: module globals may already be gone when
        # the interpreter shuts down
        h = getattr(self, "handle", None)
        if h:
            _destroy(h)
            self.handle = None

    # ---- raw buffer views (for tests and diagnostics) -----------------------------------------
    def _view(self, i, dtype, shape):
        n = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
        return self.bufs[i][:n].view(dtype).view(*shape)

    def ring_k8(self):
        return self._view(N.NOMAS_BUF_K8, torch.int8, (self.H, self.C * self.T, self.D))

    def ring_v8(self):
        return self._view(N.NOMAS_BUF_V8, torch.int8, (self.H, self.C * self.T, self.D))

    def ring_ks(self):
        return self._view(N.NOMAS_BUF_KS, torch.float32, (self.H, self.C * self.T))

    def ring_vs(self):
        return self._view(N.NOMAS_BUF_VS, torch.float32, (self.H, self.C * self.T))

    def head_k8(self):
        return self._view(N.NOMAS_BUF_HK8, torch.int8, (self.H, self.HS, self.D))

    def head_v8(self):
        return self._view(N.NOMAS_BUF_HV8, torch.int8, (self.H, self.HS, self.D))

    def head_ks(self):
        return self._view(N.NOMAS_BUF_HKS, torch.float32, (self.H, self.HS))

    def head_vs(self):
        return self._view(N.NOMAS_BUF_HVS, torch.float32, (self.H, self.HS))

    # ---- operations ------------------------------------------------------------------------------
    def state(self):
        return N.nomas_kv_cache_state(self.handle)

    def append(self, k: Optional[torch.Tensor], v: Optional[torch.Tensor], n_frames: int,
               head_k: Optional[torch.Tensor] = None, head_v: Optional[torch.Tensor] = None, stream=None):
        ref = k if k is not None else head_k
        ts, hs = _bf16_strides(ref)
        for t in (v, head_k, head_v):
            if t is not None and _bf16_strides(t) != (ts, hs):
                raise ValueError("all K/V tensors of one append must share strides")
        head_len = 0 if head_k is None else head_k.shape[0]
        rc = N.nomas_kv_append(self.handle, k.data_ptr() if k is not None else 0,
                               v.data_ptr() if v is not None else 0, ts, hs, n_frames,
                               head_k.data_ptr() if head_k is not None else 0,
                               head_v.data_ptr() if head_v is not None else 0, head_len, _stream_handle(stream))
        N._check(rc, "nomas_kv_append")

    def mask_layout(self, seg, mode=N.NOMAS_MODE_DENSE, keep_frac=0.25):
        return N.nomas_mask_layout_query(self.handle, seg, mode, keep_frac)

    def build_mask(self, seg, mode=N.NOMAS_MODE_DENSE, keep_frac=0.25, q=None, kcur=None, mask_buf=None,
                   stream=None):
        lay = self.mask_layout(seg, mode, keep_frac)
        if mask_buf is None:
            mask_buf = torch.empty(lay["total_bytes"], dtype=torch.uint8, device=self.device)
        ts = hs = 8
        if mode == N.NOMAS_MODE_SPARSE:
            ts, hs = _bf16_strides(q)
            if _bf16_strides(kcur) != (ts, hs):
                raise ValueError("q and kcur must share strides")
        rc = N.nomas_mask_build(self.handle, seg, mode, keep_frac, q.data_ptr() if q is not None else 0,
                                kcur.data_ptr() if kcur is not None else 0, ts, hs, mask_buf.data_ptr(),
                                _stream_handle(stream))
        N._check(rc, "nomas_mask_build")
        return mask_buf, lay

    def workspace(self, seg):
        """A device buffer of the size nomas_attn_fwd needs for this segment (torch-allocated)."""
        n = N.nomas_attn_workspace_bytes(self.handle, seg)
        if n == 0:
            raise ValueError("invalid segment text")
        return torch.empty(n, dtype=torch.uint8, device=self.device)

    def attention(self, seg, mask_buf, q, kcur, vcur, ktxt, vtxt, softmax_scale=None, mode=N.NOMAS_MODE_DENSE,
                  keep_frac=0.25, out=None, lse=None, want_lse=False, workspace=None, stream=None):
        ts, hs = _bf16_strides(q)
        for t in (kcur, vcur) + ((ktxt, vtxt) if ktxt is not None and ktxt.shape[0] else ()):
            if _bf16_strides(t) != (ts, hs):
                raise ValueError("all bf16 inputs of one attention call must share strides")
        nq, H, D = q.shape
        if out is None:
            out = torch.empty((nq, H, D), dtype=torch.float32, device=self.device)
        if lse is None and want_lse:
            lse = torch.empty((H, nq), dtype=torch.float32, device=self.device)
        scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(D)
        has_txt = ktxt is not None and ktxt.shape[0] > 0
        if workspace is None:
            workspace = self.workspace(seg)
        rc = N.nomas_attn_fwd(self.handle, seg, mode, keep_frac, mask_buf.data_ptr(), q.data_ptr(),
                              kcur.data_ptr(), vcur.data_ptr(), ktxt.data_ptr() if has_txt else 0,
                              vtxt.data_ptr() if has_txt else 0, ts, hs, scale, out.data_ptr(),
                              lse.data_ptr() if lse is not None else 0, workspace.data_ptr(),
                              _stream_handle(stream))
        N._check(rc, "nomas_attn_fwd")
        return out, lse

    # ---- archive of evicted frames and selection of the retained history ------------------------
    def record_bytes(self) -> int:
        return N.nomas_kv_frame_record_bytes(self.dims)

    def retained(self):
        return N.nomas_kv_retained(self.handle)

    def evicted_by(self, n_frames: int):
        return N.nomas_kv_evicted_by(self.handle, n_frames)

    def archive(self, frame: int, record: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Copy retained `frame` into a host record (a pinned uint8 tensor, allocated when not given)."""
        if record is None:
            record = torch.empty(self.record_bytes(), dtype=torch.uint8).pin_memory()
        N._check(N.nomas_kv_archive(self.handle, frame, record.data_ptr(), _stream_handle(stream)), "nomas_kv_archive")
        return record

    def select(self, frames, records: Optional[dict] = None, stream=None):
        """Make `frames` the retained history (age order); records: frame -> host record for frames that
        are not retained now."""
        recs = None if records is None else [records[f].data_ptr() if f in records else 0 for f in frames]
        N._check(N.nomas_kv_select(self.handle, list(frames), recs, _stream_handle(stream)), "nomas_kv_select")

    def dequant(self, stream=None):
        st = self.state()
        n = st["history_tokens"]
        k = torch.empty((n, self.H, self.D), dtype=torch.float32, device=self.device)
        v = torch.empty_like(k)
        N._check(N.nomas_kv_dequant(self.handle, k.data_ptr(), v.data_ptr(), _stream_handle(stream)),
                 "nomas_kv_dequant")
        return k, v

    def status(self, stream=None) -> int:
        return N.nomas_device_status(self.handle, _stream_handle(stream))


def mask_views(mask_buf: torch.Tensor, lay: dict):
    """Class map, kept candidates and scores inside a mask buffer (device tensors)."""
    nqb, nt, H, keep, nc = lay["n_qblocks"], lay["n_tiles"], lay["heads"], lay["keep"], lay["n_cand"]
    cls = mask_buf[lay["off_class"]:lay["off_class"] + nqb * nt].view(torch.int8).view(nqb, nt)
    out = {"class": cls}
    if lay["mode"] == N.NOMAS_MODE_SPARSE:
        out["sel"] = mask_buf[lay["off_sel"]:lay["off_sel"] + H * nqb * keep * 4].view(torch.int32).view(H, nqb, keep)
        out["score"] = mask_buf[lay["off_score"]:lay["off_score"] + H * nqb * nc * 4].view(torch.float32).view(
            H, nqb, nc)
    nl, cap = lay["n_lists"], lay["list_cap"]
    out["count"] = mask_buf[lay["off_count"]:lay["off_count"] + nl * 4].view(torch.int32)
    out["list"] = mask_buf[lay["off_list"]:lay["off_list"] + nl * cap * 16].view(torch.int32).view(nl, cap, 4)
    return out


class Int8Linear:
    """A DiT linear layer with INT8 weights and float scales per output channel, computed in BF16
    (include/nomas.h): codes int8 [N][K] and scales fp32 [N] stay resident; every call dequantises the
    codes into a transient bf16 workspace and runs the tensor-core GEMM y = x W^T."""

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor):
        if codes.dtype != torch.int8 or codes.dim() != 2 or not codes.is_contiguous():
            raise ValueError("codes: contiguous int8 [N, K]")
        if scales.dtype != torch.float32 or scales.shape != (codes.shape[0],):
            raise ValueError("scales: float32 [N]")
        self.codes, self.scales = codes, scales
        self.n_out, self.k_in = codes.shape
        self.workspace = torch.empty(N.nomas_w8a16_workspace_bytes(self.n_out, self.k_in), dtype=torch.uint8,
                                     device=codes.device)
        self.status_word = torch.zeros(4, dtype=torch.int32, device=codes.device)

    @classmethod
    def from_weights(cls, w: torch.Tensor, stream=None) -> "Int8Linear":
        """Quantise bf16 weights [N, K] on the device."""
        if w.dtype != torch.bfloat16 or w.dim() != 2 or w.stride(1) != 1:
            raise ValueError("w: bf16 [N, K] with contiguous rows")
        n, k = w.shape
        codes = torch.empty((n, k), dtype=torch.int8, device=w.device)
        scales = torch.empty(n, dtype=torch.float32, device=w.device)
        N._check(N.nomas_w8_quantize(w.data_ptr(), n, k, w.stride(0), codes.data_ptr(), scales.data_ptr(),
                                     _stream_handle(stream)), "nomas_w8_quantize")
        return cls(codes, scales)

    def dequantized(self, stream=None) -> torch.Tensor:
        w = torch.empty((self.n_out, self.k_in), dtype=torch.bfloat16, device=self.codes.device)
        N._check(N.nomas_w8_dequant(self.codes.data_ptr(), self.scales.data_ptr(), self.n_out, self.k_in,
                                    w.data_ptr(), _stream_handle(stream)), "nomas_w8_dequant")
        return w

    def __call__(self, x: torch.Tensor, out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1 or x.shape[1] != self.k_in:
            raise ValueError("x: bf16 [M, K] with contiguous rows")
        m = x.shape[0]
        if out is None:
            out = torch.empty((m, self.n_out), dtype=out_dtype, device=x.device)
        dt = N.NOMAS_DTYPE_BF16 if out.dtype == torch.bfloat16 else N.NOMAS_DTYPE_F32
        N._check(N.nomas_w8a16_linear(x.data_ptr(), m, self.k_in, x.stride(0), self.codes.data_ptr(),
                                      self.scales.data_ptr(), self.n_out, out.data_ptr(), out.stride(0), dt,
                                      self.workspace.data_ptr(), self.status_word.data_ptr(),
                                      _stream_handle(stream)), "nomas_w8a16_linear")
        return out

    def status(self, stream=None) -> int:
        return N.nomas_status_read(self.status_word.data_ptr(), _stream_handle(stream))
