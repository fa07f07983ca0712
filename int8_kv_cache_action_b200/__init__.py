"""B200-native action-aware segment-causal attention over an INT8 KV cache (Hy-Nomas hot path).

The compute path is libnomas.so (hand-written sm_100a kernels behind the C ABI in
include/nomas.h); this package is its thin ctypes binding (`_nomas`), a convenience wrapper that
owns torch-allocated device buffers (`runtime.KVCache`), host-side text-layout helpers
(`text_layout`) and the seeded synthetic workloads (`workloads`).
"""
__all__ = ["workloads", "text_layout"]
