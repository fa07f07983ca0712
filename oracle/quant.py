"""INT8 quantiser with a per-(token, head) float scale.  Test infrastructure (see package header).

Follows fluxbbs.com "单卡 4090 怎么做到的", first technique: K/V are stored as
INT8 with float scale factors and dequantised back to BF16 for compute;
quantisation happens on the storage side only.  The pages give no formula.
Reading adopted (symmetric absmax, the plainest form of "INT8 + float scale"):

    a = max_c |x_c|              (fp32, exact)
    s = a / 127                  (fp32 IEEE division, round to nearest even)
    q_c = clamp(rint(x_c / s), -127, 127)   (fp32 IEEE division, rint = half-even)
    a == 0  ->  s = 0, q = 0

The division is by the stored fp32 scale, so q * s is the dequantised value.
Everything is done in numpy float32 (IEEE-correct division, np.rint is
round-half-even), so the result is exactly defined.
"""
from __future__ import annotations

import numpy as np

_F127 = np.float32(127.0)


def quantize(x: np.ndarray):
    """Quantise the last axis of `x` (float32 holding exact bf16 values).

    Returns (q int8 same shape, s float32 shape[:-1]).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.max(np.abs(x), axis=-1)
    s = (a / _F127).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    y = (x / safe[..., None]).astype(np.float32)
    q = np.clip(np.rint(y), -127, 127)
    q = np.where((s > 0)[..., None], q, 0).astype(np.int8)
    return q, s


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Exact dequantised values in float64: q * s (q <= 127 in magnitude, s fp32)."""
    return q.astype(np.float64) * s.astype(np.float64)[..., None]
