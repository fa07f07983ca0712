"""INT8-weight / BF16-compute linear layer of the DiT.  Test infrastructure (see package header).

Follows fluxbbs.com "单卡 4090 怎么做到的", first technique: model weights (like the cached keys and
values) are stored as INT8 with float scale factors and dequantised back to BF16 at compute time;
the DiT's linear layers compute in BF16.  The pages give no formula and no scale granularity.
Readings adopted (the plainest ones the rest supports):

    scales per output channel: row n of W [N][K] is one vector for the K/V quantiser of
    oracle.quant (s_n = fp32(absmax / 127), codes rint(w / s_n) half-even)
    dequantised weight   w_nk = bf16(RN(fp32(q_nk * s_n)))   (one fp32 product, rounded to bf16
                                                              half-even)
    output               y_mn = sum_k x_mk * w_nk            (x bf16; exact sum here, in fp64)

The device accumulates in fp32; the tests bound the difference by the fp32 accumulation error.
"""
from __future__ import annotations

import numpy as np

from oracle.quant import quantize


def quantize_weights(w: np.ndarray):
    """w: float32 [N][K] holding bf16 values.  Returns (codes int8 [N][K], scales float32 [N])."""
    return quantize(np.asarray(w, dtype=np.float32))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding bf16 values.
    Finite inputs only."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32)


def dequantize_bf16(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """bf16(RN(fp32(code * scale))) for every weight, as float32."""
    prod = (codes.astype(np.float32) * np.asarray(scales, dtype=np.float32)[:, None]).astype(np.float32)
    return round_bf16(prod)


def linear(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, rows=None) -> np.ndarray:
    """y = x W^T with W the dequantised bf16 weights, in fp64.  x: float32 [M][K] (bf16 values).
    rows: optional index array of the rows of x to compute."""
    w = dequantize_bf16(codes, scales).astype(np.float64)
    xs = np.asarray(x, dtype=np.float64)
    if rows is not None:
        xs = xs[rows]
    return xs @ w.T


def abs_product_sum(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, rows=None) -> np.ndarray:
    """sum_k |x_mk| |w_nk| per output element, the scale of the fp32 accumulation error bound."""
    w = np.abs(dequantize_bf16(codes, scales).astype(np.float64))
    xs = np.abs(np.asarray(x, dtype=np.float64))
    if rows is not None:
        xs = xs[rows]
    return xs @ w.T
