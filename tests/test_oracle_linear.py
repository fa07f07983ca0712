"""Pins for the oracle's INT8-weight linear layer (reading in oracle/linear.py; fluxbbs.com
"单卡 4090 怎么做到的", first technique).  The bf16 rounding is checked against torch's conversion and
hand-derived ties, the dequantised weights against exact rational products, and the product's
orientation (y = x W^T) against a pure-Python triple loop."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.linear import abs_product_sum, dequantize_bf16, linear, quantize_weights, round_bf16
from oracle.quant import quantize


def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(round_bf16(x).view(np.uint32), want.view(np.uint32))


def test_round_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between bf16 1 and 1 + 2^-7: even mantissa (1) wins;
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even mantissa (1 + 2^-6) wins
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -20], dtype=np.float32)
    assert round_bf16(x).tolist() == [1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7]


def test_dequantised_weights_are_the_rounded_exact_products():
    rng = np.random.default_rng(1)
    codes = rng.integers(-127, 128, (7, 33)).astype(np.int8)
    scales = (rng.random(7) * 0.05 + 1e-4).astype(np.float32)
    got = dequantize_bf16(codes, scales)
    for n in range(7):
        for k in range(33):
            exact = Fraction(int(codes[n, k])) * Fraction(float(scales[n]))
            p32 = Fraction(float(np.float32(float(exact))))        # one fp32 rounding of the product
            b = round_bf16(np.array([float(p32)], dtype=np.float32))[0]
            assert Fraction(float(got[n, k])) == Fraction(float(b))
    # a power-of-two scale keeps every code exact
    assert np.array_equal(dequantize_bf16(codes, np.full(7, 0.25, np.float32)), codes.astype(np.float32) * 0.25)


def test_quantisation_is_per_output_row():
    rng = np.random.default_rng(2)
    w = torch.randn(5, 48, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).float().numpy()
    w[2] *= 1000.0                                  # one loud row does not change the others
    q, s = quantize_weights(w)
    for n in range(5):
        qn, sn = quantize(w[n:n + 1])
        assert np.array_equal(q[n], qn[0]) and s[n] == sn[0]
    assert np.all(np.abs(q).max(axis=1) == 127)
    assert rng is not None


def test_linear_orientation_against_a_triple_loop():
    rng = np.random.default_rng(4)
    M, N, K = 3, 4, 5
    x = rng.integers(-3, 4, (M, K)).astype(np.float32)
    codes = rng.integers(-127, 128, (N, K)).astype(np.int8)
    scales = np.full(N, 0.5, np.float32)
    y = linear(x, codes, scales)
    for m in range(M):
        for n in range(N):
            assert y[m, n] == sum(float(x[m, k]) * float(codes[n, k]) * 0.5 for k in range(K))
    assert np.array_equal(linear(x, codes, scales, rows=np.array([2, 0])), y[[2, 0]])
    assert np.array_equal(abs_product_sum(x, codes, scales), np.abs(x).astype(np.float64) @ (np.abs(codes) * 0.5).T)


@pytest.mark.parametrize("n", [1, 9])
def test_identity_weights_reproduce_the_input(n):
    K = 16
    codes = np.zeros((K, K), np.int8)
    np.fill_diagonal(codes, 127)
    scales = np.full(K, 1.0 / 127.0, np.float32)   # 127 * fp32(1/127) rounds to 1 in bf16
    x = torch.randn(n, K, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(linear(x, codes, scales), x.astype(np.float64))
