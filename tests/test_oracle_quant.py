"""Pins for the oracle's INT8 quantiser (fp32, absmax/127, round-half-even)."""
import os

import numpy as np
import pytest
import torch

from oracle.quant import quantize, dequantize

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_cases.txt")


def _bf16(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b, c = [p.strip() for p in line.split("|")]
            rows.append(([float(v) for v in a.split()], [int(v) for v in b.split()], int(c, 16)))
    return rows


@pytest.mark.parametrize("d", [64, 128])
def test_golden_halfway_cases(d):
    for vals, codes, scale_bits in _golden_rows():
        x = np.zeros(d, np.float32)
        x[:len(vals)] = vals
        assert np.array_equal(_bf16(x), x), "fixture values must be bf16-exact"
        q, s = quantize(x[None])
        assert s.view(np.uint32)[0] == scale_bits
        assert list(q[0, :len(codes)]) == codes
        assert not q[0, len(codes):].any()


def test_absmax_maps_to_127():
    rng = np.random.default_rng(1)
    x = _bf16(rng.standard_normal((500, 128)) * rng.uniform(0.01, 100, (500, 1)))
    q, s = quantize(x)
    i = np.argmax(np.abs(x), axis=1)
    assert np.array_equal(np.abs(q[np.arange(500), i]), np.full(500, 127))
    assert np.array_equal(np.sign(q[np.arange(500), i]), np.sign(x[np.arange(500), i]).astype(np.int8))
    assert np.abs(q).max() <= 127 and q.min() >= -127


def test_exact_round_trip_for_scaled_integers():
    # x = c * 2^-e with |c| <= 127 and one |c| == 127: the scale is exactly 2^-e, codes are exactly c
    rng = np.random.default_rng(2)
    for e in [-3, 0, 4, 9]:
        c = rng.integers(-127, 128, (64, 128))
        c[:, 7] = 127 * np.where(rng.random(64) < 0.5, 1, -1)
        x = (c * 2.0 ** -e).astype(np.float32)
        assert np.array_equal(_bf16(x), x)
        q, s = quantize(x)
        assert np.array_equal(q.astype(np.int64), c)
        assert np.all(s == np.float32(2.0 ** -e))
        assert np.array_equal(dequantize(q, s), x.astype(np.float64))


def test_error_bound_with_outliers():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2000, 128)).astype(np.float32)
    x[:, [5, 77, 100]] *= 20
    x = _bf16(x)
    q, s = quantize(x)
    err = np.abs(x.astype(np.float64) - dequantize(q, s))
    # |x/s - q| <= 1/2 from rint plus the fp32 rounding of x/s itself, |x/s| * 2^-24 <= 128 * 2^-24
    bound = s.astype(np.float64)[:, None] * (0.5 + 2.0 ** -17)
    assert np.all(err <= bound)
    # and the bound is not loose by more than that rounding term
    assert (err / s[:, None]).max() > 0.5 - 2.0 ** -17


def test_zero_row_and_single_nonzero():
    q, s = quantize(np.zeros((3, 64), np.float32))
    assert not q.any() and not s.any()
    x = np.zeros((1, 64), np.float32)
    x[0, 10] = -3.0
    q, s = quantize(x)
    assert q[0, 10] == -127 and np.count_nonzero(q) == 1
    assert s[0] == np.float32(3.0) / np.float32(127.0)


def test_scale_is_per_row_not_per_tensor():
    x = np.zeros((2, 64), np.float32)
    x[0, 0], x[1, 0] = 1.0, 100.0
    q, s = quantize(x)
    assert q[0, 0] == 127 and q[1, 0] == 127
    assert s[0] != s[1]


def _exact_quantize_row(x):
    """The quantiser's definition in exact rational arithmetic, with each fp32 rounding done exactly:
    s = RN32(a / 127), q_c = clamp(round_half_even(RN32(x_c / s)), -127, 127), a = 0 -> s = 0, q = 0."""
    from fractions import Fraction
    from tests.helpers import rn32
    xs = [Fraction(float(v)) for v in x]
    a = max(abs(v) for v in xs)
    if a == 0:
        return [0] * len(xs), Fraction(0)
    s = rn32(a / 127)
    return [max(-127, min(127, round(rn32(v / s)))) for v in xs], s


def test_matches_exact_rational_definition():
    """Random, tie-constructed, tiny (subnormal scale) and huge bf16 rows: codes and scale equal the
    definition evaluated in exact rationals with exact fp32 roundings."""
    rng = np.random.default_rng(11)
    rows = [_bf16(rng.standard_normal(64) * 10.0 ** rng.uniform(-30, 30)) for _ in range(120)]
    for k in (-20, 0, 7):                       # s = 2^k exactly: (j + 1/2) 2^k are exact ties
        j = rng.integers(-127, 127, 64).astype(np.float32)
        x = ((j + np.float32(0.5)) * np.float32(2.0 ** k)).astype(np.float32)
        x[0] = np.float32(127 * 2.0 ** k)
        rows.append(x)
    for e in (-133, -128, -120):                # subnormal and near-subnormal absmax
        rows.append(_bf16(rng.uniform(-1, 1, 64) * 2.0 ** e))
    rows.append(_bf16(rng.choice([-1.0, 1.0], 64) * 3.3e38))
    # x = absmax / 2 where x / s lies just below 63.5 but its fp32 quotient is exactly 63.5: the
    # definition (fp32 division, then half-even) gives 64, a wider division would give 63
    for a_bits in (0x4238, 0x3F17, 0x423B):
        a = np.uint32(a_bits << 16).view(np.float32)
        x = np.zeros(64, np.float32)
        x[0], x[1], x[2] = a, a / 2, -a / 2
        rows.append(x)
    x = np.stack(rows).astype(np.float32)
    assert np.array_equal(_bf16(x), x)
    q, s = quantize(x)
    for i in range(x.shape[0]):
        codes, scale = _exact_quantize_row(x[i])
        assert s[i] == float(scale), i
        assert q[i].tolist() == codes, i
    assert [q[-3 + k, 1] for k in range(3)] == [64, 64, 64] and [q[-3 + k, 2] for k in range(3)] == [-64, -64, -64]
