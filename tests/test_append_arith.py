"""Host check of the append kernel's scale arithmetic (no GPU): s = RN(a / 127) computed without a
division as q0 = RN(a c), c = RN(1/127), then s = RN(q0 + (a - 127 q0) c) with the remainder exact
(Markstein's correction step).  Exact rational arithmetic over every bf16 absmax a in the range where
the kernel takes this path ([2^-110, max finite bf16]): the remainder is exact (a subnormal at the
low end) and s is a normal equal to the correctly rounded quotient.  The kernel sends zero,
subnormal and non-finite a elsewhere."""
import struct
from fractions import Fraction

from tests.helpers import rn32


def _bf16(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", bits << 16))[0])


def test_rounding_helper_matches_fp32_casts():
    import numpy as np
    rng = np.random.default_rng(0)
    for v in np.concatenate([rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200),
                             rng.standard_normal(50) * 1e-40]):                  # fp32 subnormals
        assert rn32(Fraction(float(v))) == Fraction(float(np.float32(v)))


def test_division_by_127_without_division_is_exact():
    c = rn32(Fraction(1, 127))
    assert float(c) == float.fromhex("0x1.020408p-7")
    lo = (127 - 110) << 7                                # bf16 bits of 2^-110
    checked = 0
    for bits in range(lo, 0x7F80):
        a = _bf16(bits)
        q0 = rn32(a * c)
        rem = rn32(a - 127 * q0)
        assert rem == a - 127 * q0, "remainder not exact"
        s = rn32(rem * c + q0) if rem else q0
        assert s == rn32(a / 127) and s >= Fraction(2) ** -126, hex(bits)
        checked += 1
    assert checked == 0x7F80 - lo


def _rint_even(x: Fraction) -> int:
    fl = x.numerator // x.denominator
    rem = x - fl
    return fl + 1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl & 1) else fl


def _fast_code(x: Fraction, s: Fraction, r0: Fraction):
    """The kernel's fast path in exact arithmetic: r = RN(r0 + r0 RN(1 - s r0)) (two FMAs),
    t = RN(x r + 1.5 * 2^23), q = t - 1.5 * 2^23, d = RN(x r - q).  Returns (q, |d| < 1/2 - 2^-15)."""
    magic = Fraction(3 * 2 ** 22)
    r = rn32(r0 * rn32(1 - s * r0) + r0)
    q = rn32(x * r + magic) - magic
    d = rn32(x * r - q)
    return int(q), abs(d) < Fraction(1, 2) - Fraction(1, 2 ** 15)


def _r0_candidates(s: Fraction):
    """Reciprocal approximations within the hardware's one-ulp bound: RN(1/s) and its fp32 neighbours."""
    r = rn32(1 / s)
    e = r.numerator.bit_length() - r.denominator.bit_length()
    if r < Fraction(2) ** e:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    return [r - ulp, r, r + ulp]


def test_fast_path_codes_equal_the_rounded_exact_quotient():
    """Whenever the fast path keeps its code (|d| small), the code is rint(RN(x / s)) half-to-even; near
    ties fall through to the exact quotient.  Every bf16 x in [-a, a] for absmax values with many exact
    half-integer quotients (s a power of two) and for a few ordinary ones, with each reciprocal
    approximation the hardware may return."""
    import numpy as np
    c = rn32(Fraction(1, 127))
    absmaxes = [Fraction(127), Fraction(127, 2 ** 9), _bf16(0x4000 | 0x35), _bf16(0x3F80 | 0x11)]
    rng = np.random.default_rng(7)
    kept = fell_through = 0
    for a in absmaxes:
        q0 = rn32(a * c)
        s = rn32(rn32(a - 127 * q0) * c + q0)
        assert s == rn32(a / 127)
        abits = int(np.array([float(a)], dtype=np.float32).view(np.uint32)[0] >> 16)
        xs = [_bf16(b) for b in range(0, abits + 1, 1 if a == 127 else 7)]
        xs += [-x for x in xs[1::3]]
        for r0 in _r0_candidates(s):
            for x in xs:
                q, keep = _fast_code(x, s, r0)
                if keep:
                    assert q == _rint_even(rn32(x / s)), (float(x), float(s), float(r0))
                    kept += 1
                else:
                    fell_through += 1
        # a few random bf16 x below a, with random tie-adjacent offsets
        for x in rng.uniform(-float(a), float(a), 200):
            xf = _bf16(int(np.array([x], dtype=np.float32).view(np.uint32)[0] >> 16))
            q, keep = _fast_code(xf, s, _r0_candidates(s)[1])
            assert not keep or q == _rint_even(rn32(xf / s))
    assert kept > 10000 and fell_through > 0
