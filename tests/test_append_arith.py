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
