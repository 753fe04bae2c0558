"""The quantize kernel takes the block scale's RN(amax / 6) not by an IEEE
division but by one Markstein correction step (P. W. Markstein, IBM J. Res.
Dev. 34(1), 1990): q0 = RN(a·y) with y = RN(1/6), r = RN(a − 6·q0) (one FMA),
q = RN(r·y + q0) (one FMA), and keeps the IEEE division where a/6 is below the
normal range.  The claim it rests on — q equals the correctly rounded a/6 for
every finite a >= 6·2^-126 — is checked here in exact rational arithmetic
(every FMA emulated as one rounding of the exact value), on the values where a
wrong rounding would show: every exponent's smallest, largest and
near-multiple-of-3 mantissas, plus a large seeded sample.  The kernel's own
outputs are held to the oracle's IEEE division bit for bit by the GPU tests."""
from fractions import Fraction

import numpy as np


def rn32(x):
    """Round a non-negative rational to the nearest fp32 value (ties to even),
    returned exactly as a Fraction; subnormals are multiples of 2^-149."""
    if x == 0:
        return Fraction(0)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    assert e <= 127, e
    e = max(e, -126)                                # subnormal: the quantum stays 2^-149
    scaled = x / (Fraction(2) ** (e - 23))          # in [2^23, 2^24), or below for subnormals
    m = scaled.numerator // scaled.denominator
    rem = scaled - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    return Fraction(m) * Fraction(2) ** (e - 23)


Y = rn32(Fraction(1, 6))


def markstein_div6(a):
    q0 = rn32(a * Y)
    r = a - 6 * q0                         # exact; one FMA rounds it once
    r = rn32(abs(r)) * (1 if r >= 0 else -1)
    return rn32(r * Y + q0)


def test_reciprocal_constant_is_the_kernels():
    assert float(Y) == float(np.float32(1.0) / np.float32(6.0))
    assert np.float32(float(Y)).view(np.uint32) == 0x3E2AAAAB


def test_markstein_step_is_the_correctly_rounded_quotient():
    rng = np.random.default_rng(0)
    mants = list(range(0, 8)) + list(range((1 << 23) - 8, 1 << 23))
    mants += [(k * ((1 << 23) // 3)) % (1 << 23) for k in range(1, 7)]
    mants += [int(v) for v in rng.integers(0, 1 << 23, 40)]
    vals = []
    for e in list(range(-123, -118)) + list(range(-10, 11)) + list(range(120, 128)):
        for m in mants:
            vals.append(Fraction((1 << 23) + m) * Fraction(2) ** (e - 23))
    bits = rng.integers(0x04000000, 0x7F000000, 4000, dtype=np.int64).astype(np.uint32)
    vals += [Fraction(float(v)) for v in bits.view(np.float32) if np.isfinite(v)]
    bad = [a for a in vals if a / 6 >= Fraction(2) ** -126 and markstein_div6(a) != rn32(a / 6)]
    assert not bad, [float(b) for b in bad[:5]]
