"""CPU check of the division method of the tensor-core epilogue.

The epilogue computes RN(a / s_x) for an integer-valued a (|a| <= 2^24) and
s_x > 0 from r = RN(1 / s_x), by Markstein's FMA correction (IBM J. Res.
Dev. 34(1), 1990; Muller et al., "Handbook of Floating-Point Arithmetic"):
q = RN(a*r), then twice e = RN(a - s_x*q) (exact, one FMA) and
q = RN(q + e*r). Here every step is emulated with exact rationals and one
fp32 rounding, and the result is compared with the correctly rounded
quotient, on random operands and on the ones next to powers of two where a
single correction is weakest. The GPU tests compare the kernel's outputs with
the oracle's IEEE division bit for bit.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest


def rn32(v: Fraction) -> np.float32:
    """Nearest fp32 to a rational (normal range), ties to even significand."""
    if v == 0:
        return np.float32(0.0)
    sign = -1 if v < 0 else 1
    v = abs(v)
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    quantum = Fraction(2) ** (e - 23)
    scaled = v / quantum
    sig, rem = divmod(scaled.numerator, scaled.denominator)
    if 2 * rem > scaled.denominator or (2 * rem == scaled.denominator and sig % 2 == 1):
        sig += 1
    return np.float32(sign * float(sig * quantum))


def fr(x) -> Fraction:
    return Fraction(float(x))


def corrected_div(a: np.float32, s: np.float32) -> np.float32:
    r = rn32(1 / fr(s))
    q = rn32(fr(a) * fr(r))
    for _ in range(2):
        e = rn32(fr(a) - fr(s) * fr(q))
        q = rn32(fr(q) + fr(e) * fr(r))
    return q


def operands(seed: int, n: int):
    rng = random.Random(seed)
    for i in range(n):
        kind = i % 3
        if kind == 0:  # scales of real tokens: s_x = RN(127 / max|x|)
            s = rn32(Fraction(127) / fr(np.float32(abs(rng.gauss(0, 1)) * 10 ** rng.uniform(-3, 4) + 1e-5)))
        elif kind == 1:  # 1/s next to a power of two
            s = np.float32(math.ldexp(2.0 - 2.0 ** -23 * rng.randint(1, 4), rng.randint(-20, 20)))
        else:
            s = np.float32(math.ldexp(1.0 + 2.0 ** -23 * rng.randint(0, 3), rng.randint(-20, 20)))
        k = rng.randint(1, 24)
        a = np.float32(rng.choice([rng.randint(-2 ** 24, 2 ** 24), rng.randint(-300, 300), 2 ** k - 1,
                                   -(2 ** k - rng.randint(1, 3)), 2 ** k]))
        yield a, s


@pytest.mark.parametrize("seed", range(3))
def test_corrected_division_is_correctly_rounded(seed):
    bad = []
    for a, s in operands(seed, 700):
        want = rn32(fr(a) / fr(s))
        got = corrected_div(a, s)
        if np.float32(got).view(np.uint32) != np.float32(want).view(np.uint32):
            bad.append((float(a), float(s)))
    assert not bad, bad[:5]


def test_corrected_division_zero_and_sign():
    for s in (np.float32(1.0), np.float32(127.0), np.float32(3.1e-7)):
        assert corrected_div(np.float32(0.0), s) == np.float32(0.0)
        for a in (np.float32(5.0), np.float32(-5.0)):
            assert corrected_div(a, s) == rn32(fr(a) / fr(s))


def test_operands_catch_an_uncorrected_quotient():
    """The operand set is not trivial: RN(a * RN(1/s)) alone misses the
    correctly rounded quotient on a good share of it."""
    miss = 0
    for a, s in operands(0, 700):
        q = rn32(fr(a) * fr(rn32(1 / fr(s))))
        miss += np.float32(q).view(np.uint32) != np.float32(rn32(fr(a) / fr(s))).view(np.uint32)
    assert miss > 50
