"""The quantizers' quotient: Markstein's correction of the reciprocal quotient (P. Markstein,
IBM J. Res. Dev. 34(1), 1990) gives the correctly rounded float32 quotient a / b.

The kernels compute y = RN(1/b), q0 = RN(a y), r = RN(a - q0 b) (one fused multiply-add)
and q = RN(q0 + r y) (one fused multiply-add). This test carries out the same steps with
exact rational arithmetic and one float32 rounding per operation, and checks q against the
exactly rounded a / b, on the operands the quantizers meet: a = x - z for float32 x and a
float16 zero-point z, b a positive float16 scale; half of the samples are placed within a
few ulps of a rounding tie of the quotient (the cases where a plain reciprocal multiply
can round to the other side). The codes rint(clamp(q)) must then equal the definition's.
"""
from fractions import Fraction

import numpy as np
import pytest


def rn32(x: Fraction) -> Fraction:
    """Round a rational to the nearest float32 (ties to even), exactly."""
    if x == 0:
        return Fraction(0)
    f = np.float32(float(x))                      # within an ulp of the answer
    cands = {f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))}
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - x)
        key = (d, int(np.array(c, np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return Fraction(float(best[1]))


def markstein(a: Fraction, b: Fraction) -> Fraction:
    y = rn32(1 / b)
    q0 = rn32(a * y)
    r = rn32(a - q0 * b)
    return rn32(q0 + r * y)


def operands(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        b = np.float16(rng.uniform(2.0 ** -14, 60000.0))
        while not np.isfinite(b) or b <= 0:
            b = np.float16(rng.uniform(2.0 ** -14, 60000.0))
        z = np.float16(rng.normal(0, 4))
        if i % 2 == 0:
            x = np.float32(np.float32(z) + np.float32(b) * np.float32(rng.uniform(-2, 18)))
        else:
            # x - z near (k + 1/2) b: the quotient within a few ulps of a rounding tie
            k = rng.integers(-1, 16)
            t = np.array([np.float32(z) + np.float32((k + 0.5) * np.float32(b))], np.float32)
            x = (t.view(np.int32) + np.int32(rng.integers(-3, 4))).view(np.float32)[0]
        a = np.float32(np.float32(x) - np.float32(z))      # f32(x - z), as the kernels
        if not np.isfinite(a):
            continue
        out.append((Fraction(float(a)), Fraction(float(b))))
    return out


def rint_clamp(q: Fraction, qmax: int) -> int:
    q = min(max(q, Fraction(0)), Fraction(qmax))
    f = q.numerator // q.denominator
    rem = q - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


@pytest.mark.parametrize("seed", [1, 2])
def test_markstein_quotient_is_correctly_rounded(seed):
    for a, b in operands(3000, seed):
        q = markstein(a, b)
        exact = rn32(a / b)
        assert q == exact, (float(a), float(b), float(q), float(exact))
        for qmax in (3, 15):
            assert rint_clamp(q, qmax) == rint_clamp(exact, qmax)


def test_plain_reciprocal_product_is_not_always_correctly_rounded():
    """Why the correction is there: RN(a RN(1/b)) alone misses the correctly rounded
    quotient on some of the same operands."""
    misses = sum(rn32(a * rn32(1 / b)) != rn32(a / b) for a, b in operands(3000, 3))
    assert misses > 0
