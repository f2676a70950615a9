"""Host-side check of the RoPE angle reduction the kernels use before the
single-precision sine/cosine (prefill operand pass, decode query, cache
writer).

The angle a = pos * freq is formed in double precision.  The kernels then
subtract the nearest multiple n of 2 pi in two fused multiply-adds, with
2 pi split into a double head and its tail.  This test restates those steps
with exact rational arithmetic for the fused operations.  It checks that
the reduced angle is the double-rounded product modulo 2 pi, computed in
60-digit decimals, to within 1e-15 absolute (a few ulps of pi), for
positions up to 2^31.  A reduction by the double 2 pi alone would be off by
n * 2.4e-16, up to 1e-7 there.  It also checks that the reduced angle lies
in [-pi, pi].  The product itself is one double rounding, a relative error
of 2^-53.
"""
import math
import random
from decimal import Decimal, getcontext
from fractions import Fraction

import pytest

getcontext().prec = 60
PI = Decimal("3.14159265358979323846264338327950433288419716939937510582097494")
TWO_PI_HI = 6.283185307179586232
TWO_PI_LO = 2.4492935982947064e-16
INV_TWO_PI = 0.15915494309189533577


def fma(a: float, b: float, c: float) -> float:
    """a * b + c with one rounding (exact rational arithmetic, then round)."""
    return float(Fraction(a) * Fraction(b) + Fraction(c))


def reduce_angle(pos: int, freq: float) -> float:
    a = float(pos) * freq
    n = float(round(a * INV_TWO_PI))     # rint: nearest, ties to even
    r = fma(-n, TWO_PI_HI, a)
    return fma(-n, TWO_PI_LO, r)


def exact_reduced(a: float) -> Decimal:
    x = Decimal(a)
    two_pi = 2 * PI
    k = (x / two_pi).to_integral_value()
    return x - k * two_pi


def test_split_of_two_pi():
    assert Decimal(TWO_PI_HI) + Decimal(TWO_PI_LO) - 2 * PI < Decimal("1e-31")
    assert Decimal(TWO_PI_HI) + Decimal(TWO_PI_LO) - 2 * PI > Decimal("-1e-31")


@pytest.mark.parametrize("D,theta", [(128, 1e6), (64, 1e4)])
def test_reduced_angle_is_the_product_modulo_two_pi(D, theta):
    rng = random.Random(D)
    for _ in range(400):
        pos = rng.randrange(0, 1 << 31)
        t = rng.randrange(D // 2)
        freq = math.exp(-2.0 * t / D * math.log(theta))
        a = float(pos) * freq
        r = reduce_angle(pos, freq)
        assert -math.pi - 1e-12 <= r <= math.pi + 1e-12
        err = abs(Decimal(r) - exact_reduced(a))
        # n * 2pi_hi is exact inside the first fma; what is left is the two
        # final roundings of numbers below 2 pi in magnitude
        assert err <= Decimal("1e-15"), (pos, t, float(err))
