"""Host-side check of the decode kernel's correction phase arithmetic.

The decode kernel forms the correction angle Delta * omega_t of a cached key
(Jet-Long paper, §3.2: Delta = f(j) - j with omega_t = theta_t; or, for the
frequency-interpolation remote map of §4.7, Delta = j with omega_t =
theta'_t - theta_t < 0) as a phase in turns:

  * omega_t / (2 pi) is held as a 64-bit two's-complement binary fraction,
    rounded from a double;
  * Delta times it wraps modulo 2^64, which is exact arithmetic modulo one
    turn;
  * the top 32 bits, read as a signed integer, are the phase in units of
    2^-32 turn, so the angle given to the sine/cosine lies in [-pi, pi).

This test restates those integer steps in Python and compares the phase
with Delta * omega_t / (2 pi) modulo 1, evaluated in 60-digit decimal
arithmetic from the same doubles.  The error must stay within 2^-31 turn
for every cache position up to 2^21.
"""
import math
import random
from decimal import Decimal, getcontext

import pytest

getcontext().prec = 60
PI = Decimal("3.14159265358979323846264338327950433288419716939937510582097494")
TURN_Q64 = 0.15915494309189533577 * 18446744073709551616.0  # 2^64 / (2 pi), a double
MASK64 = (1 << 64) - 1


def to_q64(x: float) -> int:
    """A double of magnitude < 2^63 rounded to the nearest integer, as uint64."""
    return int(round(x)) & MASK64


def kernel_phase_turns(delta: int, omega_q64: int) -> float:
    prod = (delta * omega_q64) & MASK64     # 64-bit product, wraps
    top = prod >> 32
    if top >= 1 << 31:                      # signed 32-bit phase
        top -= 1 << 32
    return top / 2.0**32


def exact_phase_turns(delta: int, omega: float) -> Decimal:
    t = Decimal(delta) * Decimal(omega) / (2 * PI)
    t -= t.to_integral_value(rounding="ROUND_FLOOR")
    return t - 1 if t >= Decimal("0.5") else t  # into [-1/2, 1/2)


def turn_distance(a: float, b: Decimal) -> float:
    d = abs(Decimal(a) - b)
    return float(min(d, 1 - d))


def rope_freq(t: int, D: int, theta: float) -> float:
    return math.exp(-2.0 * t / D * math.log(theta))


def interp_factor(freq: float, L: int, wp: int, alpha: float, beta: float) -> float:
    s = max(1.0, L / wp)
    turns = wp * freq * 0.15915494309189533577
    gam = min(1.0, max(0.0, (turns - alpha) / (beta - alpha)))
    return (1.0 - gam) / s + gam


CASES = [(128, 1e6), (128, 1e4), (64, 1e4)]


@pytest.mark.parametrize("D,theta", CASES)
def test_aliasing_correction_phase(D, theta):
    # Delta = f(j) - j <= 0 against a positive omega
    rng = random.Random(D + int(theta))
    for G in (2, 3, 4, 32):
        for _ in range(200):
            j = rng.randrange(0, 1 << 21)
            t = rng.randrange(D // 2)
            f = rope_freq(t, D, theta)
            om = to_q64(f * TURN_Q64)
            delta = j // G - j
            got = kernel_phase_turns(delta, om)
            assert -0.5 <= got < 0.5
            assert turn_distance(got, exact_phase_turns(delta, f)) <= 2.0**-31


@pytest.mark.parametrize("D,theta", CASES)
def test_interpolation_correction_phase(D, theta):
    # Delta = j >= 0 against a negative omega (theta' - theta), two's complement
    rng = random.Random(7 * D + int(theta))
    for L, wp, alpha, beta in ((131072, 32768, 1.0, 32.0), (1 << 20, 32768, 1.0, 32.0),
                               (700, 1, 1.0, 32.0), (4096, 1000, 0.5, 3.0)):
        for _ in range(200):
            j = rng.randrange(0, 1 << 21)
            t = rng.randrange(D // 2)
            f = rope_freq(t, D, theta)
            kappa = interp_factor(f, L, wp, alpha, beta)
            assert 0.0 < kappa <= 1.0
            om = to_q64(f * (kappa - 1.0) * TURN_Q64)
            got = kernel_phase_turns(j, om)
            assert -0.5 <= got < 0.5
            exact = exact_phase_turns(j, f * (kappa - 1.0))
            assert turn_distance(got, exact) <= 2.0**-31


def test_fractions_fit_the_signed_64_bit_range():
    # |omega| / (2 pi) < 1/(2 pi) < 1/2 turn: both signs fit in int64 before
    # the conversion, for every frequency theta^(-2t/D) <= 1
    assert 1.0 * TURN_Q64 < 2.0**63
    assert -1.0 * TURN_Q64 > -(2.0**63)
