"""The decode kernel computes f(j) = floor(j / G) (Jet-Long paper, §3.1) by a
multiply-high, a shift and an add instead of an integer division (Granlund
and Montgomery's method for unsigned division by an invariant integer).
This test restates that arithmetic in Python and checks the quotient
exactly for every group size up to 4096. Numerators are sampled, plus the
edges of every quotient step and the extremes of the 32-bit range."""
import random

import pytest

M32 = (1 << 32) - 1


def make_divider(G):
    l = 0
    while (1 << l) < G:
        l += 1
    m = ((1 << 32) * ((1 << l) - G)) // G + 1
    assert m <= M32
    return m, min(l, 1), max(l - 1, 0)


def divide(x, dv):
    m, sh1, sh2 = dv
    t = (m * x) >> 32                       # mulhi
    return (t + (((x - t) & M32) >> sh1)) >> sh2


@pytest.mark.parametrize("G", list(range(1, 65)) + [100, 127, 128, 129, 1000, 4095, 4096])
def test_quotient_is_exact(G):
    dv = make_divider(G)
    rng = random.Random(G)
    xs = set(range(0, 4 * G + 3))
    xs |= {M32, M32 - 1, (1 << 31) - 1, 1 << 31, (1 << 31) + 1}
    for _ in range(2000):
        q = rng.randrange(0, M32 // G + 1)
        for d in (-1, 0, 1, G - 1):
            x = q * G + d
            if 0 <= x <= M32:
                xs.add(x)
    for x in xs:
        assert divide(x, dv) == x // G, (G, x)
