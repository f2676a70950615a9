"""The decode kernel computes f(j) = floor(j / G) (Jet-Long paper, §3.1) by a
multiply-high, a shift and an add instead of an integer division (Granlund
and Montgomery's method for unsigned division by an invariant integer).
This test restates that arithmetic and checks the quotient exactly against
integer division: for every group size G from 1 to 2^16, at every quotient
step j = mG - 1, mG, mG + 1 for a spread of m up to the 2^31 position range,
and on a dense random sample of j below 2^31; plus larger G up to 2^31 - 1."""
import random

import numpy as np
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


def dividers(G):
    """make_divider over an array of G (vectorised, exact in uint64)."""
    G = np.asarray(G, dtype=np.uint64)
    # l = ceil(log2 G) = bit length of G - 1 (exact through frexp below 2^53)
    l = np.frexp((G - np.uint64(1)).astype(np.float64))[1].astype(np.uint64)
    m = ((np.uint64(1) << np.uint64(32)) * ((np.uint64(1) << l) - G)) // G + np.uint64(1)
    return m, np.minimum(l, np.uint64(1)), np.where(l > 1, l - np.uint64(1), np.uint64(0))


def divide_arr(x, m, sh1, sh2):
    t = (m * x) >> np.uint64(32)
    return (t + (((x - t) & np.uint64(M32)) >> sh1)) >> sh2


def test_vectorised_divider_agrees_with_the_scalar_one():
    for G in list(range(1, 300)) + [4095, 4096, 4097, 65535, 65536]:
        m, a, b = dividers([G])
        assert (int(m[0]), int(a[0]), int(b[0])) == make_divider(G), G


def test_every_group_size_to_2_16_at_every_quotient_step():
    G = np.arange(1, (1 << 16) + 1, dtype=np.uint64)
    m, sh1, sh2 = dividers(G)
    assert np.all(m <= np.uint64(M32))
    rng = np.random.default_rng(0)
    qmax = (np.uint64((1 << 31) - 1) // G).astype(np.float64)
    # quotients 0..3, the largest below 2^31, and 24 spread between
    qs = [np.zeros_like(G), np.ones_like(G), np.full_like(G, 2), np.full_like(G, 3),
          qmax.astype(np.uint64)]
    for _ in range(24):
        qs.append(np.floor(rng.random(G.shape) * qmax).astype(np.uint64))
    for q in qs:
        for d in (-1, 0, 1):
            x = q.astype(np.int64) * G.astype(np.int64) + d
            ok = (x >= 0) & (x < (1 << 31))
            xu = x[ok].astype(np.uint64)
            got = divide_arr(xu, m[ok], sh1[ok], sh2[ok])
            assert np.array_equal(got, xu // G[ok])


def test_dense_random_positions_below_2_31():
    rng = np.random.default_rng(1)
    G = rng.integers(1, (1 << 16) + 1, size=1 << 20, dtype=np.uint64)
    x = rng.integers(0, 1 << 31, size=G.shape, dtype=np.uint64)
    m, sh1, sh2 = dividers(G)
    assert np.array_equal(divide_arr(x, m, sh1, sh2), x // G)


@pytest.mark.parametrize("G", [(1 << 16) + 1, 98305, 1 << 20, (1 << 20) + 3, 12345679,
                               (1 << 30) - 1, 1 << 30, (1 << 31) - 1])
def test_large_group_sizes(G):
    dv = make_divider(G)
    rng = random.Random(G)
    xs = {0, 1, G - 1, G, G + 1, (1 << 31) - 1, M32, M32 - 1}
    for _ in range(2000):
        q = rng.randrange(0, M32 // G + 1)
        for d in (-1, 0, 1):
            x = q * G + d
            if 0 <= x <= M32:
                xs.add(x)
    for x in xs:
        assert divide(x, dv) == x // G, (G, x)
