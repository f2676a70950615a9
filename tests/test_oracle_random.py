"""Randomised checks of the oracle against its own independent formulations,
over small random shapes (hypothesis, derandomised so every run draws the
same cases):

* the vectorised prefill against the literal per-pair loop (positions and
  masks written out for each (i, j));
* the direct rule against the three-pass inclusion-exclusion merge (§3.3);
* the cache formulation (chunked prefill over keys stored at true positions,
  remote scores through the correction rotation) against the direct rule.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@st.composite
def problems(draw, max_L=24):
    L = draw(st.integers(1, max_L))
    Hkv = draw(st.integers(1, 2))
    grp = draw(st.integers(1, 3))
    D = draw(st.sampled_from([4, 8]))
    wp = draw(st.integers(1, max(1, L)))
    w0 = draw(st.integers(0, L + 1))
    theta = draw(st.sampled_from([1e4, 1e6]))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, L, Hkv * grp, D))
    k = rng.standard_normal((1, L, Hkv, D))
    v = rng.standard_normal((1, L, Hkv, D))
    return q, k, v, wp, w0, theta


@SETTINGS
@given(problems(max_L=16))
def test_vectorised_prefill_equals_the_literal_per_pair_loop(prob):
    q, k, v, wp, w0, theta = prob
    o1, l1 = oracle.prefill(q, k, v, wp, w0, theta)
    o2, l2 = oracle.prefill_literal(q, k, v, wp, w0, theta)
    np.testing.assert_allclose(o1, o2, atol=1e-11)
    np.testing.assert_allclose(l1, l2, atol=1e-11)


@SETTINGS
@given(problems())
def test_direct_rule_equals_the_three_pass_merge(prob):
    q, k, v, wp, w0, theta = prob
    o1, l1 = oracle.prefill(q, k, v, wp, w0, theta)
    o2, l2 = oracle.merge_three_pass(q, k, v, wp, w0, theta)
    np.testing.assert_allclose(o1, o2, atol=1e-9)
    np.testing.assert_allclose(l1, l2, atol=1e-9)


@SETTINGS
@given(problems(), st.data())
def test_cache_formulation_equals_the_direct_rule(prob, data):
    q, k, v, wp, w0, theta = prob
    L = q.shape[1]
    P0 = data.draw(st.integers(0, L - 1))
    cache = oracle.rope_cache(k, 0, theta)
    oc, lc = oracle.prefill_chunk(q[:, P0:], cache, v, P0, wp, w0, theta)
    o, lse = oracle.prefill(q, k, v, wp, w0, theta)
    np.testing.assert_allclose(oc, o[:, P0:], atol=1e-10)
    np.testing.assert_allclose(lc, lse[:, :, P0:], atol=1e-10)


# ---------------------------------------------------------------- frequency-interpolation map
RAMPS = st.sampled_from([(1.0, 32.0), (0.5, 3.0), (-2.0, -1.0), (1e6, 2e6), (2.0, 8.0)])


@SETTINGS
@given(problems(max_L=14), RAMPS)
def test_interp_vectorised_prefill_equals_the_literal_per_pair_loop(prob, ramp):
    q, k, v, wp, w0, theta = prob
    o1, l1 = oracle.prefill_interp(q, k, v, wp, w0, theta, *ramp)
    o2, l2 = oracle.prefill_interp_literal(q, k, v, wp, w0, theta, *ramp)
    np.testing.assert_allclose(o1, o2, atol=1e-11)
    np.testing.assert_allclose(l1, l2, atol=1e-11)


@SETTINGS
@given(problems(), RAMPS, st.data())
def test_interp_cache_formulation_equals_the_direct_rule(prob, ramp, data):
    q, k, v, wp, w0, theta = prob
    L = q.shape[1]
    P0 = data.draw(st.integers(0, L - 1))
    cache = oracle.rope_cache(k, 0, theta)
    oc, lc = oracle.prefill_chunk_interp(q[:, P0:], cache, v, P0, wp, w0, theta, *ramp)
    o, lse = oracle.prefill_interp(q, k, v, wp, w0, theta, *ramp)
    np.testing.assert_allclose(oc, o[:, P0:], atol=1e-10)
    np.testing.assert_allclose(lc, lse[:, :, P0:], atol=1e-10)


@SETTINGS
@given(problems(), RAMPS)
def test_interp_decode_equals_the_last_prefill_row(prob, ramp):
    q, k, v, wp, w0, theta = prob
    L = q.shape[1]
    cache = oracle.rope_cache(k, 0, theta)
    od, ld = oracle.decode_interp(q[:, L - 1], cache, v, L, wp, w0, theta, *ramp)
    o, lse = oracle.prefill_interp_rows(q, k, v, wp, w0, theta, [L - 1], *ramp)
    np.testing.assert_allclose(od, o[:, 0], atol=1e-10)
    np.testing.assert_allclose(ld, lse[:, :, 0], atol=1e-10)
