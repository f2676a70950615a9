"""Pins for the fp64 CPU oracle: each test checks it against something other
than itself (values printed in the Jet-Long paper, library routines, closed
forms, brute force, invariants), so that a plausible slip anywhere in the
oracle (a dropped term, a sign, an index, an off-by-one window edge) fails
one of them.  See ``test_oracle_mutations.py`` for planted mistakes."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, prefill_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def rope_complex(x, pos, theta):
    """RoPE written as complex multiplication, independent of the oracle:
    pair (x_i, x_{i+D/2}) is the complex number x_i + 1j*x_{i+D/2}, multiplied
    by exp(1j * pos * omega_i) with omega_i = exp(-(2i/D) ln theta)."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    omega = np.exp(-(2.0 * np.arange(h) / D) * math.log(theta))
    z = x[..., :h] + 1j * x[..., h:]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * omega)
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa_with_positions(q, k, v, qpos, kpos, theta, mask=None):
    """Plain (textbook) causal RoPE attention via torch's fp64 SDPA on CPU,
    with caller-chosen position ids.  Returns o [B,L,Hq,D], lse [B,Hq,L]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, D = q.shape
    grp = Hq // k.shape[2]
    qr = torch.from_numpy(rope_complex(q, np.asarray(qpos)[None, :, None], theta)).permute(0, 2, 1, 3)
    kr = torch.from_numpy(rope_complex(k, np.asarray(kpos)[None, :, None], theta)).permute(0, 2, 1, 3)
    vv = torch.from_numpy(v).permute(0, 2, 1, 3)
    kr = kr.repeat_interleave(grp, dim=1)
    vv = vv.repeat_interleave(grp, dim=1)
    if mask is None:
        mask = np.tril(np.ones((L, L), dtype=bool))
    m = torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(qr, kr, vv, attn_mask=m)
    s = (qr @ kr.transpose(-1, -2)) / math.sqrt(D)
    s = s.masked_fill(~m, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def tiny_inputs(name="tiny", **over):
    w = WORKLOADS[name].with_(**over) if over else WORKLOADS[name]
    x = prefill_inputs(w)
    f64 = lambda t: t.to(torch.float64).numpy()
    return w, f64(x.q), f64(x.k), f64(x.v)


# ---------------------------------------------------------------- schedule
def read_golden_schedule():
    rows = []
    with open(os.path.join(GOLDEN, "schedule_pages.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                L, w, G = (int(t) for t in line.split())
                rows.append((L, w, G))
    return rows


def test_group_size_matches_page_values():
    rows = read_golden_schedule()
    assert len(rows) >= 4
    for L, w, G in rows:
        assert oracle.group_size(L, w) == G, (L, w, G)


def test_group_size_is_minimal_integer_compression():
    # §3.1: G is the smallest integer compression that keeps every remote
    # position f(x), x < L, inside the pretrained range [0, w_pretrained).
    # Brute force that search and compare.
    for w in (1, 2, 3, 7, 16, 128):
        for L in range(1, 8 * w + 3):
            G = 1
            while (L - 1) // G > w - 1:
                G += 1
            assert oracle.group_size(L, w) == G, (L, w)


def test_remap_identity_iff_native_and_monotone():
    w = 128
    for L in (1, 5, 96, 127, 128, 129, 256, 257, 512, 1000):
        G = oracle.group_size(L, w)
        x = np.arange(L)
        f = oracle.remap(x, G)
        assert np.all(np.diff(f) >= 0)                      # monotone
        assert np.all(np.diff(f) <= 1)                      # no gaps in the remote grid
        assert f[-1] <= w - 1                               # remote positions in range
        assert np.array_equal(f, x) == (L <= w)             # identity iff L <= w_pretrained
        assert np.array_equal(f, np.floor(x / G).astype(np.int64))


# ---------------------------------------------------------------- RoPE
def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    for D, theta in ((2, 10000.0), (8, 10000.0), (64, 1e4), (128, 1e6)):
        x = rng.standard_normal((5, D))
        pos = np.array([0, 1, 17, 4096, 131071])
        np.testing.assert_allclose(oracle.rope(x, pos, theta), rope_complex(x, pos, theta),
                                   rtol=0, atol=1e-9)


def test_rope_relative_position_invariance():
    # §2.1: scores depend only on the relative position.
    rng = np.random.default_rng(2)
    D, theta = 64, 1e4
    x, y = rng.standard_normal(D), rng.standard_normal(D)
    for a, b, s in ((5, 3, 11), (1000, 7, -7), (0, 0, 123456)):
        lhs = oracle.rope(x, a, theta) @ oracle.rope(y, b, theta)
        rhs = oracle.rope(x, a + s, theta) @ oracle.rope(y, b + s, theta)
        rel = x @ oracle.rope(y, b - a, theta)
        assert abs(lhs - rhs) < 1e-9 and abs(lhs - rel) < 1e-9


def test_rope_norm_identity_and_composition():
    rng = np.random.default_rng(3)
    D, theta = 128, 1e6
    x = rng.standard_normal((4, D))
    np.testing.assert_allclose(oracle.rope(x, 0, theta), x, atol=0)
    r = oracle.rope(x, 98305, theta)
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, 70000, theta), -3000, theta),
                               oracle.rope(x, 67000, theta), atol=1e-9)


def test_correction_rotation_recovers_remote_phase():
    # §3.2: rotating the true-position cache entry by Delta k = f(k) - k gives
    # exactly RoPE(x_k, f(k)).
    rng = np.random.default_rng(4)
    D, theta, w = 64, 1e4, 128
    k = rng.standard_normal((1, 700, 2, D))
    G = oracle.group_size(700, w)
    cache = oracle.rope_cache(k, 0, theta)
    pos = np.arange(700)
    corr = oracle.correction_rotate(cache, pos[None, :, None], G, theta)
    want = rope_complex(k, (pos // G)[None, :, None], theta)
    np.testing.assert_allclose(corr, want, atol=1e-9)


def test_rope_cache_offset():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((2, 9, 3, 16))
    np.testing.assert_allclose(oracle.rope_cache(k, 40, 1e4),
                               rope_complex(k, (40 + np.arange(9))[None, :, None], 1e4), atol=1e-9)


# ---------------------------------------------------------------- whole result
def test_native_window_reduces_to_plain_rope_attention():
    # L = 96 <= w_pretrained = 128: G = 1 and the bifocal rule is plain causal
    # RoPE attention (§2.2 / Appendix H "Native-window fallback").
    w, q, k, v = tiny_inputs("tiny_native")
    assert oracle.group_size(w.L, w.w_pretrained) == 1
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    pos = np.arange(w.L)
    o_ref, lse_ref = sdpa_with_positions(q, k, v, pos, pos, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


def test_wide_window_equals_true_position_attention():
    # w0 >= L - 1: every pair is local, so G > 1 does not matter.
    w, q, k, v = tiny_inputs("tiny", L=200, w0=199)
    assert oracle.group_size(w.L, w.w_pretrained) == 2
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    pos = np.arange(w.L)
    o_ref, lse_ref = sdpa_with_positions(q, k, v, pos, pos, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


def test_zero_window_equals_remote_position_attention():
    # w0 = 0 keeps only self-attention local (§4.6); at distance 0 the local and
    # remote scores coincide, so the whole result is plain attention with
    # position ids f(.) -- a textbook routine with remapped positions.
    w, q, k, v = tiny_inputs("tiny", w0=0)
    G = oracle.group_size(w.L, w.w_pretrained)
    assert G == 4
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, 0, w.theta)
    f = np.arange(w.L) // G
    o_ref, lse_ref = sdpa_with_positions(q, k, v, f, f, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


def test_rows_inside_local_window_see_true_positions():
    # Rows i <= w0 only have keys at distance <= w0: plain RoPE attention rows.
    w, q, k, v = tiny_inputs("tiny")
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    pos = np.arange(w.L)
    o_ref, lse_ref = sdpa_with_positions(q, k, v, pos, pos, w.theta)
    n = w.w0 + 1
    np.testing.assert_allclose(o[:, :n], o_ref[:, :n], atol=1e-10)
    np.testing.assert_allclose(lse[:, :, :n], lse_ref[:, :, :n], atol=1e-10)
    # ... and rows past the window do differ (the remote branch is live).
    assert np.abs(o[:, n + 8:] - o_ref[:, n + 8:]).max() > 1e-3


def test_band_and_remote_parts_via_masked_library_attention():
    # Split the bifocal softmax into its two disjoint key sets, each computed
    # by the library with a mask, and recombine by log-sum-exp.
    w, q, k, v = tiny_inputs("tiny")
    G = oracle.group_size(w.L, w.w_pretrained)
    pos = np.arange(w.L)
    dist = pos[:, None] - pos[None, :]
    band = (dist >= 0) & (dist <= w.w0)
    far = dist > w.w0
    ob, lb = sdpa_with_positions(q, k, v, pos, pos, w.theta, mask=band)
    far_rows = far.any(axis=1)
    far_m = far.copy()
    far_m[~far_rows, 0] = True          # keep SDPA finite on rows with no far keys
    orr, lr = sdpa_with_positions(q, k, v, pos // G, pos // G, w.theta, mask=far_m)
    lr[:, :, ~far_rows] = -np.inf
    M = np.maximum(lb, lr)
    wb, wr = np.exp(lb - M), np.exp(lr - M)
    tot = wb + wr
    o_ref = (wb / tot).transpose(0, 2, 1)[..., None] * ob + (wr / tot).transpose(0, 2, 1)[..., None] * np.nan_to_num(orr)
    lse_ref = M + np.log(tot)
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


def test_grouped_query_heads_share_kv_heads_in_blocks():
    # GQA layout: query head h reads KV head h // (Hq / Hkv) (the grouped-query
    # layout torch's repeat_interleave builds).  Hq = 6, Hkv = 2, both branches live.
    rng = np.random.default_rng(8)
    B, L, Hq, Hkv, D, wp, w0, theta = 2, 150, 6, 2, 16, 64, 9, 1e4
    q = rng.standard_normal((B, L, Hq, D))
    k = rng.standard_normal((B, L, Hkv, D))
    v = rng.standard_normal((B, L, Hkv, D))
    o, lse = oracle.prefill(q, k, v, wp, w0, theta)
    G = oracle.group_size(L, wp)
    pos = np.arange(L)
    o_near, l_near = sdpa_with_positions(q, k, v, pos, pos, theta)
    o_far, l_far = sdpa_with_positions(q, k, v, pos // G, pos // G, theta)
    n = w0 + 1
    np.testing.assert_allclose(o[:, :n], o_near[:, :n], atol=1e-10)
    np.testing.assert_allclose(lse[:, :, :n], l_near[:, :, :n], atol=1e-10)
    o0, l0 = oracle.prefill(q, k, v, wp, 0, theta)
    np.testing.assert_allclose(o0, o_far, atol=1e-10)
    np.testing.assert_allclose(l0, l_far, atol=1e-10)


def test_inclusion_exclusion_merge_identity():
    # §3.3: the three-pass merge equals the direct per-pair rule.
    w, q, k, v = tiny_inputs("tiny")
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    o3, lse3 = oracle.merge_three_pass(q, k, v, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(o, o3, atol=1e-9)
    np.testing.assert_allclose(lse, lse3, atol=1e-9)


def test_literal_per_pair_brute_force():
    # A tiny case small enough for the pure-Python per-pair loop: G = 4.
    rng = np.random.default_rng(6)
    B, L, Hq, Hkv, D = 1, 40, 2, 1, 8
    q = rng.standard_normal((B, L, Hq, D))
    k = rng.standard_normal((B, L, Hkv, D))
    v = rng.standard_normal((B, L, Hkv, D))
    for w0 in (0, 5, 39):
        o1, l1 = oracle.prefill(q, k, v, 10, w0, 1e4)
        o2, l2 = oracle.prefill_literal(q, k, v, 10, w0, 1e4)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_prefill_rows_subset_matches_full():
    w, q, k, v = tiny_inputs("tiny")
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    rows = [0, 31, 32, 33, 127, 128, 511]
    o2, l2 = oracle.prefill_rows(q, k, v, w.w_pretrained, w.w0, w.theta, rows)
    np.testing.assert_allclose(o2, o[:, rows], atol=0)
    np.testing.assert_allclose(l2, lse[:, :, rows], atol=0)
    o3, l3 = oracle.prefill_rows(q[:, rows], k, v, w.w_pretrained, w.w0, w.theta, rows,
                                 q_holds_rows=True)
    np.testing.assert_array_equal(o3, o2)
    np.testing.assert_array_equal(l3, l2)


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("L", [96, 128, 129, 300, 512])
def test_decode_equals_last_prefill_row(L):
    # With an unrounded fp64 cache RoPE'd at true positions (§3.2), one decode
    # step at position L-1 is the last row of a prefill of length L.
    w, q, k, v = tiny_inputs("tiny")
    q, k, v = q[:, :L], k[:, :L], v[:, :L]
    o, lse = oracle.prefill_rows(q, k, v, w.w_pretrained, w.w0, w.theta, [L - 1])
    cache = oracle.rope_cache(k, 0, w.theta)
    od, ld = oracle.decode(q[:, L - 1], cache, v, L, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(od, o[:, 0], atol=1e-10)
    np.testing.assert_allclose(ld, lse[:, :, 0], atol=1e-10)


def test_decode_reads_only_first_L_cache_slots():
    w, q, k, v = tiny_inputs("tiny")
    cache = oracle.rope_cache(k, 0, w.theta)
    L = 300
    o1, l1 = oracle.decode(q[:, L - 1], cache, v, L, w.w_pretrained, w.w0, w.theta)
    cache2, v2 = cache.copy(), v.copy()
    cache2[:, L:] = 1e6
    v2[:, L:] = -1e6
    o2, l2 = oracle.decode(q[:, L - 1], cache2, v2, L, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_decode_group_transition_page_boundary():
    # Appendix E boundary, scaled down: w_pretrained = 32, L = 96 -> 97 moves G
    # 3 -> 4 (the page's 98,304 -> 98,305 with w_pretrained = 32,768 in
    # miniature).  The same cache serves both steps; only G changes.
    rng = np.random.default_rng(7)
    D, theta, wp, w0 = 16, 1e4, 32, 4
    k = rng.standard_normal((1, 97, 1, D))
    v = rng.standard_normal((1, 97, 1, D))
    q = rng.standard_normal((1, 97, 2, D))
    cache = oracle.rope_cache(k, 0, theta)
    assert oracle.group_size(96, wp) == 3 and oracle.group_size(97, wp) == 4
    for L in (96, 97):
        od, ld = oracle.decode(q[:, L - 1], cache, v, L, wp, w0, theta)
        o, lse = oracle.prefill_rows(q[:, :L], k[:, :L], v[:, :L], wp, w0, theta, [L - 1])
        np.testing.assert_allclose(od, o[:, 0], atol=1e-10)


# ---------------------------------------------------------------- chunked prefill
def test_chunk_of_the_whole_prompt_is_the_prefill():
    # The cache formulation (keys stored at true positions, remote scores via
    # the correction rotation R(f(j) - j), §3.2) against the direct rule of §3
    # on pre-RoPE keys: two independent routes to the same numbers.
    w, q, k, v = tiny_inputs("tiny")
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk(q, cache, v, 0, w.w_pretrained, w.w0, w.theta)
    o, lse = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(oc, o, atol=1e-10)
    np.testing.assert_allclose(lc, lse, atol=1e-10)


@pytest.mark.parametrize("P0", [1, 128, 300, 511])
def test_chunk_tail_rows_are_the_prefill_rows(P0):
    # A chunk that ends at L uses G(L), the prefill's G, so its rows are the
    # prefill's rows P0..L-1 (G(P0) differs from G(L) for P0 = 300: 3 vs 4).
    w, q, k, v = tiny_inputs("tiny")
    L = q.shape[1]
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk(q[:, P0:], cache, v, P0, w.w_pretrained, w.w0, w.theta)
    o, lse = oracle.prefill_rows(q, k, v, w.w_pretrained, w.w0, w.theta, list(range(P0, L)))
    np.testing.assert_allclose(oc, o, atol=1e-10)
    np.testing.assert_allclose(lc, lse, atol=1e-10)


def test_sampled_chunk_rows_are_the_prefill_rows():
    # The rows option computes only the listed queries of a chunk, with the
    # chunk's G (from P0 + n); each equals the direct rule's row, and the
    # unlisted rows stay zero.
    w, q, k, v = tiny_inputs("tiny")
    L = q.shape[1]
    P0 = 200
    rows = [0, 5, 111, L - P0 - 1]
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk(q[:, P0:], cache, v, P0, w.w_pretrained, w.w0, w.theta,
                                  rows=rows)
    o, lse = oracle.prefill_rows(q, k, v, w.w_pretrained, w.w0, w.theta, [P0 + i for i in rows])
    np.testing.assert_allclose(oc[:, rows], o, atol=1e-10)
    np.testing.assert_allclose(lc[:, :, rows], lse, atol=1e-10)
    others = [i for i in range(L - P0) if i not in rows]
    assert not oc[:, others].any() and not lc[:, :, others].any()


def test_one_token_chunk_is_a_decode_step():
    w, q, k, v = tiny_inputs("tiny")
    cache = oracle.rope_cache(k, 0, w.theta)
    for L in (97, 300, 512):
        oc, lc = oracle.prefill_chunk(q[:, L - 1:L], cache, v, L - 1, w.w_pretrained, w.w0,
                                      w.theta)
        od, ld = oracle.decode(q[:, L - 1], cache, v, L, w.w_pretrained, w.w0, w.theta)
        np.testing.assert_allclose(oc[:, 0], od, atol=1e-12)
        np.testing.assert_allclose(lc[:, :, 0], ld, atol=1e-12)
