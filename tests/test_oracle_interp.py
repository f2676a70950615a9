"""Pins for the oracle's frequency-interpolation remote map (the ablation of
§4.7 / Table 6 of the Jet-Long page): each test checks it against something
other than itself -- special cases of the ramp with hand-derived values,
textbook attention through torch's SDPA with complex-number rotations, a
pure-Python per-pair loop, and the cache + correction-rotation route."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from test_oracle_pins import sdpa_with_positions, tiny_inputs


# ---------------------------------------------------------------- helpers
def rotate_complex(x, pos, omega):
    """Pair (x_t, x_{t+D/2}) as the complex number x_t + 1j x_{t+D/2}, times
    exp(1j * pos * omega_t): RoPE with caller-chosen frequencies."""
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(
        1j * np.asarray(pos, dtype=np.float64)[..., None] * np.asarray(omega))
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa_with_freqs(q, k, v, omega, mask):
    """Masked textbook attention (torch fp64 SDPA) with queries and keys at
    their true positions, rotated with frequencies omega."""
    B, L, Hq, D = q.shape
    grp = Hq // k.shape[2]
    pos = np.arange(L)[None, :, None]
    qr = torch.from_numpy(rotate_complex(q, pos, omega)).permute(0, 2, 1, 3)
    kr = torch.from_numpy(rotate_complex(k, pos, omega)).permute(0, 2, 1, 3)
    vv = torch.from_numpy(np.asarray(v, dtype=np.float64)).permute(0, 2, 1, 3)
    kr = kr.repeat_interleave(grp, dim=1)
    vv = vv.repeat_interleave(grp, dim=1)
    m = torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(qr, kr, vv, attn_mask=m)
    s = (qr @ kr.transpose(-1, -2)) / math.sqrt(D)
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


# ---------------------------------------------------------------- the ramp
def test_scale_is_the_continuous_dynamic_factor():
    # §3.1: s = max(1, L / w_pretrained), a real number (not the integer G).
    assert oracle.interp_scale(96, 128) == 1.0
    assert oracle.interp_scale(128, 128) == 1.0
    assert oracle.interp_scale(96, 40) == 2.4
    assert oracle.interp_scale(131072, 32768) == 4.0
    assert oracle.interp_scale(98305, 32768) == 98305 / 32768


def test_native_length_keeps_every_frequency():
    # L <= w_pretrained: s = 1 and (1 - gamma) / s + gamma = 1 for any gamma.
    base = 1e4 ** (-2.0 * np.arange(32) / 64)
    np.testing.assert_array_equal(oracle.interp_freq(64, 1e4, 100, 128), base)


def test_slow_frequencies_are_divided_by_s():
    # alpha above every channel's turn count: gamma = 0, theta' = theta / s
    # with s = 96 / 40 = 2.4 (G would be 3).
    base = 1e4 ** (-2.0 * np.arange(8) / 16)
    got = oracle.interp_freq(16, 1e4, 96, 40, alpha=1e6, beta=2e6)
    np.testing.assert_allclose(got, base / 2.4, rtol=1e-15)


def test_fast_frequencies_are_kept():
    # beta below every channel's turn count (all counts are >= 0): gamma = 1.
    base = 1e4 ** (-2.0 * np.arange(8) / 16)
    got = oracle.interp_freq(16, 1e4, 96, 40, alpha=-2.0, beta=-1.0)
    np.testing.assert_allclose(got, base, rtol=1e-15)


def test_ramp_is_linear_in_turns_within_the_pretrained_window():
    # D = 4, theta = 100: channel 1 has frequency 0.1 rad per position, so
    # within w_pretrained = 64 positions it turns 6.4 / (2 pi) times.  With
    # alpha = turns - 1 and beta = turns + 3, gamma = 1/4 exactly, and with
    # L = 256 (s = 4): theta'_1 = 0.1 * (0.75 / 4 + 0.25) = 0.04375.
    turns = 6.4 / (2.0 * math.pi)
    got = oracle.interp_freq(4, 100.0, 256, 64, alpha=turns - 1.0, beta=turns + 3.0)
    assert got[1] == pytest.approx(0.04375, rel=1e-13)
    # channel 0 (1 rad per position, 10.19 turns) sits above beta: kept.
    assert got[0] == 1.0


def test_default_ramp_on_the_tiny_workload():
    # Defaults alpha = 1, beta = 32; w_pretrained = 128, L = 512 (s = 4),
    # D = 64, theta = 1e4.  Channel 0 turns 128 / (2 pi) = 20.37 times:
    # gamma = 19.37 / 31.  Channel 16 (0.01 rad) turns 0.204 times: gamma = 0.
    got = oracle.interp_freq(64, 1e4, 512, 128)
    g0 = (128.0 / (2.0 * math.pi) - 1.0) / 31.0
    assert got[0] == pytest.approx((1.0 - g0) / 4.0 + g0, rel=1e-13)
    assert got[16] == pytest.approx(0.01 / 4.0, rel=1e-12)
    ratio = got / (1e4 ** (-2.0 * np.arange(32) / 64))
    assert np.all(np.diff(ratio) <= 1e-15) and ratio.min() >= 0.25 - 1e-15


# ---------------------------------------------------------------- attention
def test_native_length_is_plain_rope_attention():
    w, q, k, v = tiny_inputs("tiny_native")
    o, lse = oracle.prefill_interp(q, k, v, w.w_pretrained, w.w0, w.theta)
    pos = np.arange(w.L)
    o_ref, lse_ref = sdpa_with_positions(q, k, v, pos, pos, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


def test_kept_frequencies_give_plain_rope_attention_at_any_length():
    # gamma = 1 everywhere: the remote branch equals the local one, so the
    # whole result is causal RoPE attention at true positions, L = 4 w_p.
    w, q, k, v = tiny_inputs("tiny")
    o, lse = oracle.prefill_interp(q, k, v, w.w_pretrained, w.w0, w.theta, alpha=-2.0, beta=-1.0)
    pos = np.arange(w.L)
    o_ref, lse_ref = sdpa_with_positions(q, k, v, pos, pos, w.theta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-10)


@pytest.mark.parametrize("alpha,beta", [(1.0, 32.0), (1e6, 2e6)])
def test_band_and_remote_parts_via_masked_library_attention(alpha, beta):
    # Disjoint key sets: the band at pretrained frequencies, the rest at the
    # interpolated ones, each by the library with a mask, merged by LSE.
    w, q, k, v = tiny_inputs("tiny")
    omega = np.exp(-(2.0 * np.arange(w.D // 2) / w.D) * math.log(w.theta))
    omega_i = oracle.interp_freq(w.D, w.theta, w.L, w.w_pretrained, alpha, beta)
    pos = np.arange(w.L)
    dist = pos[:, None] - pos[None, :]
    band = (dist >= 0) & (dist <= w.w0)
    far = dist > w.w0
    ob, lb = sdpa_with_freqs(q, k, v, omega, band)
    far_rows = far.any(axis=1)
    far_m = far.copy()
    far_m[~far_rows, 0] = True
    orr, lr = sdpa_with_freqs(q, k, v, omega_i, far_m)
    lr[:, :, ~far_rows] = -np.inf
    M = np.maximum(lb, lr)
    wb, wr = np.exp(lb - M), np.exp(lr - M)
    tot = wb + wr
    o_ref = ((wb / tot).transpose(0, 2, 1)[..., None] * ob
             + (wr / tot).transpose(0, 2, 1)[..., None] * np.nan_to_num(orr))
    o, lse = oracle.prefill_interp(q, k, v, w.w_pretrained, w.w0, w.theta, alpha, beta)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(lse, M + np.log(tot), atol=1e-10)
    # and it is not the aliasing variant
    oa, _ = oracle.prefill(q, k, v, w.w_pretrained, w.w0, w.theta)
    assert np.abs(o - oa).max() > 1e-3


def test_literal_per_pair_brute_force():
    rng = np.random.default_rng(16)
    B, L, Hq, Hkv, D = 1, 40, 2, 1, 8
    q = rng.standard_normal((B, L, Hq, D))
    k = rng.standard_normal((B, L, Hkv, D))
    v = rng.standard_normal((B, L, Hkv, D))
    for w0, alpha, beta in ((0, 1.0, 32.0), (5, 0.5, 2.0), (39, 1.0, 32.0)):
        o1, l1 = oracle.prefill_interp(q, k, v, 12, w0, 1e2, alpha, beta)
        o2, l2 = oracle.prefill_interp_literal(q, k, v, 12, w0, 1e2, alpha, beta)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_correction_rotation_turns_the_cache_into_the_interpolated_key():
    # R(j (theta' - theta)) RoPE(x, j) = RoPE'(x, j): rotations compose.
    rng = np.random.default_rng(17)
    x = rng.standard_normal((50, 16))
    j = np.arange(1000, 1050)
    fr = oracle.interp_freq(16, 1e4, 5000, 100)
    omega = np.exp(-(2.0 * np.arange(8) / 16) * math.log(1e4))
    got = oracle.correction_rotate_interp(rotate_complex(x, j, omega), j, fr, 1e4)
    np.testing.assert_allclose(got, rotate_complex(x, j, fr), atol=1e-9)


# ---------------------------------------------------------------- cache route
def test_chunk_of_the_whole_prompt_is_the_prefill():
    w, q, k, v = tiny_inputs("tiny")
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk_interp(q, cache, v, 0, w.w_pretrained, w.w0, w.theta)
    o, lse = oracle.prefill_interp(q, k, v, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(oc, o, atol=1e-10)
    np.testing.assert_allclose(lc, lse, atol=1e-10)


@pytest.mark.parametrize("P0", [1, 300, 511])
def test_chunk_tail_rows_are_the_prefill_rows(P0):
    w, q, k, v = tiny_inputs("tiny")
    L = q.shape[1]
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk_interp(q[:, P0:], cache, v, P0, w.w_pretrained, w.w0, w.theta)
    o, lse = oracle.prefill_interp_rows(q, k, v, w.w_pretrained, w.w0, w.theta, list(range(P0, L)))
    np.testing.assert_allclose(oc, o, atol=1e-10)
    np.testing.assert_allclose(lc, lse, atol=1e-10)


def test_sampled_chunk_rows_are_the_prefill_rows():
    w, q, k, v = tiny_inputs("tiny")
    L = q.shape[1]
    P0 = 200
    rows = [0, 7, 150, L - P0 - 1]
    cache = oracle.rope_cache(k, 0, w.theta)
    oc, lc = oracle.prefill_chunk_interp(q[:, P0:], cache, v, P0, w.w_pretrained, w.w0, w.theta,
                                         rows=rows)
    o, lse = oracle.prefill_interp_rows(q, k, v, w.w_pretrained, w.w0, w.theta,
                                        [P0 + i for i in rows])
    np.testing.assert_allclose(oc[:, rows], o, atol=1e-10)
    np.testing.assert_allclose(lc[:, :, rows], lse, atol=1e-10)


@pytest.mark.parametrize("L", [129, 300, 512])
def test_decode_equals_last_prefill_row(L):
    w, q, k, v = tiny_inputs("tiny")
    q, k, v = q[:, :L], k[:, :L], v[:, :L]
    o, lse = oracle.prefill_interp_rows(q, k, v, w.w_pretrained, w.w0, w.theta, [L - 1])
    cache = oracle.rope_cache(k, 0, w.theta)
    od, ld = oracle.decode_interp(q[:, L - 1], cache, v, L, w.w_pretrained, w.w0, w.theta)
    np.testing.assert_allclose(od, o[:, 0], atol=1e-10)
    np.testing.assert_allclose(ld, lse[:, :, 0], atol=1e-10)


def test_rows_subset_matches_full():
    w, q, k, v = tiny_inputs("tiny")
    o, lse = oracle.prefill_interp(q, k, v, w.w_pretrained, w.w0, w.theta)
    rows = [0, 32, 33, 128, 300, 511]
    o2, l2 = oracle.prefill_interp_rows(q[:, rows], k, v, w.w_pretrained, w.w0, w.theta, rows,
                                        q_holds_rows=True)
    np.testing.assert_array_equal(o2, o[:, rows])
    np.testing.assert_array_equal(l2, lse[:, :, rows])
