"""Planted mistakes: each plausible slip in the oracle must fail a pin.

Every case rewrites one oracle function (on the CPU, in this process only),
runs the pins that should notice, and checks that at least one of them fails.
"""
import contextlib
import inspect
import textwrap

import pytest

import oracle
import oracle.bifocal_ref as ref
import test_oracle_interp as ipins
import test_oracle_pins as pins


@contextlib.contextmanager
def mutated(func_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(ref, func_name)))
    assert old in src, (func_name, old)
    ns = dict(ref.__dict__)
    exec(compile(src.replace(old, new, 1), f"<mutant {func_name}>", "exec"), ns)
    saved_ref = getattr(ref, func_name)
    saved_pkg = getattr(oracle, func_name, None)
    setattr(ref, func_name, ns[func_name])
    setattr(oracle, func_name, ns[func_name])
    try:
        yield
    finally:
        setattr(ref, func_name, saved_ref)
        if saved_pkg is not None:
            setattr(oracle, func_name, saved_pkg)


def some_pin_fails(tests):
    # a pin that fails an assertion, or that the mutant makes raise, caught it
    for t in tests:
        try:
            t()
        except Exception:  # noqa: BLE001
            return True
    return False


PREFILL_PINS = [
    pins.test_native_window_reduces_to_plain_rope_attention,
    pins.test_wide_window_equals_true_position_attention,
    pins.test_zero_window_equals_remote_position_attention,
    pins.test_rows_inside_local_window_see_true_positions,
    pins.test_band_and_remote_parts_via_masked_library_attention,
    pins.test_literal_per_pair_brute_force,
    pins.test_grouped_query_heads_share_kv_heads_in_blocks,
]


def decode_pins():
    return [lambda L=L: pins.test_decode_equals_last_prefill_row(L) for L in (129, 300, 512)] + [
        pins.test_decode_group_transition_page_boundary]


def chunk_pins():
    return [pins.test_chunk_of_the_whole_prompt_is_the_prefill,
            lambda: pins.test_chunk_tail_rows_are_the_prefill_rows(300),
            pins.test_one_token_chunk_is_a_decode_step]


RAMP_PINS = [ipins.test_scale_is_the_continuous_dynamic_factor,
             ipins.test_native_length_keeps_every_frequency,
             ipins.test_slow_frequencies_are_divided_by_s,
             ipins.test_fast_frequencies_are_kept,
             ipins.test_ramp_is_linear_in_turns_within_the_pretrained_window,
             ipins.test_default_ramp_on_the_tiny_workload]


def interp_pins():
    return [ipins.test_native_length_is_plain_rope_attention,
            ipins.test_kept_frequencies_give_plain_rope_attention_at_any_length,
            lambda: ipins.test_band_and_remote_parts_via_masked_library_attention(1.0, 32.0),
            ipins.test_literal_per_pair_brute_force]


def interp_cache_pins():
    return [ipins.test_correction_rotation_turns_the_cache_into_the_interpolated_key,
            ipins.test_chunk_of_the_whole_prompt_is_the_prefill,
            lambda: ipins.test_chunk_tail_rows_are_the_prefill_rows(300),
            lambda: ipins.test_decode_equals_last_prefill_row(300)]


MUTANTS = [
    # schedule
    ("group_size", "max(1, -((-L) // w))", "max(1, L // w)",
     [pins.test_group_size_matches_page_values, pins.test_group_size_is_minimal_integer_compression]),
    ("group_size", "max(1, -((-L) // w))", "max(1, -((-L) // w) + (L % w == 0))",
     [pins.test_group_size_matches_page_values]),
    ("remap", "np.floor_divide(np.asarray(x, dtype=np.int64), int(G))",
     "-np.floor_divide(-np.asarray(x, dtype=np.int64), int(G))",
     [pins.test_remap_identity_iff_native_and_monotone] + PREFILL_PINS),
    # RoPE
    ("rope", "a * c - b * s, a * s + b * c", "a * c + b * s, -a * s + b * c",
     [pins.test_rope_matches_complex_rotation]),
    ("rope", "a * c - b * s, a * s + b * c", "a * c - b * s, b * s + a * c",
     [pins.test_rope_matches_complex_rotation, pins.test_rope_norm_identity_and_composition]),
    ("inv_freq", "-2.0 * i / np.float64(D)", "-2.0 * (i + 1) / np.float64(D)",
     [pins.test_rope_matches_complex_rotation]),
    ("inv_freq", "-2.0 * i / np.float64(D)", "-1.0 * i / np.float64(D)",
     [pins.test_rope_matches_complex_rotation]),
    # score rule
    ("prefill_rows", "dist <= w0", "dist < w0", PREFILL_PINS),
    ("prefill_rows", "np.where(dist <= w0, s_local, s_remote)", "np.where(dist <= w0, s_remote, s_local)",
     PREFILL_PINS),
    ("prefill_rows", "n = i + 1", "n = i if i > 0 else 1", PREFILL_PINS),
    ("prefill_rows", "scale = 1.0 / math.sqrt(D)", "scale = 1.0 / D", PREFILL_PINS),
    ("prefill_rows", "q_remote = rope(xq, remap(np.int64(i), G), theta)",
     "q_remote = rope(xq, np.int64(i), theta)", PREFILL_PINS),
    ("prefill_rows", "heads = np.arange(g * grp, (g + 1) * grp)",
     "heads = np.arange(g, Hq, Hkv)", PREFILL_PINS),
    ("prefill_rows", "lse[b, heads, r] = m + np.log(tot)", "lse[b, heads, r] = np.log(tot)",
     PREFILL_PINS),
    # decode / correction
    ("correction_rotate", "delta = remap(kpos, G) - kpos", "delta = kpos - remap(kpos, G)",
     [pins.test_correction_rotation_recovers_remote_phase] + decode_pins()),
    ("decode", "    p = L - 1\n", "    p = L\n", decode_pins()),
    ("decode", "local = (p - jpos) <= w0", "local = (p - jpos) < w0", decode_pins()),
    ("decode", "q_remote = rope(q[b, heads], remap(np.int64(p), G), theta)",
     "q_remote = rope(q[b, heads], np.int64(p), theta)", decode_pins()),
    ("rope_cache", "+ int(pos0)", "+ int(pos0) + 1", [pins.test_rope_cache_offset] + decode_pins()),
    # chunked prefill
    ("prefill_chunk", "G = group_size(L, w_pretrained)", "G = group_size(P0 + 1, w_pretrained)",
     chunk_pins()),
    ("prefill_chunk", "                p = P0 + i\n", "                p = P0 + i + 1\n", chunk_pins()),
    ("prefill_chunk", "c, cc, vv = c_all[: p + 1], c_corr_all[: p + 1], v_all[: p + 1]",
     "c, cc, vv = c_all[:p], c_corr_all[:p], v_all[:p]", chunk_pins()),
    # frequency-interpolation remote map (§4.7)
    ("interp_scale", "max(1.0, L / w)", "max(1.0, L // w)", RAMP_PINS),
    ("interp_freq", "(1.0 - gamma) / s + gamma", "gamma / s + (1.0 - gamma)", RAMP_PINS),
    ("interp_freq", "s = interp_scale(L, w_pretrained)", "s = group_size(L, w_pretrained)",
     RAMP_PINS),
    ("interp_freq", "turns = float(w_pretrained) * base", "turns = float(L) * base", RAMP_PINS),
    ("interp_freq", "turns = float(w_pretrained) * base / (2.0 * math.pi)",
     "turns = float(w_pretrained) / base / (2.0 * math.pi)", RAMP_PINS),
    ("interp_freq", "(turns - alpha) / (beta - alpha)", "(turns - alpha) / beta", RAMP_PINS),
    ("rope_at_freq", "a * c - b * s, a * s + b * c", "a * c + b * s, -a * s + b * c",
     interp_pins()),
    ("prefill_interp_rows", "dist <= w0", "dist < w0", interp_pins()),
    ("prefill_interp_rows", "q_remote = rope_at_freq(xq, np.int64(i), fr)",
     "q_remote = rope_at_freq(xq, remap(np.int64(i), group_size(L, w_pretrained)), fr)",
     interp_pins()),
    ("prefill_interp_rows", "k_true = rope(xk, jpos, theta)", "k_true = rope_at_freq(xk, jpos, fr)",
     interp_pins()),
    ("correction_rotate_interp", "np.asarray(freq_interp) - inv_freq(D, theta)",
     "inv_freq(D, theta) - np.asarray(freq_interp)", interp_cache_pins()),
    ("prefill_chunk_interp", "fr = interp_freq(D, theta, L, w_pretrained, alpha, beta)",
     "fr = interp_freq(D, theta, P0 + 1, w_pretrained, alpha, beta)", interp_cache_pins()),
    ("prefill_chunk_interp", "local = (p - jpos_all[: p + 1]) <= w0",
     "local = (p - jpos_all[: p + 1]) < w0", interp_cache_pins()),
]


@pytest.mark.parametrize("case", range(len(MUTANTS)))
def test_planted_mistake_is_caught(case):
    name, old, new, tests = MUTANTS[case]
    with mutated(name, old, new):
        assert some_pin_fails(tests), f"mutant of {name} ({new!r}) passed every pin"


def test_unmutated_oracle_passes_the_same_pins():
    for _, _, _, tests in MUTANTS:
        for t in tests:
            t()
