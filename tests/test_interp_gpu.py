"""GPU parity of the frequency-interpolation remote map (the §4.7 / Table 6
ablation of the Jet-Long page) through the C ABI: jetlong_prefill_interp,
jetlong_decode_interp and jetlong_prefill_chunk_interp against the fp64
oracle's prefill_interp / decode_interp / prefill_chunk_interp.

Decode and chunk comparisons read the same BF16 cache, built by the oracle
(true-position RoPE in fp64, rounded to BF16), as in the aliasing tests.
"""
import pytest
import torch
from hypothesis import given, settings, strategies as st

import oracle
from parity_util import assert_lse, assert_o, f64, workloads
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import (WORKLOADS, Workload, decode_inputs,
                                               generation_inputs, prefill_inputs, sample_rows)

pytestmark = pytest.mark.gpu


def prefill_both(w: Workload, alpha=1.0, beta=32.0):
    x = prefill_inputs(w)
    out, lse = jl.jetlong_prefill_interp(x.q.cuda(), x.k.cuda(), x.v.cuda(), w.w_pretrained, w.w0,
                                         w.theta, alpha, beta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_interp(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0,
                                           w.theta, alpha, beta)
    return out, lse, o_ref, lse_ref


def cache_bf16(k_raw, theta):
    return torch.from_numpy(oracle.rope_cache(f64(k_raw), 0, theta)).to(torch.bfloat16)


@pytest.mark.parametrize("alpha,beta", [(1.0, 32.0), (1e6, 2e6), (-2.0, -1.0), (0.5, 3.0)])
def test_tiny_prefill_every_row(alpha, beta):
    # defaults; every frequency divided by s; every frequency kept; a narrow ramp
    w = WORKLOADS["tiny"]
    out, lse, o_ref, lse_ref = prefill_both(w, alpha, beta)
    assert_o(f64(out), o_ref, f"tiny alpha={alpha}")
    assert_lse(f64(lse), lse_ref, f"tiny alpha={alpha}")


@pytest.mark.parametrize("L,wp,w0,Hq,Hkv,D", [
    (1, 128, 32, 2, 1, 64),       # one token
    (96, 128, 32, 2, 1, 64),      # native window: s = 1
    (129, 128, 0, 2, 1, 64),      # just past it, only self-attention local
    (300, 64, 17, 4, 2, 64),      # ragged tail, s = 4.69
    (777, 200, 800, 2, 1, 64),    # w0 >= L: every pair local
    (1000, 256, 100, 3, 1, 128),  # GQA 3, D = 128
])
def test_edge_prefill_every_row(L, wp, w0, Hq, Hkv, D):
    w = Workload("edge_interp", 1, Hq, Hkv, D, L, wp, w0, 1e4, 51 + L, True)
    out, lse, o_ref, lse_ref = prefill_both(w)
    assert_o(f64(out), o_ref, f"edge L={L}")
    assert_lse(f64(lse), lse_ref, f"edge L={L}")


def test_qwen3_8b_prefill_at_128k_sampled_rows():
    w = WORKLOADS["qwen3_8b_128k"]
    x = prefill_inputs(w, device="cuda")
    out, lse = jl.jetlong_prefill_interp(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta,
                                         out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    rows = sample_rows(w.L, w.w0, w.w_pretrained, 10, w.seed)
    ridx = torch.tensor(rows, device="cuda")
    o_ref, lse_ref = oracle.prefill_interp_rows(f64(x.q.index_select(1, ridx)), f64(x.k),
                                                f64(x.v), w.w_pretrained, w.w0, w.theta, rows,
                                                q_holds_rows=True)
    assert_o(f64(out.index_select(1, ridx)), o_ref, "8B 128K interp")
    assert_lse(f64(lse.index_select(2, ridx)), lse_ref, "8B 128K interp")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


TINY = WORKLOADS["tiny"].with_(kind="decode")


@pytest.mark.parametrize("L", [1, 33, 34, 128, 129, 300, 512])
def test_tiny_decode_lengths(L):
    d = decode_inputs(TINY, Lcap=512)
    cache = cache_bf16(d.k_raw, TINY.theta)
    out, lse = jl.jetlong_decode_interp(d.q.cuda(), cache.cuda(), d.v.cuda(), L, TINY.w_pretrained,
                                        TINY.w0, TINY.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode_interp(f64(d.q), f64(cache), f64(d.v), L, TINY.w_pretrained,
                                          TINY.w0, TINY.theta)
    assert_o(f64(out), o_ref, f"L={L}")
    assert_lse(f64(lse), lse_ref, f"L={L}")


def test_native_length_decode_is_the_aliasing_decode():
    # L <= w_pretrained: s = 1 and G = 1, the same plain-RoPE kernel runs
    d = decode_inputs(TINY, Lcap=512)
    cache = cache_bf16(d.k_raw, TINY.theta).cuda()
    q, v = d.q.cuda(), d.v.cuda()
    a = jl.jetlong_decode(q, cache, v, 100, TINY.w_pretrained, TINY.w0, TINY.theta)
    b = jl.jetlong_decode_interp(q, cache, v, 100, TINY.w_pretrained, TINY.w0, TINY.theta)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("Hq,Hkv,D,wp,w0,L", [
    (8, 2, 128, 64, 0, 1000), (16, 16, 128, 300, 50, 3000), (24, 12, 64, 500, 20, 4100)])
def test_decode_shapes(Hq, Hkv, D, wp, w0, L):
    w = Workload("dec_interp", 2, Hq, Hkv, D, L, wp, w0, 1e6, 60 + L, False, kind="decode")
    d = decode_inputs(w, Lcap=L + 5)
    cache = cache_bf16(d.k_raw, w.theta)
    out, lse = jl.jetlong_decode_interp(d.q.cuda(), cache.cuda(), d.v.cuda(), L, wp, w0, w.theta,
                                        out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode_interp(f64(d.q), f64(cache), f64(d.v), L, wp, w0, w.theta)
    assert_o(f64(out), o_ref, "decode shapes")
    assert_lse(f64(lse), lse_ref, "decode shapes")


@pytest.mark.parametrize("name", ["decode_8b_128k"])
def test_qwen3_8b_decode(name):
    w = WORKLOADS[name]
    d = decode_inputs(w)
    cache = cache_bf16(d.k_raw, w.theta)
    out, lse = jl.jetlong_decode_interp(d.q.cuda(), cache.cuda(), d.v.cuda(), w.L, w.w_pretrained,
                                        w.w0, w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode_interp(f64(d.q), f64(cache), f64(d.v), w.L, w.w_pretrained,
                                          w.w0, w.theta)
    assert_o(f64(out), o_ref, name)
    assert_lse(f64(lse), lse_ref, name)


@pytest.mark.parametrize("B,Hq,Hkv,D,wp,w0,P0,n", [
    (1, 2, 1, 64, 128, 32, 0, 512),     # the whole tiny prompt as one chunk
    (1, 2, 1, 64, 128, 32, 300, 212),
    (2, 8, 2, 128, 256, 40, 700, 33),
    (1, 32, 8, 128, 32768, 4096, 131072 - 64, 64),  # Qwen3-8B layer, 128K
])
def test_chunks(B, Hq, Hkv, D, wp, w0, P0, n):
    w = Workload("chunk_interp", B, Hq, Hkv, D, 0, wp, w0, 1e6 if D == 128 else 1e4, 71 + P0,
                 False, kind="decode")
    x = generation_inputs(w, P0, n)
    cache = cache_bf16(x.k_raw, w.theta)
    q = torch.randn((B, n, Hq, D), generator=torch.Generator().manual_seed(w.seed + 5))
    q = q.to(torch.bfloat16)
    out, lse = jl.jetlong_prefill_chunk_interp(q.cuda(), cache.cuda(), x.v.cuda(), P0, wp, w0,
                                               w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_chunk_interp(f64(q), f64(cache), f64(x.v), P0, wp, w0,
                                                 w.theta)
    assert_o(f64(out), o_ref, f"chunk P0={P0}")
    assert_lse(f64(lse), lse_ref, f"chunk P0={P0}")


# ---------------------------------------------------------------- random shapes
RAMPS = st.sampled_from([(1.0, 32.0), (0.5, 3.0), (-2.0, -1.0), (1e6, 2e6), (2.0, 8.0)])
RANDOM = settings(max_examples=8, deadline=None, derandomize=True)


@RANDOM
@given(workloads(grps=[1, 2, 3, 4], max_L=700), RAMPS)
def test_prefill_random_shapes(w, ramp):
    x = prefill_inputs(w)
    out, lse = jl.jetlong_prefill_interp(x.q.cuda(), x.k.cuda(), x.v.cuda(), w.w_pretrained, w.w0,
                                         w.theta, *ramp, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_interp(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0,
                                           w.theta, *ramp)
    assert_o(f64(out), o_ref, f"{w} {ramp}")
    assert_lse(f64(lse), lse_ref, f"{w} {ramp}")


@RANDOM
@given(workloads(grps=[1, 2, 4, 8], max_L=3000), RAMPS)
def test_decode_random_shapes(w, ramp):
    d = decode_inputs(w, Lcap=w.L + 2)
    cache = cache_bf16(d.k_raw, w.theta)
    out, lse = jl.jetlong_decode_interp(d.q.cuda(), cache.cuda(), d.v.cuda(), w.L, w.w_pretrained,
                                        w.w0, w.theta, *ramp, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode_interp(f64(d.q), f64(cache), f64(d.v), w.L, w.w_pretrained,
                                          w.w0, w.theta, *ramp)
    assert_o(f64(out), o_ref, f"{w} {ramp}")
    assert_lse(f64(lse), lse_ref, f"{w} {ramp}")


def chunk_case(w, ramp, n):
    P0 = w.L - n
    x = prefill_inputs(w)
    cache = cache_bf16(x.k, w.theta)
    qc = x.q[:, P0:].contiguous()
    out, lse = jl.jetlong_prefill_chunk_interp(qc.cuda(), cache.cuda(), x.v.cuda(), P0,
                                               w.w_pretrained, w.w0, w.theta, *ramp,
                                               out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_chunk_interp(f64(qc), f64(cache), f64(x.v), P0,
                                                 w.w_pretrained, w.w0, w.theta, *ramp)
    assert_o(f64(out), o_ref, f"{w} {ramp}")
    assert_lse(f64(lse), lse_ref, f"{w} {ramp}")


@RANDOM
@given(workloads(grps=[1, 2, 4, 8], max_L=1500), RAMPS, st.data())
def test_prefill_chunk_random_shapes(w, ramp, data):
    chunk_case(w, ramp, data.draw(st.integers(1, min(w.L, 40))))


# The random draw that exposed a lost rescale in the D = 64 decode kernel: a
# running max that jumps inside a 16-token stage must reweigh the stage's
# first 8-token block too.  Pinned, with its neighbours, so that a change of
# the random strategy cannot drop it.
PINNED_D64 = Workload("rand", 1, 4, 1, 64, 1484, 1, 0, 1e4, 0, True)


@pytest.mark.parametrize("wp", [1, 2, 8, 64])
@pytest.mark.parametrize("n", [1, 7])
def test_prefill_chunk_pinned_d64(wp, n):
    chunk_case(PINNED_D64.with_(w_pretrained=wp), (1.0, 32.0), n)
