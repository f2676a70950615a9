"""Randomised GPU parity (through the C ABI) against the fp64 oracle over
small random shapes: ragged lengths, every supported GQA ratio, both head
dimensions, w0 from 0 to beyond L, G from 1 up.  Hypothesis is derandomised,
so every run draws the same cases; inputs come from the seeded generators.
"""
import pytest
import torch
from hypothesis import example, given, settings, strategies as st

import oracle
from parity_util import assert_lse, assert_o, f64, workloads
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import Workload, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu
SETTINGS = settings(max_examples=12, deadline=None, derandomize=True)

# D = 64 with four query heads per KV head at L = 1484: a shape on which a
# running max that jumps inside a 16-token decode stage once went unweighed
# for the stage's first 8-token block.  Pinned, so that a change of the
# random strategy cannot drop it.
PINNED_D64 = Workload("rand", 1, 4, 1, 64, 1484, 8, 0, 1e4, 0, True)


@SETTINGS
@given(workloads(grps=[1, 2, 3, 4], max_L=700))
def test_prefill_random_shapes(w):
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    out, lse = jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert_o(f64(out), o_ref, str(w))
    assert_lse(f64(lse), lse_ref, str(w))


@SETTINGS
@given(workloads(grps=[1, 2, 4, 8], max_L=3000))
@example(PINNED_D64)
@example(PINNED_D64.with_(w_pretrained=64))
def test_decode_random_shapes(w):
    d = decode_inputs(w, Lcap=w.L + 2)
    cache = torch.from_numpy(oracle.rope_cache(f64(d.k_raw), 0, w.theta)).to(torch.bfloat16)
    out, lse = jl.jetlong_decode(d.q.cuda(), cache.cuda(), d.v.cuda(), w.L, w.w_pretrained, w.w0,
                                 w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode(f64(d.q), f64(cache), f64(d.v), w.L, w.w_pretrained, w.w0,
                                   w.theta)
    assert_o(f64(out), o_ref, str(w))
    assert_lse(f64(lse), lse_ref, str(w))


def chunk_case(w, n):
    P0 = w.L - n
    x = prefill_inputs(w)
    cache = torch.from_numpy(oracle.rope_cache(f64(x.k), 0, w.theta)).to(torch.bfloat16)
    qc = x.q[:, P0:].contiguous()
    out, lse = jl.jetlong_prefill_chunk(qc.cuda(), cache.cuda(), x.v.cuda(), P0, w.w_pretrained,
                                        w.w0, w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_chunk(f64(qc), f64(cache), f64(x.v), P0, w.w_pretrained,
                                          w.w0, w.theta)
    assert_o(f64(out), o_ref, str(w))
    assert_lse(f64(lse), lse_ref, str(w))


@SETTINGS
@given(workloads(grps=[1, 2, 4, 8], max_L=1500), st.data())
def test_prefill_chunk_random_shapes(w, data):
    chunk_case(w, data.draw(st.integers(1, min(w.L, 40))))


@pytest.mark.parametrize("n", [1, 7, 40])
def test_prefill_chunk_pinned_d64(n):
    chunk_case(PINNED_D64, n)


@SETTINGS
@given(workloads(grps=[1, 2, 3], max_L=600))
def test_three_pass_random_shapes(w):
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    out, lse = jl.jetlong_prefill_three_pass(q, k, v, w.w_pretrained, w.w0, w.theta,
                                             out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert_o(f64(out), o_ref, str(w))
    assert_lse(f64(lse), lse_ref, str(w))
