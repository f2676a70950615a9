"""GPU checks of the two-form key cache: jetlong_remote_cache writes the
FP16 remote form R(f(j) - j) k_cache[j] of the true-position cache (Jet-Long
paper, §3.2 correction rotation, applied once per G instead of every step),
and jetlong_decode_two_form reads remote keys from it.

The remote form is checked against the oracle's correction rotation. The
two-form decode is checked against the oracle and against jetlong_decode:
both hand the tensor core the same FP16 operands, so their outputs agree to
float rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, Workload, decode_inputs, generation_inputs

pytestmark = pytest.mark.gpu


def cache_bf16(k_raw, theta):
    return torch.from_numpy(oracle.rope_cache(f64(k_raw), 0, theta)).to(torch.bfloat16)


def both(w, L, q, cache, v):
    kr = torch.empty(cache.shape, dtype=torch.float16, device="cuda")
    jl.jetlong_remote_cache(cache, kr, 0, L, L, w.w_pretrained, w.theta)
    o1, l1 = jl.jetlong_decode_two_form(q, cache, kr, v, L, w.w_pretrained, w.w0, w.theta,
                                        out_dtype=torch.float32)
    o2, l2 = jl.jetlong_decode(q, cache, v, L, w.w_pretrained, w.w0, w.theta,
                               out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    return kr, o1, l1, o2, l2


def test_remote_form_is_the_correction_rotation():
    w = WORKLOADS["tiny"].with_(kind="decode")
    d = decode_inputs(w, Lcap=512)
    cache = cache_bf16(d.k_raw, w.theta).cuda()
    L = 512
    kr = torch.zeros(cache.shape, dtype=torch.float16, device="cuda")
    jl.jetlong_remote_cache(cache, kr, 0, L, L, w.w_pretrained, w.theta)
    assert jl.jetlong_device_status() == jl.JL_OK
    G = oracle.group_size(L, w.w_pretrained)
    ref = oracle.correction_rotate(f64(cache)[0], np.arange(L)[:, None], G, w.theta)
    got = f64(kr)[0]
    # one FP16 rounding (2^-11 relative) of an fp32 rotation
    assert np.all(np.abs(got - ref) <= 2.0 ** -10 * np.abs(ref) + 1e-4)


def test_partial_rows_leave_the_rest_untouched():
    w = WORKLOADS["tiny"].with_(kind="decode")
    d = decode_inputs(w, Lcap=512)
    cache = cache_bf16(d.k_raw, w.theta).cuda()
    kr = torch.full(cache.shape, 7.0, dtype=torch.float16, device="cuda")
    jl.jetlong_remote_cache(cache, kr, 100, 117, 512, w.w_pretrained, w.theta)
    assert jl.jetlong_device_status() == jl.JL_OK
    assert torch.all(kr[:, :100] == 7.0) and torch.all(kr[:, 117:] == 7.0)
    assert not torch.all(kr[:, 100:117] == 7.0)


@pytest.mark.parametrize("L", [1, 34, 129, 300, 512])
def test_tiny_decode_matches_oracle_and_the_rotating_decode(L):
    w = WORKLOADS["tiny"].with_(kind="decode")
    d = decode_inputs(w, Lcap=512)
    cache = cache_bf16(d.k_raw, w.theta)
    kr, o1, l1, o2, l2 = both(w, L, d.q.cuda(), cache.cuda(), d.v.cuda())
    o_ref, l_ref = oracle.decode(f64(d.q), f64(cache), f64(d.v), L, w.w_pretrained, w.w0, w.theta)
    assert_o(f64(o1), o_ref, f"L={L}")
    assert_lse(f64(l1), l_ref, f"L={L}")
    assert (o1 - o2).abs().max().item() <= 1e-6 and (l1 - l2).abs().max().item() <= 1e-5


@pytest.mark.parametrize("Hq,Hkv,D,wp,w0,L", [
    (8, 2, 128, 64, 0, 1000), (16, 16, 128, 300, 50, 3000), (24, 12, 64, 500, 20, 4100)])
def test_decode_shapes(Hq, Hkv, D, wp, w0, L):
    w = Workload("two_form", 2, Hq, Hkv, D, L, wp, w0, 1e6, 80 + L, False, kind="decode")
    d = decode_inputs(w, Lcap=L + 5)
    cache = cache_bf16(d.k_raw, w.theta)
    kr, o1, l1, o2, l2 = both(w, L, d.q.cuda(), cache.cuda(), d.v.cuda())
    o_ref, l_ref = oracle.decode(f64(d.q), f64(cache), f64(d.v), L, wp, w0, w.theta)
    assert_o(f64(o1), o_ref, "two-form shapes")
    assert_lse(f64(l1), l_ref, "two-form shapes")
    assert (o1 - o2).abs().max().item() <= 1e-6


def test_qwen3_8b_decode_at_128k():
    w = WORKLOADS["decode_8b_128k"]
    d = decode_inputs(w)
    cache = cache_bf16(d.k_raw, w.theta)
    kr, o1, l1, o2, l2 = both(w, w.L, d.q.cuda(), cache.cuda(), d.v.cuda())
    o_ref, l_ref = oracle.decode(f64(d.q), f64(cache), f64(d.v), w.L, w.w_pretrained, w.w0,
                                 w.theta)
    assert_o(f64(o1), o_ref, "8B 128K two-form")
    assert_lse(f64(l1), l_ref, "8B 128K two-form")
    assert (o1 - o2).abs().max().item() <= 1e-6


def test_generation_loop_rebuilds_on_a_group_change():
    # Appendix E boundary in miniature: w_pretrained = 32, L = 90 .. 100
    # crosses G 3 -> 4 at L = 97.  After each append the new row's remote
    # form is written; when G changes every row is rewritten.
    w = Workload("two_form_gen", 1, 8, 2, 128, 0, 32, 4, 1e4, 91, False, kind="decode")
    L0, n = 90, 10
    x = generation_inputs(w, L0, n)
    cache = cache_bf16(x.k_raw, w.theta).cuda()
    v = x.v.cuda()
    kr = torch.empty(cache.shape, dtype=torch.float16, device="cuda")
    jl.jetlong_remote_cache(cache, kr, 0, L0, L0, w.w_pretrained, w.theta)
    for i in range(n):
        L = L0 + i + 1
        if jl.jetlong_group_size(L, w.w_pretrained) != jl.jetlong_group_size(L - 1, w.w_pretrained):
            jl.jetlong_remote_cache(cache, kr, 0, L, L, w.w_pretrained, w.theta)
        else:
            jl.jetlong_remote_cache(cache, kr, L - 1, L, L, w.w_pretrained, w.theta)
        q = x.q[i].cuda()
        o1, _ = jl.jetlong_decode_two_form(q, cache, kr, v, L, w.w_pretrained, w.w0, w.theta,
                                           out_dtype=torch.float32)
        o2, _ = jl.jetlong_decode(q, cache, v, L, w.w_pretrained, w.w0, w.theta,
                                  out_dtype=torch.float32)
        assert jl.jetlong_device_status() == jl.JL_OK
        assert (o1 - o2).abs().max().item() <= 1e-6, L
