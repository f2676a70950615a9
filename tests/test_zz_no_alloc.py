"""The decode entry point that allocates nothing (jetlong_decode_noalloc).

It serves callers that cannot allocate device memory for a workspace: the
split partials live in a fixed 8 MiB buffer inside the library's device image.
This file is collected last, so a run that stops at its first failure has
already run every other test; it passes both alone in a fresh process and
after the rest of the suite.
"""
import ctypes

import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, Workload, decode_inputs

pytestmark = pytest.mark.gpu


def _call_noalloc(w, L, q, kc, v, out, lse):
    # straight through the C ABI: the caller passes inputs and outputs only
    return jl.lib().jetlong_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), w.B, w.Hq, w.Hkv, L,
        kc.shape[1], w.D, w.w_pretrained, w.w0, w.theta, jl.JL_F32,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    # Qwen3-8B heads, a cache long enough for G = 2 and both windows
    w = Workload("noalloc", 1, 32, 8, 128, 40000, 32768, 4096, 1e6, 77, False, kind="decode")
    d = decode_inputs(w, device="cuda")
    kc = torch.empty_like(d.k_raw)
    jl.jetlong_rope_cache(d.k_raw, kc, 0, w.theta)
    for L in (40000, 39999):  # two calls in a row, different lengths
        ref_o, ref_l = jl.jetlong_decode(d.q, kc, d.v, L, w.w_pretrained, w.w0, w.theta,
                                         out_dtype=torch.float32)
        out = torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda")
        lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
        assert _call_noalloc(w, L, d.q, kc, d.v, out, lse) == jl.JL_OK
        assert jl.jetlong_device_status() == jl.JL_OK
        assert_o(f64(out), f64(ref_o), f"noalloc L={L}")
        assert_lse(f64(lse), f64(ref_l), f"noalloc L={L}")


def test_noalloc_decode_matches_the_oracle_on_the_tiny_case():
    # the tiny workload (G = 4 at L = 512) against the fp64 oracle directly
    w = WORKLOADS["tiny"].with_(kind="decode")
    d = decode_inputs(w)
    kc = torch.from_numpy(oracle.rope_cache(f64(d.k_raw), 0, w.theta)).to(torch.bfloat16)
    q, kc, v = d.q.cuda(), kc.cuda(), d.v.cuda()
    for L in (w.L, w.L - 200):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda")
        lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
        assert _call_noalloc(w, L, q, kc, v, out, lse) == jl.JL_OK
        assert jl.jetlong_device_status() == jl.JL_OK
        o_ref, l_ref = oracle.decode(f64(d.q), f64(kc), f64(d.v), L, w.w_pretrained, w.w0,
                                     w.theta)
        assert_o(f64(out), o_ref, f"noalloc tiny L={L}")
        assert_lse(f64(lse), l_ref, f"noalloc tiny L={L}")


def test_noalloc_rejects_sizes_beyond_its_buffer():
    # a batch of 512 decodes at once needs ~8.5 MB of partials: above the 8 MiB buffer
    w = Workload("big", 512, 32, 8, 128, 16, 32768, 4096, 1e6, 78, False, kind="decode")
    assert jl.jetlong_decode_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D) > (8 << 20)
    q = torch.zeros((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((w.B, w.L, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((w.B, w.Hq), dtype=torch.float32, device="cuda")
    assert _call_noalloc(w, w.L, q, kc, kc, out, lse) == jl.JL_ERR_WORKSPACE
    assert jl.jetlong_device_status() == jl.JL_OK


def test_calls_after_shutdown_look_everything_up_again():
    # jetlong_shutdown forgets the cached buffer address and kernel settings;
    # the next calls find them again and give the same results
    w = Workload("noalloc_shutdown", 1, 32, 8, 128, 5000, 1024, 256, 1e6, 79, False, kind="decode")
    d = decode_inputs(w, device="cuda")
    kc = torch.empty_like(d.k_raw)
    jl.jetlong_rope_cache(d.k_raw, kc, 0, w.theta)
    outs = []
    for _ in range(2):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda")
        lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
        assert _call_noalloc(w, w.L, d.q, kc, d.v, out, lse) == jl.JL_OK
        ref = jl.jetlong_decode(d.q, kc, d.v, w.L, w.w_pretrained, w.w0, w.theta,
                                out_dtype=torch.float32)
        assert jl.jetlong_device_status() == jl.JL_OK
        outs.append((out, lse, ref[0]))
        jl.lib().jetlong_shutdown()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])
