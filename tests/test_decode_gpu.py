"""GPU parity of jetlong_decode and jetlong_rope_cache (through the C ABI)
against the fp64 oracle.

Both sides of a decode comparison read the same BF16 cache: the oracle
rotates the raw keys to their true positions in float64 (§3.2) and torch
rounds that to BF16; the CUDA decode and the oracle decode then both consume
those stored values, so the comparison isolates the decode kernel.  The cache
writer kernel is checked separately against the oracle's rotation.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, assert_o_bf16, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, Workload, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu


def oracle_cache_bf16(k_raw: torch.Tensor, theta: float) -> torch.Tensor:
    c = oracle.rope_cache(f64(k_raw), 0, theta)
    return torch.from_numpy(c).to(torch.bfloat16)


def decode_both(w: Workload, L: int, q, cache_bf16, v_bf16, out_dtype=torch.float32):
    out, lse = jl.jetlong_decode(q.cuda(), cache_bf16.cuda(), v_bf16.cuda(), L, w.w_pretrained,
                                 w.w0, w.theta, out_dtype=out_dtype)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode(f64(q), f64(cache_bf16), f64(v_bf16), L, w.w_pretrained, w.w0,
                                   w.theta)
    return out, lse, o_ref, lse_ref


TINY = WORKLOADS["tiny"].with_(kind="decode")


@pytest.mark.parametrize("L", [1, 2, 33, 34, 96, 128, 129, 300, 383, 384, 385, 512])
def test_tiny_decode_lengths(L):
    d = decode_inputs(TINY, Lcap=512)
    cache = oracle_cache_bf16(d.k_raw, TINY.theta)
    out, lse, o_ref, lse_ref = decode_both(TINY, L, d.q, cache, d.v)
    assert_o(f64(out), o_ref, f"L={L}")
    assert_lse(f64(lse), lse_ref, f"L={L}")


@pytest.mark.parametrize("Hq,Hkv,D,wp,w0,L", [
    (8, 2, 128, 64, 0, 1000), (3, 3, 64, 100, 7, 777), (8, 1, 128, 512, 600, 2048),
    (32, 8, 128, 1024, 100, 5000), (4, 2, 64, 1, 3, 200), (16, 16, 128, 300, 50, 3000),
    (64, 8, 128, 2048, 1000, 9000), (24, 12, 64, 500, 20, 4100), (8, 8, 128, 128, 10, 17)])
def test_decode_shapes(Hq, Hkv, D, wp, w0, L):
    w = Workload("dec", 2, Hq, Hkv, D, L, wp, w0, 1e6, 30 + L, False, kind="decode")
    d = decode_inputs(w, Lcap=L + 5)
    cache = oracle_cache_bf16(d.k_raw, w.theta)
    out, lse, o_ref, lse_ref = decode_both(w, L, d.q, cache, d.v)
    assert_o(f64(out), o_ref, "decode shapes")
    assert_lse(f64(lse), lse_ref, "decode shapes")


def test_decode_bf16_output():
    d = decode_inputs(TINY, Lcap=512)
    cache = oracle_cache_bf16(d.k_raw, TINY.theta)
    out, lse, o_ref, lse_ref = decode_both(TINY, 400, d.q, cache, d.v, out_dtype=torch.bfloat16)
    assert_o_bf16(f64(out), o_ref, "decode bf16")


def test_group_transition_of_appendix_e():
    # The page's boundary: w_pretrained = 32,768, L = 98,304 -> 98,305 moves G
    # from 3 to 4.  One cache, two consecutive steps.
    w = Workload("transition", 1, 8, 2, 128, 98305, 32768, 2048, 1e6, 41, False, kind="decode")
    d = decode_inputs(w)
    cache = oracle_cache_bf16(d.k_raw, w.theta)
    for L in (98304, 98305):
        out, lse, o_ref, lse_ref = decode_both(w, L, d.q, cache, d.v)
        assert_o(f64(out), o_ref, f"L={L}")
        assert_lse(f64(lse), lse_ref, f"L={L}")


@pytest.mark.parametrize("name", ["decode_8b_32k", "decode_8b_64k", "decode_8b_128k"])
def test_qwen3_8b_decode(name):
    w = WORKLOADS[name]
    d = decode_inputs(w)
    cache = oracle_cache_bf16(d.k_raw, w.theta)
    out, lse, o_ref, lse_ref = decode_both(w, w.L, d.q, cache, d.v)
    assert_o(f64(out), o_ref, name)
    assert_lse(f64(lse), lse_ref, name)


@pytest.mark.parametrize("pos0,n", [(0, 512), (100, 37), (4095, 1)])
def test_rope_cache_kernel(pos0, n):
    w = Workload("rc", 2, 4, 2, 128, 5000, 32768, 4096, 1e6, 51, True)
    k = prefill_inputs(w.with_(L=n)).k
    cap = pos0 + n + 3
    cache = torch.zeros((w.B, cap, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    jl.jetlong_rope_cache(k.cuda(), cache, pos0, w.theta)
    ref = oracle.rope_cache(f64(k), pos0, w.theta)
    got = f64(cache[:, pos0:pos0 + n])
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)
    assert torch.count_nonzero(cache[:, :pos0]) == 0 and torch.count_nonzero(cache[:, pos0 + n:]) == 0


def test_decode_after_prefill_matches_last_row():
    # Prefill writes the true-position cache; a decode of the last token on it
    # must agree with the prefill's last row (both against the oracle).
    w = WORKLOADS["tiny"].with_(L=700, w_pretrained=128, w0=40)
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    cache = torch.empty((w.B, w.L, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    out_p, lse_p = jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta,
                                      out_dtype=torch.float32, k_cache_out=cache)
    out_d, lse_d = jl.jetlong_decode(q[:, -1].contiguous(), cache, v, w.L, w.w_pretrained, w.w0,
                                     w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_rows(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0,
                                         w.theta, [w.L - 1])
    assert_o(f64(out_d), o_ref[:, 0], "decode after prefill")
    assert_lse(f64(lse_d), lse_ref[:, :, 0], "decode after prefill")
    assert_o(f64(out_d), f64(out_p[:, -1]), "decode vs prefill row")


def test_decode_calls_replay_from_a_cuda_graph():
    # After a first (eager) call has set the kernels' shared-memory limits, a
    # call makes no CUDA API call besides its launches, so a decode loop can
    # be captured once and replayed; the replay equals the eager calls bit
    # for bit.
    w = WORKLOADS["decode_8b_32k"].with_(w_pretrained=8192)  # G = 4 at 32K
    d = decode_inputs(w)
    cache = oracle_cache_bf16(d.k_raw, w.theta).cuda()
    v, q = d.v.cuda(), d.q.cuda()
    Ls = [w.L - 3, w.L - 2, w.L - 1, w.L]
    ws = torch.empty(jl.jetlong_decode_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D),
                     dtype=torch.uint8, device="cuda")
    outs = [torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda") for _ in Ls]
    lses = [torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda") for _ in Ls]

    def loop(stream=None):
        for L, o, l in zip(Ls, outs, lses):
            jl.jetlong_decode(q, cache, v, L, w.w_pretrained, w.w0, w.theta, out=o, lse=l,
                              workspace=ws, stream=stream)

    loop()
    eager = [(o.clone(), l.clone()) for o, l in zip(outs, lses)]
    for o, l in zip(outs, lses):
        o.fill_(float("nan"))
        l.fill_(float("nan"))
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        loop(cap)
    g.replay()
    torch.cuda.synchronize()
    assert jl.jetlong_device_status() == jl.JL_OK
    for (eo, el), o, l in zip(eager, outs, lses):
        assert torch.equal(eo, o) and torch.equal(el, l)


@pytest.mark.parametrize("D,grp,wp,w0,L,jstar", [
    (64, 2, 64, 64, 40, 10),    # G = 1, the jump in the second 8-token block of a stage
    (64, 4, 16, 35, 40, 26),    # G = 3, the key that jumps is local
    (64, 1, 8, 3, 48, 42),      # G = 6, the key that jumps is remote
    (128, 4, 16, 35, 40, 26),   # 8-token stages: one block per stage
])
def test_running_max_jumps_inside_a_stage(D, grp, wp, w0, L, jstar):
    # One cached key is aligned with the first query head's rotated query, so
    # its score stands about 16 nats above the rest and the running max jumps
    # by far more than the lazy-rescale threshold in the middle of a stage.
    # Every block of the stage must then be weighed against the new max.
    w = Workload("jump", 1, grp, 1, D, L, wp, w0, 1e4, 81 + jstar, False, kind="decode")
    d = decode_inputs(w, Lcap=L)
    cache = oracle.rope_cache(f64(d.k_raw), 0, w.theta)
    p = L - 1
    G = oracle.group_size(L, wp)
    target = p if p - jstar <= w0 else p // G - jstar // G + jstar
    cache[0, jstar, 0] = 2.0 * oracle.rope(f64(d.q)[0, 0], np.int64(target), w.theta)
    cache = torch.from_numpy(cache).to(torch.bfloat16)
    out, lse, o_ref, lse_ref = decode_both(w, L, d.q, cache, d.v)
    assert lse_ref[0, 0] > 10.0  # the planted key dominates head 0
    assert_o(f64(out), o_ref, f"jump at {jstar}")
    assert_lse(f64(lse), lse_ref, f"jump at {jstar}")
