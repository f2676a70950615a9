"""Generation across group-size transitions and long contexts (GPU vs the
fp64 oracle).

* A multi-step generation loop: each step appends the new token's key (RoPE at
  its true position, jetlong_rope_cache) and value to the cache, then decodes
  at the new length.  The loop crosses the boundary the Jet-Long paper names
  in its Appendix E (w_pretrained = 32,768: L = 98,304 -> 98,305 moves G from
  3 to 4), so the correction rotations of every remote key change between two
  consecutive steps while the cache itself is never rewritten (§3.2).  The
  oracle builds its own cache from the raw keys; nothing it reads comes from
  the GPU.
* Decode and prefill at 256K, 512K and 1M tokens (G = 8, 16, 32): the
  schedule far past the 4x extension of the headline layer.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import (Workload, decode_inputs, generation_inputs,
                                               prefill_inputs, sample_rows)

pytestmark = pytest.mark.gpu


def test_generation_loop_across_group_transition():
    w = Workload("gen", 1, 8, 2, 128, 0, 32768, 2048, 1e6, 71, False, kind="decode")
    L0, n = 98300, 8
    x = generation_inputs(w, L0, n)
    cap = L0 + n
    # the oracle's cache: true-position RoPE in float64, stored as BF16
    ref_cache = torch.from_numpy(oracle.rope_cache(f64(x.k_raw), 0, w.theta)).to(torch.bfloat16)
    ref_cache64, v64 = f64(ref_cache), f64(x.v)

    kc = torch.zeros((w.B, cap, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k_raw, v = x.k_raw.cuda(), x.v.cuda()
    jl.jetlong_rope_cache(k_raw[:, :L0].contiguous(), kc, 0, w.theta)
    vc[:, :L0] = v[:, :L0]
    groups = []
    for t in range(n):
        L = L0 + t + 1
        jl.jetlong_rope_cache(k_raw[:, L - 1:L].contiguous(), kc, L - 1, w.theta)  # append
        vc[:, L - 1] = v[:, L - 1]
        out, lse = jl.jetlong_decode(x.q[t].cuda(), kc, vc, L, w.w_pretrained, w.w0, w.theta,
                                     out_dtype=torch.float32)
        assert jl.jetlong_device_status() == jl.JL_OK
        o_ref, lse_ref = oracle.decode(f64(x.q[t]), ref_cache64, v64, L, w.w_pretrained, w.w0,
                                       w.theta)
        assert_o(f64(out), o_ref, f"step L={L}")
        assert_lse(f64(lse), lse_ref, f"step L={L}")
        groups.append(jl.jetlong_group_size(L, w.w_pretrained))
    assert groups == [3, 3, 3, 3, 4, 4, 4, 4]  # L = 98301..98308
    # The appended rows are the true-position RoPE of each key.  Both sides
    # round a rotation to BF16 (the GPU's fp32 one, the oracle's fp64 one), so
    # a value near a rounding boundary may land one BF16 ulp (2^-7 relative)
    # apart; with rotations that agree to ~1e-7 that happens for ~1e-4 of
    # the entries at most.
    got, ref = f64(kc), ref_cache64
    assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6)
    assert np.mean(got != ref) < 1e-3


@pytest.mark.parametrize("L", [262144, 524288, 1048576])
def test_long_context_decode(L):
    w = Workload("long_dec", 1, 8, 2, 128, L, 32768, 4096, 1e6, 81, False, kind="decode")
    d = decode_inputs(w)
    cache = torch.from_numpy(oracle.rope_cache(f64(d.k_raw), 0, w.theta)).to(torch.bfloat16)
    out, lse = jl.jetlong_decode(d.q.cuda(), cache.cuda(), d.v.cuda(), L, w.w_pretrained, w.w0,
                                 w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.decode(f64(d.q), f64(cache), f64(d.v), L, w.w_pretrained, w.w0,
                                   w.theta)
    assert jl.jetlong_group_size(L, w.w_pretrained) == L // 32768
    assert_o(f64(out), o_ref, f"L={L}")
    assert_lse(f64(lse), lse_ref, f"L={L}")


@pytest.mark.parametrize("L", [262144, 524288, 1048576])
def test_long_context_prefill_sampled_rows(L):
    # G = 8, 16, 32: remote positions f(i) = i // G stay below w_pretrained
    w = Workload("long_pf", 1, 8, 2, 128, L, 32768, 4096, 1e6, 91, True)
    x = prefill_inputs(w, device="cuda")
    out, lse = jl.jetlong_prefill(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta,
                                  out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    rows = sample_rows(w.L, w.w0, w.w_pretrained, 10, w.seed)
    ridx = torch.tensor(rows, device="cuda")
    o_ref, lse_ref = oracle.prefill_rows(f64(x.q.index_select(1, ridx)), f64(x.k), f64(x.v),
                                         w.w_pretrained, w.w0, w.theta, rows, q_holds_rows=True)
    assert jl.jetlong_group_size(L, w.w_pretrained) == L // 32768
    assert_o(f64(out.index_select(1, ridx)), o_ref, f"L={L}")
    assert_lse(f64(lse.index_select(2, ridx)), lse_ref, f"L={L}")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
