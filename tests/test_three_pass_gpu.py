"""GPU parity of jetlong_prefill_three_pass, the unfused inclusion-exclusion
form (Jet-Long paper, §3.3): passes A (remote positions, all causal pairs),
B (true positions, band 0 <= i - j <= w0) and C (remote positions, band),
merged as (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C).

It must agree with the fp64 oracle's direct rule (same tolerances as the
fused kernel) and with the fused GPU kernel on the same inputs.
"""
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, assert_o_bf16, f64, lse_err, o_err
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, Workload, prefill_inputs, sample_rows

pytestmark = pytest.mark.gpu


def both(w: Workload, out_dtype=torch.float32):
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    o3, l3 = jl.jetlong_prefill_three_pass(q, k, v, w.w_pretrained, w.w0, w.theta,
                                           out_dtype=out_dtype)
    of, lf = jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, out_dtype=out_dtype)
    assert jl.jetlong_device_status() == jl.JL_OK
    return x, o3, l3, of, lf


@pytest.mark.parametrize("name", ["tiny", "tiny_native"])
def test_tiny_every_row(name):
    w = WORKLOADS[name]
    x, o3, l3, of, lf = both(w)
    o_ref, lse_ref = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert_o(f64(o3), o_ref, name)
    assert_lse(f64(l3), lse_ref, name)
    # the two GPU paths agree far more tightly than either does with the bar
    assert o_err(f64(o3), f64(of)) <= 2e-3
    assert lse_err(f64(l3), f64(lf)) <= 1e-4


@pytest.mark.parametrize("L,wp,w0,Hq,Hkv,D", [
    (1, 128, 32, 2, 1, 64),       # one token: every pass sees only the diagonal
    (129, 128, 0, 2, 1, 64),      # w0 = 0: the band is the diagonal
    (300, 64, 17, 4, 2, 64),      # ragged tail, GQA 2
    (640, 128, 0, 6, 2, 128),     # GQA 3, D = 128
    (777, 200, 800, 2, 1, 64),    # w0 >= L: B covers everything, A and C cancel
    (1000, 2000, 100, 4, 1, 128), # G = 1: B and C coincide and cancel
    (1300, 300, 250, 4, 4, 128),  # G = 5
])
def test_edge_shapes_every_row(L, wp, w0, Hq, Hkv, D):
    w = Workload("edge3", 1, Hq, Hkv, D, L, wp, w0, 1e4, 61 + L, True)
    x, o3, l3, of, lf = both(w)
    o_ref, lse_ref = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert_o(f64(o3), o_ref, f"three-pass L={L}")
    assert_lse(f64(l3), lse_ref, f"three-pass L={L}")
    assert o_err(f64(o3), f64(of)) <= 2e-3


def test_bf16_output():
    w = WORKLOADS["tiny"]
    x, o3, l3, _, _ = both(w, out_dtype=torch.bfloat16)
    o_ref, _ = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert o3.dtype == torch.bfloat16
    assert_o_bf16(f64(o3), o_ref, "three-pass bf16")


@pytest.mark.parametrize("name", ["qwen3_8b_64k"])
def test_qwen3_layer_sampled_rows(name):
    w = WORKLOADS[name]
    x = prefill_inputs(w, device="cuda")
    o3, l3 = jl.jetlong_prefill_three_pass(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta,
                                           out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    rows = sample_rows(w.L, w.w0, w.w_pretrained, 8, w.seed)
    ridx = torch.tensor(rows, device="cuda")
    o_ref, lse_ref = oracle.prefill_rows(f64(x.q.index_select(1, ridx)), f64(x.k), f64(x.v),
                                         w.w_pretrained, w.w0, w.theta, rows, q_holds_rows=True)
    assert_o(f64(o3.index_select(1, ridx)), o_ref, name)
    assert_lse(f64(l3.index_select(2, ridx)), lse_ref, name)
    assert torch.isfinite(o3).all() and torch.isfinite(l3).all()
