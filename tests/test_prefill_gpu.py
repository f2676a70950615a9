"""GPU parity of jetlong_prefill (through the C ABI) against the fp64 oracle.

Small cases run the oracle on every row; the Qwen3-shaped layers (16K, 64K,
128K tokens) run in the same launch configuration the benchmark uses and are
checked on sampled rows (window edges, native-window and group boundaries,
last row, seeded random rows).
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, assert_o_bf16, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, Workload, prefill_inputs, sample_rows

pytestmark = pytest.mark.gpu


def run(w: Workload, out_dtype=torch.float32, x=None, **kw):
    x = x if x is not None else prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    out, lse = jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, out_dtype=out_dtype, **kw)
    assert jl.jetlong_device_status() == jl.JL_OK
    return x, out, lse


def full_ref(w: Workload, x):
    return oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)


@pytest.mark.parametrize("name", ["tiny", "tiny_native"])
def test_tiny_every_row(name):
    w = WORKLOADS[name]
    x, out, lse = run(w)
    o_ref, lse_ref = full_ref(w, x)
    assert_o(f64(out), o_ref, name)
    assert_lse(f64(lse), lse_ref, name)


def test_tiny_bf16_output():
    w = WORKLOADS["tiny"]
    x, out, lse = run(w, out_dtype=torch.bfloat16)
    o_ref, lse_ref = full_ref(w, x)
    assert out.dtype == torch.bfloat16
    assert_o_bf16(f64(out), o_ref, "tiny bf16")
    assert_lse(f64(lse), lse_ref, "tiny bf16")


EDGE = [
    # (L, w_pretrained, w0, Hq, Hkv, D): ragged tails, both head dims, GQA
    # ratios 1..3, G = 1..5, w0 = 0 (only self-attention local), w0 >= L.
    (1, 128, 32, 2, 1, 64),
    (2, 1, 0, 2, 1, 64),
    (127, 128, 5, 2, 2, 128),
    (129, 128, 0, 2, 1, 64),
    (300, 64, 17, 4, 2, 64),
    (640, 128, 0, 6, 2, 128),
    (1000, 256, 100, 3, 1, 128),
    (777, 200, 800, 2, 1, 64),
    (1300, 300, 250, 4, 4, 128),
    (257, 64, 128, 2, 1, 128),
]


@pytest.mark.parametrize("L,wp,w0,Hq,Hkv,D", EDGE)
def test_edge_shapes_every_row(L, wp, w0, Hq, Hkv, D):
    w = Workload("edge", 1, Hq, Hkv, D, L, wp, w0, 1e4, 11 + L, True)
    x, out, lse = run(w)
    o_ref, lse_ref = full_ref(w, x)
    assert_o(f64(out), o_ref, f"edge L={L}")
    assert_lse(f64(lse), lse_ref, f"edge L={L}")


def test_batch_two_and_theta_1e6():
    w = Workload("b2", 2, 4, 2, 128, 700, 256, 64, 1e6, 21, True)
    x, out, lse = run(w)
    o_ref, lse_ref = full_ref(w, x)
    assert_o(f64(out), o_ref, "B=2")
    assert_lse(f64(lse), lse_ref, "B=2")


def test_rerun_is_bitwise_identical():
    w = WORKLOADS["tiny"].with_(L=1000, w_pretrained=200)
    x, out1, lse1 = run(w)
    _, out2, lse2 = run(w, x=x)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_k_cache_out_is_true_position_rope():
    w = WORKLOADS["tiny"]
    x = prefill_inputs(w)
    cap = w.L + 64
    cache = torch.full((w.B, cap, w.Hkv, w.D), 7.0, dtype=torch.bfloat16, device="cuda")
    run(w, x=x, k_cache_out=cache)
    ref = oracle.rope_cache(f64(x.k), 0, w.theta)
    got = f64(cache[:, : w.L])
    # one BF16 rounding of the exact rotated value (half an ulp) plus fp32 math
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)
    assert torch.all(cache[:, w.L:] == 7.0)


LARGE = [
    ("qwen3_1p7b_16k", None),
    ("qwen3_1p7b_64k", None),
    ("qwen3_8b_64k", 2048),
    ("qwen3_8b_64k", 4096),
    ("qwen3_8b_64k", 8192),
    ("qwen3_8b_128k", None),
]


@pytest.mark.parametrize("name,w0", LARGE)
def test_qwen3_layers_sampled_rows(name, w0):
    w = WORKLOADS[name] if w0 is None else WORKLOADS[name].with_(w0=w0)
    x = prefill_inputs(w, device="cuda")
    out, lse = jl.jetlong_prefill(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta,
                                  out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    rows = sample_rows(w.L, w.w0, w.w_pretrained, 12, w.seed)
    ridx = torch.tensor(rows, device="cuda")
    q_rows = f64(x.q.index_select(1, ridx))
    o_ref, lse_ref = oracle.prefill_rows(q_rows, f64(x.k), f64(x.v), w.w_pretrained, w.w0,
                                         w.theta, rows, q_holds_rows=True)
    assert_o(f64(out.index_select(1, ridx)), o_ref, name)
    assert_lse(f64(lse.index_select(2, ridx)), lse_ref, name)
    # properties that hold on every row: finite, and O inside the hull of V
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    vmax = x.v.float().abs().amax().item()
    # (BF16 probabilities make the weights sum to 1 within 2^-8)
    assert out.abs().amax().item() <= vmax * (1 + 2.0 ** -7)


def test_bad_arguments_launch_nothing():
    w = WORKLOADS["tiny"]
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    with pytest.raises(jl.JetLongError) as ei:
        jl.jetlong_prefill(q, k, v, w.w_pretrained, -1, w.theta)
    assert ei.value.status == jl.JL_ERR_SHAPE
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(jl.JetLongError) as ei:
        jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, workspace=small)
    assert ei.value.status == jl.JL_ERR_WORKSPACE
    assert jl.jetlong_device_status() == jl.JL_OK


def test_staged_calls_equal_the_fused_call():
    w = WORKLOADS["tiny"].with_(L=900, w_pretrained=256, w0=50)
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    out1, lse1 = jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, out_dtype=torch.float32)
    ws = torch.empty(jl.jetlong_prefill_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D),
                     dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(out1)
    lse2 = torch.empty_like(lse1)
    jl.jetlong_prefill_rotate(k, v, w.w_pretrained, w.theta, ws)
    jl.jetlong_prefill_attend(q, out2, lse2, w.Hkv, w.w_pretrained, w.w0, w.theta, ws)
    assert jl.jetlong_device_status() == jl.JL_OK
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_values_beyond_fp16_range_are_reported():
    w = WORKLOADS["tiny"]
    x = prefill_inputs(w)
    q = x.q.clone()
    q[0, 5, 1, 3] = 1.0e5  # beyond the FP16 operand range
    jl.jetlong_prefill(q.cuda(), x.k.cuda(), x.v.cuda(), w.w_pretrained, w.w0, w.theta)
    assert jl.jetlong_device_status() == jl.JL_ERR_RANGE
    # the report is cleared once read, and a clean call reports OK again
    run(w, x=x)
    assert jl.jetlong_device_status() == jl.JL_OK
