"""The failure path of the bounded in-kernel waits, exercised on the GPU
without a fault: a wait on an mbarrier that nothing completes gives up after
its limit, the kernel records a timeout, the host reads it through
jetlong_device_status(), and the context keeps working."""
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import WORKLOADS, prefill_inputs

pytestmark = pytest.mark.gpu


def _tiny_prefill():
    w = WORKLOADS["tiny"]
    x = prefill_inputs(w)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    out = torch.full((w.B, w.L, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((w.B, w.Hq, w.L), float("nan"), dtype=torch.float32, device="cuda")
    jl.jetlong_prefill(q, k, v, w.w_pretrained, w.w0, w.theta, out=out, lse=lse)
    return w, x, out, lse


def test_expired_wait_is_reported_and_the_context_survives():
    assert jl.jetlong_device_status() == jl.JL_OK  # start clean
    jl.jetlong_check_device_timeout(50)
    assert jl.jetlong_device_status() == jl.JL_ERR_DEVICE_TIMEOUT
    assert jl.jetlong_device_status() == jl.JL_OK  # reading clears the report
    w, x, out, lse = _tiny_prefill()
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill(f64(x.q), f64(x.k), f64(x.v), w.w_pretrained, w.w0, w.theta)
    assert_o(f64(out), o_ref, "after timeout")
    assert_lse(f64(lse), lse_ref, "after timeout")


def test_prefill_after_an_unread_timeout_ends_without_computing():
    # A prefill launched while a failure is still recorded honours it: it
    # ends at once, leaves its outputs untouched, and the report stays.
    jl.jetlong_check_device_timeout(20)
    _, _, out, lse = _tiny_prefill()
    assert jl.jetlong_device_status() == jl.JL_ERR_DEVICE_TIMEOUT
    assert torch.isnan(out).all() and torch.isnan(lse).all()
    _, _, out, lse = _tiny_prefill()
    assert jl.jetlong_device_status() == jl.JL_OK
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
