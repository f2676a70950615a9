"""Shared helpers for the GPU parity tests (comparison rules and conversions).

Tolerances: max-abs error <= 1e-2 on O (unit-variance V) and relative error
<= 1e-3 on the log-sum-exp for BF16 inputs.  The LSE error is measured as
|lse_gpu - lse_ref| / max(1, |lse_ref|) so that rows with lse near 0 (row 0 of
a prompt) do not divide by ~0.  A BF16 output adds its own rounding
(half an ulp: 2^-9 relative), so BF16-out checks allow 1e-2 + 2^-8 |ref|.
"""
import numpy as np
import torch
from hypothesis import strategies as st

from zero_shot_rope_bifocal_b200.synth import Workload

O_ATOL = 1e-2
LSE_RTOL = 1e-3
BF16_OUT_RTOL = 2.0 ** -8


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def o_err(gpu, ref) -> float:
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) if np.size(ref) else 0.0


def lse_err(gpu, ref) -> float:
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - ref) / np.maximum(1.0, np.abs(ref))))


def assert_o(gpu, ref, what=""):
    e = o_err(gpu, ref)
    assert e <= O_ATOL, f"{what} O max-abs error {e:.3e} > {O_ATOL}"
    return e


def assert_o_bf16(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    excess = np.abs(gpu - ref) - (O_ATOL + BF16_OUT_RTOL * np.abs(ref))
    assert np.max(excess) <= 0, f"{what} BF16 O error exceeds 1e-2 + 2^-8|ref| by {np.max(excess):.3e}"


def assert_lse(gpu, ref, what=""):
    e = lse_err(gpu, ref)
    assert e <= LSE_RTOL, f"{what} LSE relative error {e:.3e} > {LSE_RTOL}"
    return e


@st.composite
def workloads(draw, grps, max_L):
    """Random small workloads for the randomised parity tests: ragged L,
    GQA ratios from ``grps``, both head dimensions, w0 from 0 to beyond L,
    G from 1 up (w_pretrained from 1 to beyond L)."""
    L = draw(st.integers(1, max_L))
    Hkv = draw(st.sampled_from([1, 2, 3]))
    grp = draw(st.sampled_from(grps))
    D = draw(st.sampled_from([64, 128]))
    wp = draw(st.integers(1, L + 64))
    w0 = draw(st.integers(0, L + 8))
    B = draw(st.integers(1, 2))
    theta = draw(st.sampled_from([1e4, 1e6]))
    seed = draw(st.integers(0, 10**6))
    return Workload("rand", B, Hkv * grp, Hkv, D, L, wp, w0, theta, seed, seed % 2 == 0)
