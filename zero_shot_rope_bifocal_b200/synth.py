"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module draws random numbers and shapes them; it holds none of the
attention arithmetic (no RoPE, no schedule, no softmax), so that the CUDA
library and the CPU oracle can both be fed from it without sharing any of the
method's code.

Workloads stand in for the Qwen3 attention layers the Jet-Long paper evaluates
(§4.1 "Models": Qwen3-1.7B/4B/8B-Base with a 32K native window): single
attention layers with the Qwen3 head counts, BF16 inputs, pre-RoPE Q and K.
Q, K, V are i.i.d. N(0, 1) in fp32 and then rounded to BF16 (round to nearest
even, as ``Tensor.to(torch.bfloat16)`` does).  For the Qwen3-shaped layers the
pre-RoPE keys get a per-(KV head, channel) scale drawn from LogNormal(0, 0.5)
to mimic the outlier RoPE channels of real checkpoints.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    L: int
    w_pretrained: int
    w0: int
    theta: float
    seed: int
    k_channel_scale: bool
    kind: str = "prefill"          # "prefill" or "decode"
    note: str = ""

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The named single-layer workloads (sizes as listed in the benchmark plan).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 1, 64, 512, 128, 32, 1e4, 0, False,
                     note="GQA 2:1, G=4; oracle runs in full"),
    "tiny_native": Workload("tiny_native", 1, 2, 1, 64, 96, 128, 32, 1e4, 0, False,
                            note="L <= w_pretrained: must reduce to plain causal RoPE attention"),
    "qwen3_1p7b_16k": Workload("qwen3_1p7b_16k", 1, 16, 8, 128, 16384, 32768, 4096, 1e6, 1, True,
                               note="identity schedule (G=1)"),
    "qwen3_1p7b_64k": Workload("qwen3_1p7b_64k", 1, 16, 8, 128, 65536, 32768, 4096, 1e6, 2, True),
    "qwen3_8b_64k": Workload("qwen3_8b_64k", 1, 32, 8, 128, 65536, 32768, 4096, 1e6, 3, True,
                             note="w0 sweep {2048, 4096, 8192}"),
    "qwen3_8b_128k": Workload("qwen3_8b_128k", 1, 32, 8, 128, 131072, 32768, 4096, 1e6, 4, True,
                              note="headline prefill point (G=4)"),
    "decode_8b_32k": Workload("decode_8b_32k", 1, 32, 8, 128, 32768, 32768, 4096, 1e6, 5, False,
                              kind="decode"),
    "decode_8b_64k": Workload("decode_8b_64k", 1, 32, 8, 128, 65536, 32768, 4096, 1e6, 6, False,
                              kind="decode"),
    "decode_8b_128k": Workload("decode_8b_128k", 1, 32, 8, 128, 131072, 32768, 4096, 1e6, 7, False,
                               kind="decode"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


@dataclass
class PrefillInputs:
    q: torch.Tensor        # [B, L, Hq, D] bf16, pre-RoPE
    k: torch.Tensor        # [B, L, Hkv, D] bf16, pre-RoPE
    v: torch.Tensor        # [B, L, Hkv, D] bf16
    k_scale: torch.Tensor | None = field(default=None)


def prefill_inputs(w: Workload, device="cpu") -> PrefillInputs:
    """Draw (q, k, v) for a prefill workload on ``device`` from seed ``w.seed``.

    Draw order: per-channel K scale (if any), then Q, K, V.  The same seed on
    the same device type gives the same tensors.
    """
    g = _gen(w.seed, device)
    scale = None
    if w.k_channel_scale:
        scale = torch.exp(0.5 * torch.randn((w.Hkv, w.D), generator=g, device=device,
                                            dtype=torch.float32))
    q = torch.randn((w.B, w.L, w.Hq, w.D), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((w.B, w.L, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    if scale is not None:
        k.mul_(scale)
    v = torch.randn((w.B, w.L, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    return PrefillInputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), scale)


@dataclass
class DecodeInputs:
    q: torch.Tensor        # [B, Hq, D] bf16, pre-RoPE query of the new token
    k_raw: torch.Tensor    # [B, Lcap, Hkv, D] bf16, pre-RoPE keys (to be rotated into the cache)
    v: torch.Tensor        # [B, Lcap, Hkv, D] bf16


def decode_inputs(w: Workload, Lcap: int | None = None, device="cpu") -> DecodeInputs:
    """Draw the decode query and the raw K / V history for a cache of ``Lcap`` slots."""
    Lcap = w.L if Lcap is None else int(Lcap)
    g = _gen(w.seed, device)
    q = torch.randn((w.B, w.Hq, w.D), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((w.B, Lcap, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((w.B, Lcap, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    return DecodeInputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


@dataclass
class GenerationInputs:
    q: torch.Tensor      # [n_steps, B, Hq, D] bf16, the query of each step (pre-RoPE)
    k_raw: torch.Tensor  # [B, L0 + n_steps, Hkv, D] bf16, pre-RoPE keys of every slot
    v: torch.Tensor      # [B, L0 + n_steps, Hkv, D] bf16


def generation_inputs(w: Workload, L0: int, n_steps: int, device="cpu") -> GenerationInputs:
    """A cache prefix of ``L0`` tokens plus ``n_steps`` generated tokens: their
    raw keys and values, and one query per step.  Draw order: K, V, queries."""
    g = _gen(w.seed, device)
    cap = L0 + n_steps
    k = torch.randn((w.B, cap, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((w.B, cap, w.Hkv, w.D), generator=g, device=device, dtype=torch.float32)
    q = torch.randn((n_steps, w.B, w.Hq, w.D), generator=g, device=device, dtype=torch.float32)
    return GenerationInputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def sample_rows(L: int, w0: int, w_pretrained: int, n: int, seed: int) -> list[int]:
    """Query rows to check on a large workload: the edges of the local window,
    the native-window and group boundaries, the last rows, then seeded random
    rows until ``n`` rows are chosen."""
    special = [0, 1, w0 - 1, w0, w0 + 1, w0 + 2, w_pretrained - 1, w_pretrained,
               w_pretrained + 1, L - 2, L - 1]
    special += [m * w_pretrained + d for m in range(1, 8) for d in (-1, 0, 1)]
    rows = sorted({r for r in special if 0 <= r < L})[:n]
    g = torch.Generator().manual_seed(int(seed) + 1000)
    for r in torch.randint(0, L, (4 * n,), generator=g).tolist():
        if len(rows) >= n:
            break
        if r not in rows:
            rows.append(r)
    return sorted(rows)
