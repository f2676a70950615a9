"""The seeded input generators shared by the tests, the benchmark and the
oracle: determinism, shapes and formats, the K channel-scale recipe, and the
row sampler used for large-workload parity."""
import torch

from zero_shot_rope_bifocal_b200.synth import (WORKLOADS, decode_inputs, generation_inputs,
                                               prefill_inputs, sample_rows)


def test_same_seed_same_tensors_and_formats():
    w = WORKLOADS["tiny"]
    a, b = prefill_inputs(w), prefill_inputs(w)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v)):
        assert torch.equal(x, y) and x.dtype == torch.bfloat16 and x.is_contiguous()
    assert a.q.shape == (w.B, w.L, w.Hq, w.D) and a.k.shape == (w.B, w.L, w.Hkv, w.D)
    c = prefill_inputs(w.with_(seed=w.seed + 1))
    assert not torch.equal(a.q, c.q)


def test_values_are_unit_normal_rounded_to_bf16():
    w = WORKLOADS["tiny"].with_(L=4096)
    x = prefill_inputs(w)
    q = x.q.float()
    assert abs(q.mean().item()) < 0.02 and abs(q.std().item() - 1.0) < 0.02
    # BF16 values: converting to fp32 and back is exact
    assert torch.equal(x.q.float().to(torch.bfloat16), x.q)


def test_key_channel_scale_is_lognormal_and_drawn_first():
    w = WORKLOADS["qwen3_1p7b_16k"].with_(L=64)
    x = prefill_inputs(w)
    assert x.k_scale is not None and x.k_scale.shape == (w.Hkv, w.D)
    logs = x.k_scale.log()
    assert abs(logs.mean().item()) < 0.15 and abs(logs.std().item() - 0.5) < 0.1
    # the scale is the first draw: the same seed reproduces it alone
    g = torch.Generator().manual_seed(w.seed)
    first = torch.exp(0.5 * torch.randn((w.Hkv, w.D), generator=g))
    assert torch.equal(first, x.k_scale)
    # and it multiplies K per (KV head, channel)
    assert prefill_inputs(w.with_(k_channel_scale=False)).k_scale is None


def test_decode_and_generation_shapes():
    w = WORKLOADS["tiny"].with_(kind="decode")
    d = decode_inputs(w, Lcap=600)
    assert d.q.shape == (w.B, w.Hq, w.D) and d.k_raw.shape == (w.B, 600, w.Hkv, w.D)
    g = generation_inputs(w, 100, 7)
    assert g.q.shape == (7, w.B, w.Hq, w.D) and g.k_raw.shape == (w.B, 107, w.Hkv, w.D)
    assert g.v.shape == g.k_raw.shape


def test_sampled_rows_cover_the_window_and_group_edges():
    L, w0, wp = 131072, 4096, 32768
    rows = sample_rows(L, w0, wp, 24, 4)
    assert rows == sorted(set(rows)) and len(rows) == 24
    assert all(0 <= r < L for r in rows)
    for r in (0, 1, w0 - 1, w0, w0 + 1, w0 + 2, wp - 1, wp, wp + 1):
        assert r in rows
    assert sample_rows(L, w0, wp, 24, 4) == rows  # seeded
    small = sample_rows(10, 4, 8, 50, 0)
    assert small == list(range(10))  # never more rows than the prompt has
