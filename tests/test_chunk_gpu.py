"""GPU parity of jetlong_prefill_chunk (through the C ABI) against the fp64
oracle's prefill_chunk: queries of a chunk at positions P0 .. P0+n-1 against
a true-position cache that already holds the chunk's keys, one G for the
call from P0 + n (Jet-Long paper, §3.1, §3.2).

Both sides read the same BF16 cache, built by the oracle (true-position RoPE
in fp64, rounded to BF16), as in the decode tests.
"""
import pytest
import torch

import oracle
from parity_util import assert_lse, assert_o, f64
from zero_shot_rope_bifocal_b200 import jetlong as jl
from zero_shot_rope_bifocal_b200.synth import Workload, generation_inputs

pytestmark = pytest.mark.gpu


def run_chunk(w: Workload, L0: int, n: int, Lcap_extra: int = 3):
    x = generation_inputs(w, L0, n + Lcap_extra)
    cap = L0 + n + Lcap_extra
    cache = torch.from_numpy(oracle.rope_cache(f64(x.k_raw), 0, w.theta)).to(torch.bfloat16)
    q = torch.randn((w.B, n, w.Hq, w.D), generator=torch.Generator().manual_seed(w.seed + 5))
    q = q.to(torch.bfloat16)
    out, lse = jl.jetlong_prefill_chunk(q.cuda(), cache.cuda(), x.v.cuda(), L0, w.w_pretrained,
                                        w.w0, w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    o_ref, lse_ref = oracle.prefill_chunk(f64(q), f64(cache), f64(x.v), L0, w.w_pretrained, w.w0,
                                          w.theta)
    assert out.shape == (w.B, n, w.Hq, w.D) and lse.shape == (w.B, w.Hq, n)
    assert cap >= L0 + n
    return out, lse, o_ref, lse_ref


@pytest.mark.parametrize("P0,n", [(0, 1), (0, 512), (300, 212), (511, 1), (100, 17), (257, 64)])
def test_tiny_chunks(P0, n):
    w = Workload("chunk_tiny", 1, 2, 1, 64, 0, 128, 32, 1e4, 11, False, kind="decode")
    out, lse, o_ref, lse_ref = run_chunk(w, P0, n)
    assert_o(f64(out), o_ref, f"P0={P0} n={n}")
    assert_lse(f64(lse), lse_ref, f"P0={P0} n={n}")


@pytest.mark.parametrize("B,Hq,Hkv,D,wp,w0,P0,n", [
    (2, 8, 2, 128, 256, 40, 700, 33),    # batch strides, GQA 4
    (1, 8, 8, 128, 300, 0, 900, 20),     # GQA 1, w0 = 0
    (1, 16, 2, 64, 100, 500, 1000, 9),   # GQA 8, w0 larger than the chunk's distance
    (3, 4, 2, 64, 64, 7, 150, 50),       # B = 3, G from 200 = 4
])
def test_chunk_shapes(B, Hq, Hkv, D, wp, w0, P0, n):
    w = Workload("chunk", B, Hq, Hkv, D, 0, wp, w0, 1e6, 21 + P0, False, kind="decode")
    out, lse, o_ref, lse_ref = run_chunk(w, P0, n)
    assert_o(f64(out), o_ref, "chunk shapes")
    assert_lse(f64(lse), lse_ref, "chunk shapes")


@pytest.mark.parametrize("Hq,Hkv,D,wp,w0,P0,n", [
    (4, 1, 64, 1024, 300, 2900, 100),   # G = 3: 24 splits of ~27 visits; splits remote-only,
                                        # local-only, and across the remote-to-local switch
    (4, 2, 128, 4096, 200, 2000, 129),  # G = 1 (plain causal), two query tiles, ragged tail
    (2, 2, 64, 512, 0, 1800, 7),        # w0 = 0, a chunk just above the path threshold
    (8, 2, 128, 256, 1000, 1500, 40),   # w0 beyond most of the chunk's keys: few remote tiles
])
def test_chunk_key_split_every_row(Hq, Hkv, D, wp, w0, P0, n):
    # Short chunks on the tensor path split each query tile's key visits
    # into ranges (one CTA each) merged by log-sum-exp; every row against the
    # oracle.
    assert n >= jl.CHUNK_TENSOR_MIN
    w = Workload("chunk_split", 1, Hq, Hkv, D, 0, wp, w0, 1e6, 61 + n, False, kind="decode")
    out, lse, o_ref, lse_ref = run_chunk(w, P0, n)
    assert_o(f64(out), o_ref, "key split")
    assert_lse(f64(lse), lse_ref, "key split")


def test_chunk_key_split_at_the_largest_split_count():
    # one query tile and one head pair: 148 splits of about one key tile each
    # (the merge's widest case), G = 5, every row against the oracle
    w = Workload("chunk_split148", 1, 2, 1, 64, 0, 4096, 1000, 1e4, 71, True, kind="decode")
    P0, n = 19000, 8
    assert jl.jetlong_prefill_chunk_workspace_size(1, 2, 1, P0, n, 64) > 3 * (P0 + n) * 64 * 2
    out, lse, o_ref, lse_ref = run_chunk(w, P0, n)
    assert_o(f64(out), o_ref, "148 splits")
    assert_lse(f64(lse), lse_ref, "148 splits")


def test_chunk_across_the_appendix_e_boundary_uses_one_group_size():
    # P0 + n = 98,308: G = 4 for every query of the chunk, although a
    # token-by-token decode would use G = 3 for the first four of them.
    w = Workload("chunk_e", 1, 8, 2, 128, 0, 32768, 2048, 1e6, 31, False, kind="decode")
    assert jl.jetlong_group_size(98300 + 8, w.w_pretrained) == 4
    assert jl.jetlong_group_size(98301, w.w_pretrained) == 3
    out, lse, o_ref, lse_ref = run_chunk(w, 98300, 8)
    assert_o(f64(out), o_ref, "Appendix E chunk")
    assert_lse(f64(lse), lse_ref, "Appendix E chunk")


def test_qwen3_8b_chunk_at_128k():
    w = Workload("chunk_8b", 1, 32, 8, 128, 0, 32768, 4096, 1e6, 41, False, kind="decode")
    out, lse, o_ref, lse_ref = run_chunk(w, 131072 - 64, 64, Lcap_extra=0)
    assert_o(f64(out), o_ref, "8B 128K chunk")
    assert_lse(f64(lse), lse_ref, "8B 128K chunk")


def test_qwen3_8b_long_chunk_at_128k_sampled_rows():
    # A 4096-token chunk closing a 128K prompt runs on the tensor-core prefill
    # kernel (queries P0.., keys [0, P0 + n) of the cache); sampled queries
    # against the oracle with the call's G (from P0 + n = 131072).
    w = Workload("chunk_8b_long", 1, 32, 8, 128, 0, 32768, 4096, 1e6, 43, False, kind="decode")
    n = 4096
    P0 = 131072 - n
    x = generation_inputs(w, P0, n)
    cache = torch.from_numpy(oracle.rope_cache(f64(x.k_raw), 0, w.theta)).to(torch.bfloat16)
    q = torch.randn((w.B, n, w.Hq, w.D), generator=torch.Generator().manual_seed(w.seed + 5))
    q = q.to(torch.bfloat16)
    out, lse = jl.jetlong_prefill_chunk(q.cuda(), cache.cuda(), x.v.cuda(), P0, w.w_pretrained,
                                        w.w0, w.theta, out_dtype=torch.float32)
    assert jl.jetlong_device_status() == jl.JL_OK
    rows = [0, 1, 127, 128, 2048, n - 2, n - 1] + sorted(
        torch.randint(2, n - 2, (3,), generator=torch.Generator().manual_seed(7)).tolist())
    o_ref, lse_ref = oracle.prefill_chunk(f64(q), f64(cache), f64(x.v), P0, w.w_pretrained, w.w0,
                                          w.theta, rows=rows)
    assert_o(f64(out[:, rows]), o_ref[:, rows], "8B 128K long chunk")
    assert_lse(f64(lse[:, :, rows]), lse_ref[:, :, rows], "8B 128K long chunk")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("n", [jl.CHUNK_TENSOR_MIN - 1, jl.CHUNK_TENSOR_MIN, 23, 24])
def test_chunks_on_both_sides_of_the_path_threshold(n):
    # n below the threshold runs on the decode kernels, n at or above it on the
    # prefill kernel (with the keys split: one query tile here): the same
    # cache, both against the oracle
    w = Workload("chunk_thr", 1, 8, 2, 128, 0, 1024, 300, 1e6, 51, True, kind="decode")
    out, lse, o_ref, lse_ref = run_chunk(w, 5000 - n, n)
    assert_o(f64(out), o_ref, f"n={n}")
    assert_lse(f64(lse), lse_ref, f"n={n}")
