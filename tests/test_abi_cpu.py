"""C-ABI checks that need no GPU: the library loads, exports every function
include/jetlong.h declares, answers the host-only queries, and rejects
invalid arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

import oracle
from zero_shot_rope_bifocal_b200 import build as jl_build
from zero_shot_rope_bifocal_b200 import jetlong as jl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jetlong.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(jl.LIB_PATH):
        jl_build.build()
    return jl.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"JL_API\s+[\w\s\*]+?\b(jetlong_\w+)\s*\(", text)


def test_header_declares_the_api():
    names = set(declared_functions())
    assert {"jetlong_prefill", "jetlong_decode", "jetlong_rope_cache", "jetlong_group_size",
            "jetlong_prefill_workspace_size", "jetlong_decode_workspace_size",
            "jetlong_status_string", "jetlong_device_status", "jetlong_version"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(jl.SIGNATURES), "binding and header disagree"


def test_only_the_c_abi_is_exported(lib):
    out = os.popen(f"nm -D --defined-only {jl.LIB_PATH}").read()
    funcs = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert funcs == set(declared_functions()), funcs ^ set(declared_functions())


def test_group_size_agrees_with_oracle(lib):
    for w in (1, 7, 128, 32768):
        for L in list(range(1, 3 * w + 5, max(1, w // 7))) + [98304, 98305, 131072, 2 ** 31 - 1]:
            assert jl.jetlong_group_size(L, w) == oracle.group_size(L, w), (L, w)
    assert lib.jetlong_group_size(0, 5) == jl.JL_ERR_SHAPE
    assert lib.jetlong_group_size(5, 0) == jl.JL_ERR_SHAPE


def test_workspace_sizes(lib):
    n = jl.jetlong_prefill_workspace_size(1, 32, 8, 131072, 128)
    assert n >= 2 * 3 * 8 * 131072 * 128
    assert jl.jetlong_prefill_workspace_size(1, 3, 2, 100, 128) == 0  # Hq % Hkv != 0
    assert jl.jetlong_prefill_workspace_size(1, 2, 1, 100, 96) == 0   # unsupported D
    prev = 0
    for L in (1, 63, 64, 65, 1000, 4096, 32768, 65536, 131072, 1 << 20):
        cur = jl.jetlong_decode_workspace_size(1, 32, 8, L, 128)
        assert cur >= prev and cur > 0
        prev = cur


def test_shutdown_can_be_called_without_a_device(lib):
    lib.jetlong_shutdown()
    lib.jetlong_shutdown()
    assert jl.jetlong_group_size(131072, 32768) == 4


def test_status_strings(lib):
    for code in range(-9, 1):
        assert jl.status_string(code).startswith("JL_")
    assert jl.status_string(5) == "unknown jl_status"


P = ctypes.c_void_p(256)  # a non-NULL, aligned stand-in pointer; never dereferenced


def prefill_call(lib, **kw):
    a = dict(q=P, k=P, v=P, out=P, lse=None, B=1, Hq=2, Hkv=1, L=512, D=64, wp=128, w0=32,
             theta=1e4, od=0, kc=None, cap=0, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.jetlong_prefill(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                               a["L"], a["D"], a["wp"], a["w0"], a["theta"], a["od"], a["kc"],
                               a["cap"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), jl.JL_ERR_NULL),
    (dict(out=None), jl.JL_ERR_NULL),
    (dict(B=0), jl.JL_ERR_SHAPE),
    (dict(L=0), jl.JL_ERR_SHAPE),
    (dict(Hq=3, Hkv=2), jl.JL_ERR_SHAPE),
    (dict(D=96), jl.JL_ERR_UNSUPPORTED),
    (dict(D=256), jl.JL_ERR_UNSUPPORTED),
    (dict(w0=-1), jl.JL_ERR_SHAPE),
    (dict(wp=0), jl.JL_ERR_SHAPE),
    (dict(theta=0.0), jl.JL_ERR_SHAPE),
    (dict(theta=float("nan")), jl.JL_ERR_SHAPE),
    (dict(od=2), jl.JL_ERR_UNSUPPORTED),
    (dict(kc=P, cap=100), jl.JL_ERR_SHAPE),
    (dict(q=ctypes.c_void_p(258)), jl.JL_ERR_ALIGN),
    (dict(lse=ctypes.c_void_p(260)), jl.JL_ERR_ALIGN),
    (dict(ws=None), jl.JL_ERR_WORKSPACE),
    (dict(wsb=10), jl.JL_ERR_WORKSPACE),
    (dict(ws=ctypes.c_void_p(272)), jl.JL_ERR_ALIGN),
    (dict(B=65536, L=1), jl.JL_ERR_SHAPE),              # grid z (batch) beyond 65535
    (dict(Hq=70000, Hkv=70000, L=1), jl.JL_ERR_SHAPE),  # grid y (head pairs) beyond 65535
])
def test_prefill_rejects_bad_arguments(lib, kw, status):
    assert prefill_call(lib, **kw) == status


def three_pass_call(lib, **kw):
    a = dict(q=P, k=P, v=P, out=P, lse=None, B=1, Hq=2, Hkv=1, L=512, D=64, wp=128, w0=32,
             theta=1e4, od=0, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.jetlong_prefill_three_pass(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"],
                                          a["Hq"], a["Hkv"], a["L"], a["D"], a["wp"], a["w0"],
                                          a["theta"], a["od"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(v=None), jl.JL_ERR_NULL),
    (dict(Hq=3, Hkv=2), jl.JL_ERR_SHAPE),
    (dict(D=32), jl.JL_ERR_UNSUPPORTED),
    (dict(w0=-1), jl.JL_ERR_SHAPE),
    (dict(od=7), jl.JL_ERR_UNSUPPORTED),
    (dict(out=ctypes.c_void_p(264)), jl.JL_ERR_ALIGN),
    (dict(ws=None), jl.JL_ERR_WORKSPACE),
])
def test_three_pass_rejects_bad_arguments(lib, kw, status):
    assert three_pass_call(lib, **kw) == status


def test_three_pass_needs_room_for_the_pass_outputs(lib):
    # Enough for the fused prefill's operands but not for the three fp32 pass
    # outputs and lse rows.
    B, Hq, Hkv, L, D = 1, 2, 1, 512, 64
    fused = jl.jetlong_prefill_workspace_size(B, Hq, Hkv, L, D)
    three = jl.jetlong_prefill_three_pass_workspace_size(B, Hq, Hkv, L, D)
    assert three >= fused + 3 * B * L * Hq * D * 4 + 3 * B * Hq * L * 4
    assert three_pass_call(lib, wsb=fused) == jl.JL_ERR_WORKSPACE
    assert three_pass_call(lib, wsb=three - 1) == jl.JL_ERR_WORKSPACE


@pytest.mark.parametrize("limit_ms", [0, -1, 2001])
def test_timeout_check_rejects_limits_out_of_range(lib, limit_ms):
    assert lib.jetlong_check_device_timeout(limit_ms, None) == jl.JL_ERR_SHAPE


def chunk_call(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, lse=None, B=1, Hq=32, Hkv=8, P0=1000, n=64, Lcap=1064,
             D=128, wp=32768, w0=4096, theta=1e6, od=0, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.jetlong_prefill_chunk(a["q"], a["kc"], a["vc"], a["out"], a["lse"], a["B"], a["Hq"],
                                     a["Hkv"], a["P0"], a["n"], a["Lcap"], a["D"], a["wp"],
                                     a["w0"], a["theta"], a["od"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), jl.JL_ERR_NULL),
    (dict(n=0), jl.JL_ERR_SHAPE),
    (dict(P0=-1), jl.JL_ERR_SHAPE),
    (dict(Lcap=1063), jl.JL_ERR_SHAPE),            # P0 + n > Lcap
    (dict(B=2, n=40000, Lcap=41000), jl.JL_ERR_SHAPE),  # B * n > 65535
    (dict(Hq=48), jl.JL_ERR_UNSUPPORTED),
    (dict(D=96), jl.JL_ERR_UNSUPPORTED),
    (dict(out=ctypes.c_void_p(260)), jl.JL_ERR_ALIGN),
    (dict(wsb=0), jl.JL_ERR_WORKSPACE),
])
def test_prefill_chunk_rejects_bad_arguments(lib, kw, status):
    assert chunk_call(lib, **kw) == status


def test_chunk_workspace_covers_a_decode_step():
    # a one-token chunk is a decode step: same plan, same workspace
    for L in (1, 1000, 131072):
        assert (jl.jetlong_prefill_chunk_workspace_size(1, 32, 8, L - 1, 1, 128) ==
                jl.jetlong_decode_workspace_size(1, 32, 8, L, 128))
    assert jl.jetlong_prefill_chunk_workspace_size(1, 32, 8, 0, 0, 128) == 0


def test_chunk_threshold_matches_the_header():
    m = re.search(r"#define JL_CHUNK_TENSOR_MIN (\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == jl.CHUNK_TENSOR_MIN


def test_chunk_workspace_holds_the_split_records():
    # tensor-core chunk path: the three FP16 key-operand arrays, then fp32
    # partial records [B, n, Hq, S, D + 2] when the keys are split into S
    # ranges (fewer than 75 query-tile x head-pair units; S = 148 / units,
    # at most the first tile's key tiles and 65535 / B), each 256-byte aligned
    al = lambda x: -(-x // 256) * 256
    for B, Hq, Hkv, P0, n, D in ((1, 32, 8, 131008, 64, 128), (1, 32, 8, 126976, 4096, 128),
                                 (1, 4, 1, 1000, 30, 64), (2, 16, 8, 300, 6, 128),
                                 (1, 8, 8, 0, 6, 64)):
        units = -(-n // 128) * Hkv * ((Hq // Hkv + 1) // 2) * B
        S = 1 if 2 * units > 148 else min(148 // units, (min(P0 + 128, P0 + n) - 1) // 128 + 1,
                                          65535 // B)
        rec = al(B * n * Hq * S * (D + 2) * 4) if S > 1 else 0
        want = 3 * al(B * Hkv * (P0 + n) * D * 2) + rec
        assert jl.jetlong_prefill_chunk_workspace_size(B, Hq, Hkv, P0, n, D) == want, (B, P0, n)
    # below the threshold a chunk is n decode problems: the decode plan's records
    n = jl.CHUNK_TENSOR_MIN - 1
    assert (jl.jetlong_prefill_chunk_workspace_size(1, 32, 8, 5000, n, 128) ==
            jl.jetlong_decode_workspace_size(n, 32, 8, 5000 + n, 128))


def decode_call(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, lse=None, B=1, Hq=32, Hkv=8, L=1000, Lcap=1000, D=128,
             wp=32768, w0=4096, theta=1e6, od=0, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.jetlong_decode(a["q"], a["kc"], a["vc"], a["out"], a["lse"], a["B"], a["Hq"],
                              a["Hkv"], a["L"], a["Lcap"], a["D"], a["wp"], a["w0"], a["theta"],
                              a["od"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(kc=None), jl.JL_ERR_NULL),
    (dict(Lcap=999), jl.JL_ERR_SHAPE),
    (dict(L=0), jl.JL_ERR_SHAPE),
    (dict(Hq=34, Hkv=2), jl.JL_ERR_UNSUPPORTED),   # group of 17 query heads
    (dict(Hq=48, Hkv=8), jl.JL_ERR_UNSUPPORTED),   # group of 6 query heads
    (dict(Hq=32, Hkv=2), jl.JL_ERR_UNSUPPORTED),   # group of 16 query heads
    (dict(D=80), jl.JL_ERR_UNSUPPORTED),
    (dict(w0=-5), jl.JL_ERR_SHAPE),
    (dict(vc=ctypes.c_void_p(8)), jl.JL_ERR_ALIGN),
    (dict(wsb=0), jl.JL_ERR_WORKSPACE),
    (dict(Hq=524288, Hkv=524288, L=1, Lcap=1), jl.JL_ERR_SHAPE),  # grid y beyond 65535
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert decode_call(lib, **kw) == status


@pytest.mark.parametrize("args,status", [
    ((None, P, 1, 4, 2, 128, 0, 8, 1e4, None), jl.JL_ERR_NULL),
    ((P, P, 1, 4, 2, 128, 5, 8, 1e4, None), jl.JL_ERR_SHAPE),     # pos0 + n > Lcap
    ((P, P, 1, 0, 2, 128, 0, 8, 1e4, None), jl.JL_ERR_SHAPE),
    ((P, P, 1, 4, 2, 48, 0, 8, 1e4, None), jl.JL_ERR_UNSUPPORTED),
    ((P, P, 1, 4, 2, 128, -1, 8, 1e4, None), jl.JL_ERR_SHAPE),
    ((P, P, 65536, 4, 2, 128, 0, 8, 1e4, None), jl.JL_ERR_SHAPE),  # grid y (batch) > 65535
])
def test_rope_cache_rejects_bad_arguments(lib, args, status):
    assert lib.jetlong_rope_cache(*args) == status


def test_stage_entry_points_check_their_own_buffers(lib):
    # rotate needs k, v; attend needs q (rotated in its load path) and out;
    # neither accepts a short workspace
    rot = lambda k=P, v=P, ws=P, wsb=1 << 40: lib.jetlong_prefill_rotate(
        k, v, 1, 1, 512, 64, 128, 1e4, None, 0, ws, wsb, None)
    att = lambda q=P, out=P, lse=None, ws=P, wsb=1 << 40: lib.jetlong_prefill_attend(
        q, out, lse, 1, 2, 1, 512, 64, 128, 32, 1e4, 0, ws, wsb, None)
    assert rot(v=None) == jl.JL_ERR_NULL
    assert rot(k=None) == jl.JL_ERR_NULL
    assert rot(v=ctypes.c_void_p(264)) == jl.JL_ERR_ALIGN
    assert rot(wsb=100) == jl.JL_ERR_WORKSPACE
    assert att(q=None) == jl.JL_ERR_NULL
    assert att(out=None) == jl.JL_ERR_NULL
    assert att(q=ctypes.c_void_p(264)) == jl.JL_ERR_ALIGN
    assert att(lse=ctypes.c_void_p(260)) == jl.JL_ERR_ALIGN
    assert att(ws=None) == jl.JL_ERR_WORKSPACE


def test_prefill_workspace_holds_only_the_key_operands():
    # the queries are rotated in the attention kernel's load path, so the
    # workspace holds k_true, k_remote and v: 3 x B.Hkv.L.D FP16 values
    for B, Hq, Hkv, L, D in ((1, 32, 8, 131072, 128), (2, 4, 2, 1000, 64)):
        n = jl.jetlong_prefill_workspace_size(B, Hq, Hkv, L, D)
        one = -(-(B * Hkv * L * D * 2) // 256) * 256
        assert n == 3 * one


# ---------------------------------------------------------------- frequency-interpolation map
def interp_calls(lib, alpha, beta, **kw):
    """The three interpolation entry points with otherwise valid arguments."""
    p = dict(q=P, k=P, v=P, out=P, lse=None, B=1, Hq=2, Hkv=1, L=512, D=64, wp=128, w0=32,
             theta=1e4, od=0, kc=None, cap=0, ws=P, wsb=1 << 40, stream=None)
    p.update(kw)
    pre = lib.jetlong_prefill_interp(p["q"], p["k"], p["v"], p["out"], p["lse"], p["B"], p["Hq"],
                                     p["Hkv"], p["L"], p["D"], p["wp"], p["w0"], p["theta"], alpha,
                                     beta, p["od"], p["kc"], p["cap"], p["ws"], p["wsb"],
                                     p["stream"])
    dec = lib.jetlong_decode_interp(p["q"], P, P, p["out"], p["lse"], p["B"], p["Hq"], p["Hkv"],
                                    p["L"], p["L"], p["D"], p["wp"], p["w0"], p["theta"], alpha,
                                    beta, p["od"], p["ws"], p["wsb"], p["stream"])
    chk = lib.jetlong_prefill_chunk_interp(p["q"], P, P, p["out"], p["lse"], p["B"], p["Hq"],
                                           p["Hkv"], p["L"] - 8, 8, p["L"], p["D"], p["wp"],
                                           p["w0"], p["theta"], alpha, beta, p["od"], p["ws"],
                                           p["wsb"], p["stream"])
    return pre, dec, chk


@pytest.mark.parametrize("alpha,beta", [(32.0, 1.0), (4.0, 4.0), (float("nan"), 32.0),
                                        (1.0, float("inf"))])
def test_interp_rejects_bad_ramp_bounds(lib, alpha, beta):
    assert interp_calls(lib, alpha, beta) == (jl.JL_ERR_SHAPE,) * 3


def test_interp_checks_the_same_arguments_as_the_aliasing_calls(lib):
    assert interp_calls(lib, 1.0, 32.0, q=None) == (jl.JL_ERR_NULL,) * 3
    assert interp_calls(lib, 1.0, 32.0, D=96) == (jl.JL_ERR_UNSUPPORTED,) * 3
    assert interp_calls(lib, 1.0, 32.0, wsb=0) == (jl.JL_ERR_WORKSPACE,) * 3


def test_decode_split_plan_fills_at_most_one_wave():
    # The decode grid is splits x ceil(Hkv / 8) x B CTAs at two CTAs per SM on
    # 148 SMs: the plan never starts a second wave (unless one split per
    # unit already does), and never splits finer than one 16-token stage.
    for B in (1, 2, 3, 4, 64, 300):
        for Hkv, Hq, D in ((8, 32, 128), (16, 16, 128), (2, 16, 64), (12, 24, 64)):
            units = B * -(-Hkv // 8)
            for L in (1, 15, 16, 17, 100, 4096, 32768, 131072, 1 << 20):
                ws = jl.jetlong_decode_workspace_size(B, Hq, Hkv, L, D)
                if B * L * Hq > 1 << 31:                  # beyond the index range: refused
                    assert ws == 0
                    continue
                per_split = B * Hq * (D + 2) * 4
                ns = ws // per_split
                assert ws - ns * per_split < 256          # only alignment padding left
                assert 1 <= ns <= -(-L // 16)
                assert units * ns <= max(2 * 148, units)


def test_binding_refuses_host_memory_as_workspace_or_operand():
    # a host pointer handed to the kernels would be dereferenced on the GPU
    import torch
    with pytest.raises(ValueError, match="workspace must be a CUDA tensor"):
        jl._workspace(torch.empty(64, dtype=torch.uint8), 64, None)
    with pytest.raises(ValueError, match="workspace must be a CUDA tensor"):
        jl._workspace(bytearray(64), 64, None)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        jl._require(torch.empty((1, 2), dtype=torch.bfloat16), "q", (1, 2), torch.bfloat16)


def noalloc_call(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, lse=None, B=1, Hq=32, Hkv=8, L=1000, Lcap=1000, D=128,
             wp=32768, w0=4096, theta=1e6, od=0, stream=None)
    a.update(kw)
    return lib.jetlong_decode_noalloc(a["q"], a["kc"], a["vc"], a["out"], a["lse"], a["B"],
                                      a["Hq"], a["Hkv"], a["L"], a["Lcap"], a["D"], a["wp"],
                                      a["w0"], a["theta"], a["od"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), jl.JL_ERR_NULL),
    (dict(out=None), jl.JL_ERR_NULL),
    (dict(L=0), jl.JL_ERR_SHAPE),
    (dict(Lcap=999), jl.JL_ERR_SHAPE),                 # L > Lcap
    (dict(Hq=48, Hkv=8), jl.JL_ERR_UNSUPPORTED),       # group of 6 query heads
    (dict(D=80), jl.JL_ERR_UNSUPPORTED),
    (dict(w0=-1), jl.JL_ERR_SHAPE),
    (dict(theta=float("nan")), jl.JL_ERR_SHAPE),
    (dict(od=3), jl.JL_ERR_UNSUPPORTED),
    (dict(kc=ctypes.c_void_p(264)), jl.JL_ERR_ALIGN),
    (dict(lse=ctypes.c_void_p(260)), jl.JL_ERR_ALIGN),
    (dict(B=512, L=16, Lcap=16), jl.JL_ERR_WORKSPACE),  # partials beyond its fixed buffer
])
def test_noalloc_decode_rejects_bad_arguments_without_a_device(lib, kw, status):
    # the same host checks as jetlong_decode, all before any CUDA call
    assert noalloc_call(lib, **kw) == status


def test_binding_refuses_an_out_that_is_not_a_tensor():
    import torch
    with pytest.raises(TypeError, match="out must be a torch.Tensor"):
        jl._out_code([0.0], torch.float32)
    with pytest.raises(ValueError, match="out dtype"):
        jl._out_code(torch.empty(1, dtype=torch.float16), None)
    assert jl._out_code(None, torch.float32) == jl.JL_F32


def test_header_states_the_fp16_range_contract():
    # a call that meets an input beyond FP16 still returns JL_OK; the report
    # comes from jetlong_device_status (prefill) or non-finite outputs (decode)
    text = " ".join(ln.strip().lstrip("*").strip() for ln in open(HEADER).read().splitlines())
    text = " ".join(text.split())
    assert "|x| <= 65504 after rotation" in text
    assert "still returns JL_OK, and its outputs may hold non-finite values" in text
    assert "the next jetlong_device_status() returns JL_ERR_RANGE" in text
    assert "record nothing" in text


# ---------------------------------------------------------------- two-form key cache
@pytest.mark.parametrize("args,status", [
    ((None, P, 1, 100, 8, 128, 0, 10, 100, 32, 1e4, None), jl.JL_ERR_NULL),
    ((P, P, 1, 100, 8, 128, 0, 10, 101, 32, 1e4, None), jl.JL_ERR_SHAPE),   # L > Lcap
    ((P, P, 1, 100, 8, 128, 5, 4, 100, 32, 1e4, None), jl.JL_ERR_SHAPE),    # j1 < j0
    ((P, P, 1, 100, 8, 128, 0, 60, 50, 32, 1e4, None), jl.JL_ERR_SHAPE),    # j1 > L
    ((P, P, 1, 100, 8, 96, 0, 10, 100, 32, 1e4, None), jl.JL_ERR_UNSUPPORTED),
    ((P, P, 1, 100, 8, 128, 0, 10, 100, 0, 1e4, None), jl.JL_ERR_SHAPE),    # w_pretrained
    ((P, ctypes.c_void_p(264), 1, 100, 8, 128, 0, 10, 100, 32, 1e4, None), jl.JL_ERR_ALIGN),
    ((P, P, 1, 100, 8, 128, 7, 7, 100, 32, 1e4, None), jl.JL_OK),          # nothing to write
])
def test_remote_cache_rejects_bad_arguments(lib, args, status):
    assert lib.jetlong_remote_cache(*args) == status


def test_two_form_decode_checks_its_remote_cache(lib):
    a = [P, P, P, P, P, None, 1, 32, 8, 1000, 1000, 128, 32768, 4096, 1e6, 0, P, 1 << 40, None]
    bad = list(a)
    bad[2] = None
    assert lib.jetlong_decode_two_form(*bad) == jl.JL_ERR_NULL
    bad = list(a)
    bad[2] = ctypes.c_void_p(264)
    assert lib.jetlong_decode_two_form(*bad) == jl.JL_ERR_ALIGN
    bad = list(a)
    bad[17] = 0
    assert lib.jetlong_decode_two_form(*bad) == jl.JL_ERR_WORKSPACE
