"""Python binding of the C ABI in include/jetlong.h (ctypes).

The functions here only marshal arguments: they check tensor shapes, dtypes
and devices, allocate outputs / workspace with torch when the caller does not
pass them, and call the library.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  If ``libjetlong.so`` has not
been built, the first call raises.

Names and argument order follow the C functions.  Tensors are the layouts the
header documents ([B, L, H, D] BF16 inputs, etc.).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjetlong.so")

JL_OK = 0
JL_ERR_NULL = -1
JL_ERR_SHAPE = -2
JL_ERR_UNSUPPORTED = -3
JL_ERR_ALIGN = -4
JL_ERR_WORKSPACE = -5
JL_ERR_CUDA = -6
JL_ERR_DEVICE_TIMEOUT = -7
JL_ERR_NO_DEVICE = -8
JL_ERR_RANGE = -9
JL_BF16 = 0
JL_F32 = 1
CHUNK_TENSOR_MIN = 6  # JL_CHUNK_TENSOR_MIN: chunks this long take the tensor-core path

# Every symbol the header declares, with its ctypes signature.
_VP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "jetlong_status_string": (ctypes.c_char_p, [_I]),
    "jetlong_version": (ctypes.c_char_p, []),
    "jetlong_shutdown": (None, []),
    "jetlong_group_size": (_I, [_I, _I]),
    "jetlong_prefill_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "jetlong_prefill": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                             _VP, _I, _VP, _SZ, _VP]),
    "jetlong_prefill_rotate": (_I, [_VP, _VP, _I, _I, _I, _I, _I, _F, _VP, _I, _VP, _SZ, _VP]),
    "jetlong_prefill_attend": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I, _VP, _SZ,
                                    _VP]),
    "jetlong_prefill_three_pass_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "jetlong_prefill_three_pass": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F,
                                        _I, _VP, _SZ, _VP]),
    "jetlong_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "jetlong_prefill_chunk_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "jetlong_prefill_chunk": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                   _F, _I, _VP, _SZ, _VP]),
    "jetlong_decode": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                            _VP, _SZ, _VP]),
    "jetlong_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                    _I, _VP]),
    "jetlong_prefill_interp": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _F,
                                    _F, _I, _VP, _I, _VP, _SZ, _VP]),
    "jetlong_decode_interp": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                   _F, _F, _I, _VP, _SZ, _VP]),
    "jetlong_prefill_chunk_interp": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I,
                                          _I, _I, _F, _F, _F, _I, _VP, _SZ, _VP]),
    "jetlong_remote_cache": (_I, [_VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _F, _VP]),
    "jetlong_decode_two_form": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I,
                                     _I, _F, _I, _VP, _SZ, _VP]),
    "jetlong_rope_cache": (_I, [_VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP]),
    "jetlong_device_status": (_I, [_VP]),
    "jetlong_check_device_timeout": (_I, [_I, _VP]),
}

_lib = None


class JetLongError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libjetlong.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m zero_shot_rope_bifocal_b200.build`")
        so = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(so, name)
            fn.restype = res
            fn.argtypes = args
        _lib = so
    return _lib


def status_string(status: int) -> str:
    return lib().jetlong_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != JL_OK:
        raise JetLongError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _require(t, name, shape, dtype):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device (and its stream)
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}; use torch.cuda.set_device")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out_dtype(dtype) -> int:
    if dtype in (torch.bfloat16, JL_BF16):
        return JL_BF16
    if dtype in (torch.float32, JL_F32):
        return JL_F32
    raise ValueError("out dtype must be torch.bfloat16 or torch.float32")


def _out_code(out, out_dtype) -> int:
    """The jl_dtype of a caller's ``out`` tensor, or of ``out_dtype`` if none."""
    if out is None:
        return _out_dtype(out_dtype)
    if not isinstance(out, torch.Tensor):
        raise TypeError("out must be a torch.Tensor")
    return _out_dtype(out.dtype)


def _ws(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns blocks aligned to at least 512 bytes.
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def _workspace(workspace, nbytes: int, device):
    """The caller's workspace (checked: a contiguous tensor on the current
    CUDA device), or a new one of ``nbytes``.  Returns (tensor, its bytes)."""
    if workspace is None:
        workspace = _ws(nbytes, device)
    elif not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    elif workspace.device.index != torch.cuda.current_device():
        raise ValueError(f"workspace is on {workspace.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}")
    elif not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    return workspace, workspace.numel() * workspace.element_size()


# ---------------------------------------------------------------- host-only helpers
def jetlong_group_size(L: int, w_pretrained: int) -> int:
    g = lib().jetlong_group_size(int(L), int(w_pretrained))
    if g < 1:
        raise JetLongError("jetlong_group_size", g)
    return g


def jetlong_prefill_workspace_size(B, Hq, Hkv, L, D) -> int:
    return int(lib().jetlong_prefill_workspace_size(B, Hq, Hkv, L, D))


def jetlong_prefill_three_pass_workspace_size(B, Hq, Hkv, L, D) -> int:
    return int(lib().jetlong_prefill_three_pass_workspace_size(B, Hq, Hkv, L, D))


def jetlong_decode_workspace_size(B, Hq, Hkv, L, D) -> int:
    return int(lib().jetlong_decode_workspace_size(B, Hq, Hkv, L, D))


# ---------------------------------------------------------------- device calls
def jetlong_prefill(q, k, v, w_pretrained: int, w0: int, rope_theta: float, *,
                    out=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                    k_cache_out=None, workspace=None, stream=None):
    """Bifocal causal attention over a prompt.  Returns (out, lse or None)."""
    return _prefill("jetlong_prefill", q, k, v, w_pretrained, w0, (float(rope_theta),), out, lse,
                    out_dtype, want_lse, k_cache_out, workspace, stream)


def jetlong_prefill_interp(q, k, v, w_pretrained: int, w0: int, rope_theta: float,
                           ramp_alpha: float = 1.0, ramp_beta: float = 32.0, *, out=None,
                           lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                           k_cache_out=None, workspace=None, stream=None):
    """jetlong_prefill with the frequency-interpolation remote map (remote
    pairs at true positions, interpolated frequencies).  Returns (out, lse)."""
    return _prefill("jetlong_prefill_interp", q, k, v, w_pretrained, w0,
                    (float(rope_theta), float(ramp_alpha), float(ramp_beta)), out, lse, out_dtype,
                    want_lse, k_cache_out, workspace, stream)


def _prefill(fn, q, k, v, w_pretrained, w0, method, out, lse, out_dtype, want_lse, k_cache_out,
             workspace, stream):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be [B, L, H, D]")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(q, "q", (B, L, Hq, D), torch.bfloat16)
    _require(k, "k", (B, L, Hkv, D), torch.bfloat16)
    _require(v, "v", (B, L, Hkv, D), torch.bfloat16)
    od = _out_code(out, out_dtype)
    if out is None:
        out = torch.empty((B, L, Hq, D), dtype=torch.bfloat16 if od == JL_BF16 else torch.float32,
                          device=q.device)
    _require(out, "out", (B, L, Hq, D), out.dtype)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    if lse is not None:
        _require(lse, "lse", (B, Hq, L), torch.float32)
    cap = 0
    if k_cache_out is not None:
        if k_cache_out.dim() != 4:
            raise ValueError("k_cache_out must be [B, Lcap, Hkv, D]")
        cap = k_cache_out.shape[1]
        _require(k_cache_out, "k_cache_out", (B, cap, Hkv, D), torch.bfloat16)
    workspace, ws_bytes = _workspace(
        workspace, jetlong_prefill_workspace_size(B, Hq, Hkv, L, D), q.device)
    st = getattr(lib(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, L, D,
                            int(w_pretrained), int(w0), *method, od, _ptr(k_cache_out), cap,
                            _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(fn, st)
    return out, lse


def jetlong_prefill_rotate(k, v, w_pretrained: int, rope_theta: float, workspace, *,
                           k_cache_out=None, stream=None):
    """Stage 1 of jetlong_prefill: the FP16 key operands into ``workspace``."""
    if k.dim() != 4:
        raise ValueError("k and v must be [B, L, Hkv, D]")
    B, L, Hkv, D = k.shape
    _require(k, "k", (B, L, Hkv, D), torch.bfloat16)
    _require(v, "v", (B, L, Hkv, D), torch.bfloat16)
    cap = 0 if k_cache_out is None else k_cache_out.shape[1]
    if k_cache_out is not None:
        _require(k_cache_out, "k_cache_out", (B, cap, Hkv, D), torch.bfloat16)
    workspace, ws_bytes = _workspace(workspace, 0, k.device)
    st = lib().jetlong_prefill_rotate(_ptr(k), _ptr(v), B, Hkv, L, D, int(w_pretrained),
                                      float(rope_theta), _ptr(k_cache_out), cap, _ptr(workspace),
                                      ws_bytes, _stream_ptr(stream))
    _check("jetlong_prefill_rotate", st)


def jetlong_prefill_attend(q, out, lse, Hkv: int, w_pretrained: int, w0: int, rope_theta: float,
                           workspace, *, stream=None):
    """Stage 2 of jetlong_prefill: the attention kernel (queries rotated as
    they are loaded) on the key operands in ``workspace``."""
    od = _out_code(out, None)
    if q.dim() != 4 or out.dim() != 4:
        raise ValueError("q and out must be [B, L, Hq, D]")
    B, L, Hq, D = q.shape
    _require(q, "q", (B, L, Hq, D), torch.bfloat16)
    _require(out, "out", (B, L, Hq, D), out.dtype)
    if lse is not None:
        _require(lse, "lse", (B, Hq, L), torch.float32)
    workspace, ws_bytes = _workspace(workspace, 0, out.device)
    st = lib().jetlong_prefill_attend(_ptr(q), _ptr(out), _ptr(lse), B, Hq, int(Hkv), L, D,
                                      int(w_pretrained), int(w0), float(rope_theta), od,
                                      _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check("jetlong_prefill_attend", st)


def jetlong_prefill_three_pass(q, k, v, w_pretrained: int, w0: int, rope_theta: float, *,
                               out=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                               workspace=None, stream=None):
    """The unfused three-pass (inclusion-exclusion) form of jetlong_prefill.
    Returns (out, lse or None)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be [B, L, H, D]")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(q, "q", (B, L, Hq, D), torch.bfloat16)
    _require(k, "k", (B, L, Hkv, D), torch.bfloat16)
    _require(v, "v", (B, L, Hkv, D), torch.bfloat16)
    od = _out_code(out, out_dtype)
    if out is None:
        out = torch.empty((B, L, Hq, D), dtype=torch.bfloat16 if od == JL_BF16 else torch.float32,
                          device=q.device)
    _require(out, "out", (B, L, Hq, D), out.dtype)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    if lse is not None:
        _require(lse, "lse", (B, Hq, L), torch.float32)
    workspace, ws_bytes = _workspace(
        workspace, jetlong_prefill_three_pass_workspace_size(B, Hq, Hkv, L, D), q.device)
    st = lib().jetlong_prefill_three_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq,
                                          Hkv, L, D, int(w_pretrained), int(w0),
                                          float(rope_theta), od, _ptr(workspace), ws_bytes,
                                          _stream_ptr(stream))
    _check("jetlong_prefill_three_pass", st)
    return out, lse


def jetlong_decode(q, k_cache, v_cache, L: int, w_pretrained: int, w0: int, rope_theta: float, *,
                   out=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                   workspace=None, stream=None):
    """One decode step at position L-1 on a true-position cache.  Returns (out, lse)."""
    return _decode("jetlong_decode", q, k_cache, v_cache, L, w_pretrained, w0,
                   (float(rope_theta),), out, lse, out_dtype, want_lse, workspace, stream)


def jetlong_decode_interp(q, k_cache, v_cache, L: int, w_pretrained: int, w0: int,
                          rope_theta: float, ramp_alpha: float = 1.0, ramp_beta: float = 32.0, *,
                          out=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                          workspace=None, stream=None):
    """jetlong_decode with the frequency-interpolation remote map."""
    return _decode("jetlong_decode_interp", q, k_cache, v_cache, L, w_pretrained, w0,
                   (float(rope_theta), float(ramp_alpha), float(ramp_beta)), out, lse, out_dtype,
                   want_lse, workspace, stream)


def _decode(fn, q, k_cache, v_cache, L, w_pretrained, w0, method, out, lse, out_dtype, want_lse,
            workspace, stream):
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and the caches [B, Lcap, Hkv, D]")
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _require(q, "q", (B, Hq, D), torch.bfloat16)
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    _require(v_cache, "v_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    od = _out_code(out, out_dtype)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16 if od == JL_BF16 else torch.float32,
                          device=q.device)
    _require(out, "out", (B, Hq, D), out.dtype)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _require(lse, "lse", (B, Hq), torch.float32)
    workspace, ws_bytes = _workspace(
        workspace, jetlong_decode_workspace_size(B, Hq, Hkv, int(L), D), q.device)
    st = getattr(lib(), fn)(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, Hq,
                            Hkv, int(L), Lcap, D, int(w_pretrained), int(w0), *method, od,
                            _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(fn, st)
    return out, lse


def jetlong_prefill_chunk_workspace_size(B, Hq, Hkv, P0, n, D) -> int:
    return int(lib().jetlong_prefill_chunk_workspace_size(B, Hq, Hkv, P0, n, D))


def jetlong_prefill_chunk(q, k_cache, v_cache, P0: int, w_pretrained: int, w0: int,
                          rope_theta: float, *, out=None, lse=None, out_dtype=torch.bfloat16,
                          want_lse: bool = True, workspace=None, stream=None):
    """Queries of a chunk at positions P0.. against a true-position cache that
    already holds the chunk's keys; one G from P0 + n.  Returns (out, lse)."""
    return _chunk("jetlong_prefill_chunk", q, k_cache, v_cache, P0, w_pretrained, w0,
                  (float(rope_theta),), out, lse, out_dtype, want_lse, workspace, stream)


def jetlong_prefill_chunk_interp(q, k_cache, v_cache, P0: int, w_pretrained: int, w0: int,
                                 rope_theta: float, ramp_alpha: float = 1.0,
                                 ramp_beta: float = 32.0, *, out=None, lse=None,
                                 out_dtype=torch.bfloat16, want_lse: bool = True, workspace=None,
                                 stream=None):
    """jetlong_prefill_chunk with the frequency-interpolation remote map."""
    return _chunk("jetlong_prefill_chunk_interp", q, k_cache, v_cache, P0, w_pretrained, w0,
                  (float(rope_theta), float(ramp_alpha), float(ramp_beta)), out, lse, out_dtype,
                  want_lse, workspace, stream)


def _chunk(fn, q, k_cache, v_cache, P0, w_pretrained, w0, method, out, lse, out_dtype, want_lse,
           workspace, stream):
    if q.dim() != 4 or k_cache.dim() != 4:
        raise ValueError("q must be [B, n, Hq, D] and the caches [B, Lcap, Hkv, D]")
    B, n, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _require(q, "q", (B, n, Hq, D), torch.bfloat16)
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    _require(v_cache, "v_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    od = _out_code(out, out_dtype)
    if out is None:
        out = torch.empty((B, n, Hq, D), dtype=torch.bfloat16 if od == JL_BF16 else torch.float32,
                          device=q.device)
    _require(out, "out", (B, n, Hq, D), out.dtype)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, n), dtype=torch.float32, device=q.device)
    if lse is not None:
        _require(lse, "lse", (B, Hq, n), torch.float32)
    workspace, ws_bytes = _workspace(
        workspace, jetlong_prefill_chunk_workspace_size(B, Hq, Hkv, int(P0), n, D), q.device)
    st = getattr(lib(), fn)(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, Hq,
                            Hkv, int(P0), n, Lcap, D, int(w_pretrained), int(w0), *method, od,
                            _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(fn, st)
    return out, lse


def jetlong_decode_noalloc(q, k_cache, v_cache, L: int, w_pretrained: int, w0: int,
                           rope_theta: float, out, lse=None, *, stream=None):
    """jetlong_decode for callers that cannot allocate device memory: the
    library keeps the split partials in its own fixed 8 MiB device buffer.
    ``out`` (and ``lse``, if given) are caller-provided; nothing is allocated."""
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _require(q, "q", (B, Hq, D), torch.bfloat16)
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    _require(v_cache, "v_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    od = _out_code(out, None)
    _require(out, "out", (B, Hq, D), out.dtype)
    if lse is not None:
        _require(lse, "lse", (B, Hq), torch.float32)
    st = lib().jetlong_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                      B, Hq, Hkv, int(L), Lcap, D, int(w_pretrained), int(w0),
                                      float(rope_theta), od, _stream_ptr(stream))
    _check("jetlong_decode_noalloc", st)
    return out, lse


def jetlong_remote_cache(k_cache, k_remote, j0: int, j1: int, L: int, w_pretrained: int,
                         rope_theta: float, *, stream=None):
    """Write rows [j0, j1) of the FP16 remote form of the key cache for the G
    of length L: k_remote[:, j] = R(f(j) - j) k_cache[:, j]."""
    B, Lcap, Hkv, D = k_cache.shape
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    _require(k_remote, "k_remote", (B, Lcap, Hkv, D), torch.float16)
    st = lib().jetlong_remote_cache(_ptr(k_cache), _ptr(k_remote), B, Lcap, Hkv, D, int(j0),
                                    int(j1), int(L), int(w_pretrained), float(rope_theta),
                                    _stream_ptr(stream))
    _check("jetlong_remote_cache", st)
    return k_remote


def jetlong_decode_two_form(q, k_cache, k_remote, v_cache, L: int, w_pretrained: int, w0: int,
                            rope_theta: float, *, out=None, lse=None, out_dtype=torch.bfloat16,
                            want_lse: bool = True, workspace=None, stream=None):
    """jetlong_decode reading remote keys from the remote form of the cache
    (written by jetlong_remote_cache for the G of this L).  Returns (out, lse)."""
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and the caches [B, Lcap, Hkv, D]")
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _require(q, "q", (B, Hq, D), torch.bfloat16)
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    _require(k_remote, "k_remote", (B, Lcap, Hkv, D), torch.float16)
    _require(v_cache, "v_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    od = _out_dtype(out_dtype if out is None else out.dtype)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16 if od == JL_BF16 else torch.float32,
                          device=q.device)
    _require(out, "out", (B, Hq, D), out.dtype)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _require(lse, "lse", (B, Hq), torch.float32)
    workspace, ws_bytes = _workspace(
        workspace, jetlong_decode_workspace_size(B, Hq, Hkv, int(L), D), q.device)
    st = lib().jetlong_decode_two_form(_ptr(q), _ptr(k_cache), _ptr(k_remote), _ptr(v_cache),
                                       _ptr(out), _ptr(lse), B, Hq, Hkv, int(L), Lcap, D,
                                       int(w_pretrained), int(w0), float(rope_theta), od,
                                       _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check("jetlong_decode_two_form", st)
    return out, lse


def jetlong_rope_cache(k, k_cache, pos0: int, rope_theta: float, *, stream=None):
    """Write RoPE(k[:, t], pos0 + t) into k_cache[:, pos0 + t] (true positions)."""
    B, n, Hkv, D = k.shape
    Lcap = k_cache.shape[1]
    _require(k, "k", (B, n, Hkv, D), torch.bfloat16)
    _require(k_cache, "k_cache", (B, Lcap, Hkv, D), torch.bfloat16)
    st = lib().jetlong_rope_cache(_ptr(k), _ptr(k_cache), B, n, Hkv, D, int(pos0), Lcap,
                                  float(rope_theta), _stream_ptr(stream))
    _check("jetlong_rope_cache", st)
    return k_cache


def jetlong_check_device_timeout(limit_ms: int = 50, *, stream=None) -> None:
    """Launch the bounded-wait timeout check (a wait that nothing completes);
    the next jetlong_device_status() returns JL_ERR_DEVICE_TIMEOUT."""
    _check("jetlong_check_device_timeout",
           lib().jetlong_check_device_timeout(int(limit_ms), _stream_ptr(stream)))


def jetlong_device_status(stream=None) -> int:
    """Synchronise the stream; return the library's device status code."""
    return int(lib().jetlong_device_status(_stream_ptr(stream)))
