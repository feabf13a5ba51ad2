"""Python binding of the B200 exact-attention C ABI (``include/attn.h``).

Argument marshalling only: every function below checks dtypes, shapes and devices of torch tensors,
allocates outputs with torch when the caller passes none, and calls the entry point of the same name
in ``libattn_b200.so``. All attention arithmetic runs in that library's CUDA kernels; there is no
other code path. The library is loaded on first use; if it is missing, that first call raises ImportError saying
how to build it.
"""
from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn_b200.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
DECODE_STATIC_SCRATCH_BYTES = 48 << 20  # ATTN_DECODE_STATIC_SCRATCH_BYTES

# Function name -> (restype, argtypes), mirroring include/attn.h.
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "attn_decode_default_chunk": (_I, [_I, _I, _I]),
    "attn_decode_splitkv": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _F, _I, _P, ctypes.c_size_t, _P]),
    "attn_decode_splitkv_static": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_combine": (_I, [_P, _P, _I, _I, _I, _P, _P, _P]),
    "attn_get_last_error": (_I, []),
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_kernel_name": (ctypes.c_char_p, [_I]),
    "attn_selftest_bounded_wait": (_I, [ctypes.c_uint, _P]),
    "attn_selftest_pair_wait": (_I, [ctypes.c_uint, _I, _P]),
    "attn_selftest_exp2_poly": (_I, [_P, _P, _I, _P]),
    "attn_fp8_quantize": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, ctypes.c_size_t, _P]),
}


class AttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m exact_io_aware_41_b200.build` "
                          "(needs nvcc with sm_100a support)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_handle = None


def lib_handle() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises ImportError if it is not built)."""
    global _handle
    if _handle is None:
        _handle = _load()
    return _handle


def status_string(code: int) -> str:
    return lib_handle().attn_status_string(int(code)).decode()


def kernel_name(which: int) -> str | None:
    r = lib_handle().attn_kernel_name(int(which))
    return None if r is None else r.decode()


def _check(fn: str, code: int) -> None:
    if code != ATTN_OK:
        raise AttnError(fn, code)


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bf16_cuda(name, t, ndim):
    import torch

    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != ndim:
        raise ValueError(f"{name} must be a contiguous {ndim}-d bf16 CUDA tensor")


def attn_fwd(q, k, v, scale: float | None = None, causal: bool = False, out=None, lse=None, stream=None):
    """Prefill forward. q [B, Nq, Hq, d], k and v [B, Nkv, Hkv, d] (bf16, CUDA, contiguous).

    Returns (O [B, Nq, Hq, d] bf16, LSE [B, Hq, Nq] fp32).
    """
    import torch

    for n, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n, t, 4)
    B, Nq, Hq, d = q.shape
    _, Nkv, Hkv, _ = k.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Nkv, Hkv, d] with q's B and d")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    code = lib_handle().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                         Nq, Nkv, d, float(scale), int(bool(causal)), _stream(stream))
    _check("attn_fwd", code)
    return out, lse


def attn_decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, Nkv_cap: int, chunk: int = 0) -> int:
    return int(lib_handle().attn_decode_workspace_bytes(B, Hq, Hkv, d, Nkv_cap, chunk))


def attn_decode_default_chunk(B: int, Hkv: int, Nkv_cap: int) -> int:
    return int(lib_handle().attn_decode_default_chunk(B, Hkv, Nkv_cap))


def attn_decode_splitkv(q, k_cache, v_cache, kv_lens, scale: float | None = None, chunk: int = 0,
                        workspace=None, out=None, lse=None, stream=None):
    """Split-KV decode + combine. q [B, Hq, d]; caches [B, Nkv_cap, Hkv, d]; kv_lens int32 [B] (CUDA).

    Returns (O [B, Hq, d] bf16, LSE [B, Hq] fp32).
    """
    import torch

    _bf16_cuda("q", q, 3)
    _bf16_cuda("k_cache", k_cache, 4)
    _bf16_cuda("v_cache", v_cache, 4)
    if kv_lens.dtype != torch.int32 or not kv_lens.is_cuda or kv_lens.dim() != 1:
        raise ValueError("kv_lens must be a 1-d int32 CUDA tensor")
    B, Hq, d = q.shape
    _, cap, Hkv, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_decode_workspace_bytes(B, Hq, Hkv, d, cap, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    code = lib_handle().attn_decode_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), kv_lens.data_ptr(), cap,
                                    out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, d, float(scale), int(chunk),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    _check("attn_decode_splitkv", code)
    return out, lse


def attn_decode_splitkv_static(q, k_cache, v_cache, kv_lens, scale: float | None = None, chunk: int = 0, out=None,
                               lse=None, stream=None):
    """attn_decode_splitkv with its partials in the library's fixed device array (no workspace).

    For callers that cannot allocate device scratch. Outputs are allocated here only when the caller
    passes none; the library call itself allocates nothing. Calls that overlap on the GPU share the
    array and race.
    """
    import torch

    _bf16_cuda("q", q, 3)
    _bf16_cuda("k_cache", k_cache, 4)
    _bf16_cuda("v_cache", v_cache, 4)
    if kv_lens.dtype != torch.int32 or not kv_lens.is_cuda or kv_lens.dim() != 1:
        raise ValueError("kv_lens must be a 1-d int32 CUDA tensor")
    B, Hq, d = q.shape
    _, cap, Hkv, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    code = lib_handle().attn_decode_splitkv_static(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), kv_lens.data_ptr(),
                                           cap, out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, d, float(scale),
                                           int(chunk), _stream(stream))
    _check("attn_decode_splitkv_static", code)
    return out, lse


def attn_decode_combine(part_o, part_lse, out=None, lse=None, stream=None):
    """Combine partial states. part_o fp32 [rows, n_splits, d], part_lse fp32 [rows, n_splits]."""
    import torch

    rows, n_splits, d = part_o.shape
    if part_o.dtype != torch.float32 or part_lse.dtype != torch.float32 or part_lse.shape != (rows, n_splits):
        raise ValueError("part_o [rows, n_splits, d] and part_lse [rows, n_splits] must be fp32")
    if out is None:
        out = torch.empty((rows, d), dtype=torch.bfloat16, device=part_o.device)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=part_o.device)
    code = lib_handle().attn_decode_combine(part_o.data_ptr(), part_lse.data_ptr(), rows, n_splits, d, out.data_ptr(),
                                    lse.data_ptr(), _stream(stream))
    _check("attn_decode_combine", code)
    return out, lse


def attn_get_last_error() -> int:
    """Reads and clears the device error word (synchronises). Returns a status code."""
    return int(lib_handle().attn_get_last_error())


def attn_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    _check("attn_selftest_bounded_wait", lib_handle().attn_selftest_bounded_wait(int(limit_us), _stream(stream)))


def attn_selftest_pair_wait(limit_us: int, cross_arrive: bool, stream=None) -> None:
    _check("attn_selftest_pair_wait",
           lib_handle().attn_selftest_pair_wait(int(limit_us), 1 if cross_arrive else 0, _stream(stream)))


def attn_selftest_exp2_poly(x, out=None, stream=None):
    """2^x through the library's FMA-pipe exponential, for a contiguous fp32 CUDA tensor x."""
    import torch

    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous() or x.numel() < 1:
        raise ValueError("x must be a non-empty contiguous fp32 CUDA tensor")
    if out is None:
        out = torch.empty_like(x)
    _check("attn_selftest_exp2_poly",
           lib_handle().attn_selftest_exp2_poly(x.data_ptr(), out.data_ptr(), x.numel(), _stream(stream)))
    return out


def attn_fp8_quantize(x, signs=None, transpose: bool = False, out=None, amax=None, stream=None):
    """e4m3 codes of x [B, N, H, d] (bf16, d = 128) with per-(batch, head) maxima.

    signs: fp32 [d] of +-1 (CUDA) to rotate by diag(signs) H / sqrt(d) first (Q and K), or None (V).
    transpose: write codes as [B, H, d, N] (the layout attn_fwd_fp8 takes V in; N % 16 == 0).
    Returns (codes uint8, amax fp32 [B, H]).
    """
    import torch

    _bf16_cuda("x", x, 4)
    B, N, H, d = x.shape
    if signs is not None and (signs.dtype != torch.float32 or not signs.is_cuda or signs.shape != (d,)):
        raise ValueError("signs must be a fp32 CUDA tensor of shape [d]")
    if out is None:
        out = torch.empty((B, H, d, N) if transpose else (B, N, H, d), dtype=torch.uint8, device=x.device)
    if amax is None:
        amax = torch.empty((B, H), dtype=torch.float32, device=x.device)
    code = lib_handle().attn_fp8_quantize(x.data_ptr(), None if signs is None else signs.data_ptr(), out.data_ptr(),
                                          amax.data_ptr(), B, N, H, d, int(bool(transpose)), _stream(stream))
    _check("attn_fp8_quantize", code)
    return out, amax


def attn_fwd_fp8(q8, k8, vt8, amax_q, amax_k, amax_v, scale: float | None = None, causal: bool = False, out=None,
                 lse=None, stream=None):
    """8-bit prefill forward. q8 [B, Nq, Hq, d], k8 [B, Nkv, Hkv, d] (rotated codes), vt8 [B, Hkv, d, Nkv]
    (transposed V codes), amax_* fp32 [B, H] from attn_fp8_quantize. Returns (O bf16 [B, Nq, Hq, d],
    LSE fp32 [B, Hq, Nq])."""
    import torch

    for n, t in (("q8", q8), ("k8", k8), ("vt8", vt8)):
        if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{n} must be a contiguous 4-d uint8 CUDA tensor")
    B, Nq, Hq, d = q8.shape
    _, Nkv, Hkv, _ = k8.shape
    if vt8.shape != (B, Hkv, d, Nkv):
        raise ValueError("vt8 must be [B, Hkv, d, Nkv]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
    code = lib_handle().attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(), amax_q.data_ptr(), amax_k.data_ptr(),
                                     amax_v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nkv, d,
                                     float(scale), int(bool(causal)), _stream(stream))
    _check("attn_fwd_fp8", code)
    return out, lse


def attn_bwd_workspace_bytes(B: int, Hq: int, Nq: int, d: int) -> int:
    return int(lib_handle().attn_bwd_workspace_bytes(B, Hq, Nq, d))


def attn_bwd(q, k, v, o, lse, dout, scale: float | None = None, causal: bool = False, workspace=None, dq=None,
             dk=None, dv=None, stream=None):
    """Backward pass. q, o, dout [B, Nq, Hq, d], k, v [B, Nkv, Hkv, d] (bf16), lse fp32 [B, Hq, Nq] from
    attn_fwd. Returns (dQ, dK, dV) in the layouts of q, k, v."""
    import torch

    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _bf16_cuda(n, t, 4)
    B, Nq, Hq, d = q.shape
    _, Nkv, Hkv, _ = k.shape
    if o.shape != q.shape or dout.shape != q.shape or v.shape != k.shape or lse.shape != (B, Hq, Nq):
        raise ValueError("o, dout like q; v like k; lse [B, Hq, Nq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_bwd_workspace_bytes(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    code = lib_handle().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nkv, d,
                                 float(scale), int(bool(causal)), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_bwd", code)
    return dq, dk, dv
