"""Python binding of libq4dec: argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module
checks tensors, takes raw device pointers and the current torch stream, and
calls the C ABI (``include/q4dec.h``).  There is no fallback: if the shared
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_HERE, "libq4dec.so")
# libq4dec_debug.so: the same library built with Q4D_DEBUG (index checks of
# every global access into the device error record); chosen with
# Q4D_DEBUG=1 in the environment or use_debug_library().
DEBUG_LIB_PATH = os.path.join(_HERE, "libq4dec_debug.so")
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("Q4D_DEBUG") == "1" else RELEASE_LIB_PATH

STATUS = {
    0: "Q4D_OK",
    1: "Q4D_ERR_INVALID_ARG",
    2: "Q4D_ERR_UNSUPPORTED_SHAPE",
    3: "Q4D_ERR_MISALIGNED",
    4: "Q4D_ERR_WORKSPACE",
    5: "Q4D_ERR_CUDA",
    6: "Q4D_ERR_DEVICE_TIMEOUT",
    7: "Q4D_ERR_DEVICE_INDEX",
}

# Sites of the device error record's first failed index check.
CHECK_SITES = {
    1: "gemv weights", 2: "gemv activations", 3: "gemv output", 4: "gemv partial slots",
    5: "gemv batch counters", 16: "attention K/V", 17: "attention query",
    18: "attention output", 19: "attention split states", 32: "K/V append", 255: "self-test",
}

EXPORTS = (
    "q4d_version", "q4d_status_string",
    "q4_gemv", "q4_gemv_ex", "q4_gemv_ex2", "q4d_gemv_workspace_bytes",
    "q4kv_attn_decode", "q4kv_attn_decode_ex", "q4d_attn_workspace_bytes",
    "q4d_plan_gemv", "q4d_plan_attn", "q4d_device_error",
    "q4kv_attn_decode_noalloc",
    "q4d_pack_q4_0_weights", "q4d_unpack_q4_0_weights", "q4d_pack_q4_0_rows",
    "q4d_unpack_q4_0_rows", "q4kv_append", "q4_gemv_swiglu_ex",
    "q4d_gemv_swiglu_workspace_bytes", "q8kv_attn_decode_ex", "q8kv_attn_workspace_bytes",
    "q8kv_plan_attn", "q4d_wait_selftest",
    "q4d_gemv_batch_desc_bytes", "q4d_gemv_batch_prepare", "q4_gemv_batch_ex",
    "q4d_device_error_record", "q4d_debug_build", "q4d_debug_limit_weights",
    "q4d_index_check_selftest",
)


class Q4DecError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({lib().q4d_status_string(status).decode()})")


class GemvPlan(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int), ("threads", ctypes.c_int),
                ("row_blocks", ctypes.c_int), ("units_per_row_block", ctypes.c_int),
                ("units", ctypes.c_int), ("slots", ctypes.c_int),
                ("stages", ctypes.c_int), ("reserved", ctypes.c_int),
                ("smem_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t)]


class GemvJob(ctypes.Structure):
    """``q4d_gemv_job``: one GEMV of a batch launch."""
    _fields_ = [("W_q4", ctypes.c_void_p), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int), ("K", ctypes.c_int), ("flags", ctypes.c_uint),
                ("wait_for", ctypes.c_int)]


class AttnPlan(ctypes.Structure):
    _fields_ = [("n_splits", ctypes.c_int), ("split_tokens", ctypes.c_int),
                ("tile_tokens", ctypes.c_int), ("row_groups", ctypes.c_int),
                ("rows_per_cta", ctypes.c_int), ("stages", ctypes.c_int),
                ("threads", ctypes.c_int), ("smem_bytes", ctypes.c_size_t),
                ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def use_debug_library(debug: bool = True) -> str:
    """Choose the library that lib() returns from now on: the debug build
    (True) or the release build (False).  Both can be loaded in one process;
    work already launched through the other one is unaffected, and a
    prepared GemvBatch descriptor serves either.  Returns the chosen path."""
    global _lib, LIB_PATH
    path = DEBUG_LIB_PATH if debug else RELEASE_LIB_PATH
    if path != LIB_PATH:
        LIB_PATH = path
        _lib = None
    return path


def lib() -> ctypes.CDLL:
    """Load the library at LIB_PATH (libq4dec.so, built in-tree, unless the
    debug build was chosen); raise if it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_weight_streaming_dequant_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.q4d_version.restype = i
    L.q4d_status_string.argtypes = [i]
    L.q4d_status_string.restype = ctypes.c_char_p
    L.q4_gemv.argtypes = [vp, vp, vp, i, i, i]
    L.q4_gemv_ex.argtypes = [vp, vp, vp, i, i, i, vp, vp, sz]
    L.q4_gemv_ex2.argtypes = [vp, vp, vp, i, i, i, vp, vp, sz, ctypes.c_uint]
    L.q4d_gemv_workspace_bytes.argtypes = [i, i, i]
    L.q4d_gemv_workspace_bytes.restype = sz
    L.q4kv_attn_decode.argtypes = [vp, vp, vp, vp, i, i, i, i, i]
    L.q4kv_attn_decode_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp, vp, sz]
    L.q4d_attn_workspace_bytes.argtypes = [i, i, i, i, i]
    L.q4d_attn_workspace_bytes.restype = sz
    L.q4d_plan_gemv.argtypes = [i, i, i, i, ctypes.POINTER(GemvPlan)]
    L.q4d_plan_attn.argtypes = [i, i, i, i, i, i, ctypes.POINTER(AttnPlan)]
    L.q4d_device_error.argtypes = [i]
    L.q4kv_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    for fn in ("q4d_pack_q4_0_weights", "q4d_unpack_q4_0_weights", "q4d_pack_q4_0_rows",
               "q4d_unpack_q4_0_rows"):
        getattr(L, fn).argtypes = [vp, vp, i, i]
        getattr(L, fn).restype = i
    L.q4kv_append.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
    L.q4kv_append.restype = i
    L.q4_gemv_swiglu_ex.argtypes = [vp, vp, vp, i, i, i, vp, vp, sz, ctypes.c_uint]
    L.q4_gemv_swiglu_ex.restype = i
    L.q4d_gemv_swiglu_workspace_bytes.argtypes = [i, i, i]
    L.q4d_gemv_swiglu_workspace_bytes.restype = sz
    L.q4d_gemv_batch_desc_bytes.argtypes = [i]
    L.q4d_gemv_batch_desc_bytes.restype = sz
    L.q4d_gemv_batch_prepare.argtypes = [ctypes.POINTER(GemvJob), i, i, i, vp, sz,
                                         ctypes.POINTER(ctypes.c_size_t)]
    L.q4d_gemv_batch_prepare.restype = i
    L.q4_gemv_batch_ex.argtypes = [vp, vp, vp, vp, sz, ctypes.c_uint]
    L.q4_gemv_batch_ex.restype = i
    L.q8kv_attn_decode_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp, vp, sz]
    L.q8kv_attn_decode_ex.restype = i
    L.q8kv_attn_workspace_bytes.argtypes = [i, i, i, i, i]
    L.q8kv_attn_workspace_bytes.restype = sz
    L.q8kv_plan_attn.argtypes = [i, i, i, i, i, i, ctypes.POINTER(AttnPlan)]
    L.q8kv_plan_attn.restype = i
    L.q4d_wait_selftest.argtypes = [vp, ctypes.c_uint, i, vp]
    L.q4d_wait_selftest.restype = i
    L.q4d_device_error_record.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
    L.q4d_device_error_record.restype = i
    L.q4d_debug_build.argtypes = []
    L.q4d_debug_build.restype = i
    L.q4d_debug_limit_weights.argtypes = [ctypes.c_ulonglong]
    L.q4d_debug_limit_weights.restype = i
    L.q4d_index_check_selftest.argtypes = [vp, ctypes.c_longlong, i, vp]
    L.q4d_index_check_selftest.restype = i
    for fn in ("q4_gemv", "q4_gemv_ex", "q4_gemv_ex2", "q4kv_attn_decode", "q4kv_attn_decode_ex",
               "q4d_plan_gemv", "q4d_plan_attn", "q4d_device_error",
               "q4kv_attn_decode_noalloc"):
        getattr(L, fn).restype = i
    _lib = L
    return L


def _check(status: int, what: str):
    if status != 0:
        raise Q4DecError(status, what)


def plan_gemv(M: int, N: int, K: int, num_sms: int) -> GemvPlan:
    p = GemvPlan()
    _check(lib().q4d_plan_gemv(M, N, K, num_sms, ctypes.byref(p)), "q4d_plan_gemv")
    return p


def plan_attn(ctx_len: int, n_q_heads: int, n_kv_heads: int, head_dim: int, M: int,
              num_sms: int, q8: bool = False) -> AttnPlan:
    """Launch plan of the attention over the Q4_0 cache (``q8``: the Q8_0 cache)."""
    p = AttnPlan()
    fn = "q8kv_plan_attn" if q8 else "q4d_plan_attn"
    _check(getattr(lib(), fn)(ctx_len, n_q_heads, n_kv_heads, head_dim, M, num_sms,
                              ctypes.byref(p)), fn)
    return p


def _host_convert(fn: str, src, rows: int, K: int, out_bytes: int, what: str):
    import numpy as np

    a = np.ascontiguousarray(src, dtype=np.uint8).reshape(-1)
    out = np.empty(out_bytes, dtype=np.uint8)
    if a.size < (rows * K // 32 * 18 if "unpack" not in fn else rows * K // 256 * 144):
        raise ValueError(f"{what}: input buffer too small")
    _check(getattr(lib(), fn)(a.ctypes.data, out.ctypes.data, rows, K), fn)
    return out


def pack_q4_0_weights(blocks18, N: int, K: int):
    """Canonical 18-byte Q4_0 blocks, row-major [N][K/32] (host bytes) -> the
    library's weight layout (host bytes, N*K/256*144)."""
    return _host_convert("q4d_pack_q4_0_weights", blocks18, N, K, N * K // 256 * 144, "blocks18")


def unpack_q4_0_weights(W_q4, N: int, K: int):
    """Inverse of :func:`pack_q4_0_weights`."""
    return _host_convert("q4d_unpack_q4_0_weights", W_q4, N, K, N * K // 32 * 18, "W_q4")


def pack_q4_0_rows(blocks18, rows: int, K: int):
    """Canonical 18-byte Q4_0 blocks [rows][K/32] -> super-blocks in row order
    (the K/V cache layout)."""
    return _host_convert("q4d_pack_q4_0_rows", blocks18, rows, K, rows * K // 256 * 144, "blocks18")


def unpack_q4_0_rows(rows_q4, rows: int, K: int):
    """Inverse of :func:`pack_q4_0_rows`."""
    return _host_convert("q4d_unpack_q4_0_rows", rows_q4, rows, K, rows * K // 32 * 18, "rows_q4")


def _torch():
    import torch

    return torch


def _dev_tensor(t, dtype, what):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t


def _stream_ptr(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes: int, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace smaller than the {nbytes} bytes needed")
        return workspace
    # zero-filled: the GEMV workspace's partial-slot entries must start at 0
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


GEMV_WEIGHT_PREFETCH = 1  # Q4D_GEMV_WEIGHT_PREFETCH
GEMV_OUT_BF16 = 2         # Q4D_GEMV_OUT_BF16
GEMV_SWIGLU = 4           # Q4D_GEMV_SWIGLU (batch jobs)


def _out_flags(out_dtype, torch):
    if out_dtype == torch.float32:
        return 0
    if out_dtype == torch.bfloat16:
        return GEMV_OUT_BF16
    raise ValueError("out_dtype must be torch.float32 or torch.bfloat16")


def q4_gemv(W, x, y=None, *, N: int, K: int, stream=None, workspace=None,
            weight_prefetch: bool = False, out_dtype=None):
    """y[M][N] = dequant(W)[N][K] @ x[M][K]^T via ``q4_gemv_ex2``.

    ``W``: uint8 CUDA tensor with N*K/256*144 bytes (super-block layout);
    ``x``: bf16 CUDA tensor [M][K]; ``y``: optional [M][N] output.
    ``out_dtype``: torch.float32 (default) or torch.bfloat16 (Q4D_GEMV_OUT_BF16:
    the fp32 result rounded to nearest even); taken from ``y`` when given.
    ``weight_prefetch``: Q4D_GEMV_WEIGHT_PREFETCH (programmatic dependent
    launch; W must not be written by earlier kernels still in flight).
    """
    torch = _torch()
    _dev_tensor(W, torch.uint8, "W")
    _dev_tensor(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError("x must be [M][K]")
    M = x.shape[0]
    if W.numel() != N * (K // 256) * 144:
        raise ValueError("W has the wrong number of bytes for N x K")
    if out_dtype is None:
        out_dtype = torch.float32 if y is None else y.dtype
    flags = _out_flags(out_dtype, torch) | (GEMV_WEIGHT_PREFETCH if weight_prefetch else 0)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _dev_tensor(y, out_dtype, "y")
    if tuple(y.shape) != (M, N):
        raise ValueError("y must be [M][N]")
    with torch.cuda.device(x.device):
        need = lib().q4d_gemv_workspace_bytes(M, N, K)
        ws = _workspace(need, x.device, workspace)
        st = lib().q4_gemv_ex2(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K,
                               _stream_ptr(stream), None if ws is None else ws.data_ptr(), need,
                               flags)
    _check(st, "q4_gemv")
    return y


def q4_gemv_swiglu(W_gu, x, h=None, *, N: int, K: int, stream=None, workspace=None,
                   weight_prefetch: bool = False, out_dtype=None):
    """h[M][N] = silu(gate) * up from one interleaved gate / up matrix
    ``W_gu`` (2N rows: gate n at row 2n, up n at 2n + 1) via ``q4_gemv_swiglu_ex``;
    ``out_dtype`` as for :func:`q4_gemv`."""
    torch = _torch()
    _dev_tensor(W_gu, torch.uint8, "W_gu")
    _dev_tensor(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError("x must be [M][K]")
    M = x.shape[0]
    if W_gu.numel() != 2 * N * (K // 256) * 144:
        raise ValueError("W_gu has the wrong number of bytes for 2N x K")
    if out_dtype is None:
        out_dtype = torch.float32 if h is None else h.dtype
    flags = _out_flags(out_dtype, torch) | (GEMV_WEIGHT_PREFETCH if weight_prefetch else 0)
    if h is None:
        h = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _dev_tensor(h, out_dtype, "h")
    if tuple(h.shape) != (M, N):
        raise ValueError("h must be [M][N]")
    with torch.cuda.device(x.device):
        need = lib().q4d_gemv_swiglu_workspace_bytes(M, N, K)
        ws = _workspace(need, x.device, workspace)
        st = lib().q4_gemv_swiglu_ex(W_gu.data_ptr(), x.data_ptr(), h.data_ptr(), M, N, K,
                                     _stream_ptr(stream), None if ws is None else ws.data_ptr(),
                                     need, flags)
    _check(st, "q4_gemv_swiglu")
    return h


def q4kv_append(Kq4, Vq4, k_new, v_new, *, pos: int, kv_stride_tokens: int, stream=None):
    """Quantise the fp32 K/V rows ``k_new`` / ``v_new`` [M][n_kv_heads][256] into
    the Q4_0 caches at token positions pos .. pos+M-1 (``q4kv_append``)."""
    torch = _torch()
    _dev_tensor(Kq4, torch.uint8, "Kq4")
    _dev_tensor(Vq4, torch.uint8, "Vq4")
    _dev_tensor(k_new, torch.float32, "k_new")
    _dev_tensor(v_new, torch.float32, "v_new")
    if k_new.dim() != 3 or k_new.shape[2] != 256 or tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("k_new / v_new must be [M][n_kv_heads][256]")
    M, n_kv = k_new.shape[0], k_new.shape[1]
    need = n_kv * kv_stride_tokens * 144
    if Kq4.numel() < need or Vq4.numel() < need:
        raise ValueError("caches are smaller than n_kv_heads * kv_stride_tokens rows")
    with torch.cuda.device(k_new.device):
        st = lib().q4kv_append(Kq4.data_ptr(), Vq4.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                               n_kv, kv_stride_tokens, pos, M, _stream_ptr(stream))
    _check(st, "q4kv_append")


def q4kv_attn_decode(Q, Kq4, Vq4, out=None, *, ctx_len: int, n_kv_heads: int,
                     head_dim: int = 256, kv_stride_tokens: int | None = None,
                     softmax_scale: float = 1.0, stream=None, workspace=None):
    """Causal GQA decode attention over Q4_0 K/V via ``q4kv_attn_decode_ex``.

    ``Q``: bf16 [M][n_q_heads][head_dim]; ``Kq4``/``Vq4``: uint8 caches of
    ``n_kv_heads * kv_stride_tokens`` super-blocks; returns fp32 ``out`` of
    Q's shape.
    """
    return _attn(Q, Kq4, Vq4, out, ctx_len, n_kv_heads, head_dim, kv_stride_tokens,
                 softmax_scale, stream, workspace, q8=False)


def q8kv_attn_decode(Q, Kq8, Vq8, out=None, *, ctx_len: int, n_kv_heads: int,
                     head_dim: int = 256, kv_stride_tokens: int | None = None,
                     softmax_scale: float = 1.0, stream=None, workspace=None):
    """The same attention over Q8_0 K/V caches (272-byte super-blocks) via
    ``q8kv_attn_decode_ex``."""
    return _attn(Q, Kq8, Vq8, out, ctx_len, n_kv_heads, head_dim, kv_stride_tokens,
                 softmax_scale, stream, workspace, q8=True)


def _attn(Q, Kc, Vc, out, ctx_len, n_kv_heads, head_dim, kv_stride_tokens, softmax_scale,
          stream, workspace, q8):
    torch = _torch()
    _dev_tensor(Q, torch.bfloat16, "Q")
    _dev_tensor(Kc, torch.uint8, "K cache")
    _dev_tensor(Vc, torch.uint8, "V cache")
    if Q.dim() != 3 or Q.shape[2] != head_dim:
        raise ValueError("Q must be [M][n_q_heads][head_dim]")
    M, n_q = Q.shape[0], Q.shape[1]
    stride = ctx_len if kv_stride_tokens is None else kv_stride_tokens
    need_bytes = n_kv_heads * stride * (head_dim // 256) * (272 if q8 else 144)
    if Kc.numel() < need_bytes or Vc.numel() < need_bytes:
        raise ValueError("K/V caches are smaller than n_kv_heads * kv_stride_tokens rows")
    if out is None:
        out = torch.empty((M, n_q, head_dim), dtype=torch.float32, device=Q.device)
    _dev_tensor(out, torch.float32, "out")
    if tuple(out.shape) != (M, n_q, head_dim):
        raise ValueError("out must match Q's shape")
    name = "q8kv_attn_decode_ex" if q8 else "q4kv_attn_decode_ex"
    with torch.cuda.device(Q.device):
        wsfn = lib().q8kv_attn_workspace_bytes if q8 else lib().q4d_attn_workspace_bytes
        need = wsfn(ctx_len, n_q, n_kv_heads, head_dim, M)
        ws = _workspace(need, Q.device, workspace)
        st = getattr(lib(), name)(Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), out.data_ptr(),
                                  ctx_len, n_q, n_kv_heads, head_dim, M, stride,
                                  float(softmax_scale), _stream_ptr(stream),
                                  None if ws is None else ws.data_ptr(), need)
    _check(st, name)
    return out


class GemvBatch:
    """Many GEMVs in one launch (``q4d_gemv_batch_prepare`` + ``q4_gemv_batch_ex``).

    ``jobs``: list of dicts with keys ``W`` (uint8 weights), ``x`` (bf16
    [M][K]), ``y`` (fp32 or bf16 output [M][N]), ``N``, ``K`` and optional
    ``swiglu`` (W holds 2N interleaved gate / up rows, y = h [M][N]) and
    ``wait_for`` (-1, or the index of the job whose output must be written
    before this job reads x; only that job is waited for, so jobs depending on
    several earlier ones, or overwriting memory an earlier job reads, need a
    chain of waits).  All tensors must stay alive and in place for as long as
    the batch is used.  The descriptor is prepared and copied to the device
    once; :meth:`run` only launches.  The workspace is allocated zero-filled,
    and every successful launch leaves it so (if a launch reports a device
    error, zero it again before the next)."""

    def __init__(self, jobs, *, device=None):
        torch = _torch()
        if not jobs:
            raise ValueError("a batch needs at least one job")
        M = None
        arr = (GemvJob * len(jobs))()
        self._keep = []
        for i, j in enumerate(jobs):
            W, x, y, N, K = j["W"], j["x"], j["y"], int(j["N"]), int(j["K"])
            swiglu = bool(j.get("swiglu", False))
            _dev_tensor(W, torch.uint8, f"jobs[{i}].W")
            _dev_tensor(x, torch.bfloat16, f"jobs[{i}].x")
            if x.dim() != 2 or x.shape[1] != K:
                raise ValueError(f"jobs[{i}].x must be [M][K]")
            if M is None:
                M = x.shape[0]
            if x.shape[0] != M:
                raise ValueError("every job of a batch has the same M")
            rows = 2 * N if swiglu else N
            if W.numel() != rows * (K // 256) * 144:
                raise ValueError(f"jobs[{i}].W has the wrong number of bytes")
            _dev_tensor(y, y.dtype, f"jobs[{i}].y")
            flags = _out_flags(y.dtype, torch) | (GEMV_SWIGLU if swiglu else 0)
            if tuple(y.shape) != (M, N):
                raise ValueError(f"jobs[{i}].y must be [M][N]")
            arr[i] = GemvJob(W.data_ptr(), x.data_ptr(), y.data_ptr(), N, K, flags,
                             int(j.get("wait_for", -1)))
            self._keep += [W, x, y]
        self.device = x.device if device is None else device
        self.M, self.n_jobs = M, len(jobs)
        L = lib()
        with torch.cuda.device(self.device):
            sms = torch.cuda.get_device_properties(self.device).multi_processor_count
            nbytes = L.q4d_gemv_batch_desc_bytes(len(jobs))
            self.desc_host = torch.zeros(nbytes, dtype=torch.uint8)
            ws = ctypes.c_size_t(0)
            _check(L.q4d_gemv_batch_prepare(arr, len(jobs), M, sms, self.desc_host.data_ptr(),
                                            nbytes, ctypes.byref(ws)), "q4d_gemv_batch_prepare")
            self.desc_dev = self.desc_host.to(self.device)
            self.workspace_bytes = ws.value
            self.workspace = torch.zeros(max(16, ws.value), dtype=torch.uint8, device=self.device)

    def run(self, stream=None, weight_prefetch: bool = False):
        torch = _torch()
        with torch.cuda.device(self.device):
            st = lib().q4_gemv_batch_ex(self.desc_host.data_ptr(), self.desc_dev.data_ptr(),
                                        _stream_ptr(stream), self.workspace.data_ptr(),
                                        self.workspace.numel(),
                                        GEMV_WEIGHT_PREFETCH if weight_prefetch else 0)
        _check(st, "q4_gemv_batch_ex")


NOALLOC_SCRATCH_BYTES = 16 << 20


def q4kv_attn_decode_noalloc(Q, Kq4, Vq4, out, *, ctx_len: int, n_kv_heads: int,
                             head_dim: int = 256, kv_stride_tokens: int | None = None,
                             softmax_scale: float = 1.0, stream=None):
    """Decode attention through ``q4kv_attn_decode_noalloc``: for callers that
    may not allocate device memory while running.  Neither this wrapper nor the
    library allocates; ``out`` (fp32, Q's shape) must be given.  The library's
    16 MiB static scratch is shared by all such calls, so calls that overlap on
    the GPU race."""
    torch = _torch()
    _dev_tensor(Q, torch.bfloat16, "Q")
    _dev_tensor(Kq4, torch.uint8, "Kq4")
    _dev_tensor(Vq4, torch.uint8, "Vq4")
    _dev_tensor(out, torch.float32, "out")
    if Q.dim() != 3 or Q.shape[2] != head_dim or tuple(out.shape) != tuple(Q.shape):
        raise ValueError("Q must be [M][n_q_heads][head_dim] and out must match it")
    M, n_q = Q.shape[0], Q.shape[1]
    stride = ctx_len if kv_stride_tokens is None else kv_stride_tokens
    need_bytes = n_kv_heads * stride * (head_dim // 256) * 144
    if Kq4.numel() < need_bytes or Vq4.numel() < need_bytes:
        raise ValueError("K/V caches are smaller than n_kv_heads * kv_stride_tokens rows")
    with torch.cuda.device(Q.device):
        st = lib().q4kv_attn_decode_noalloc(Q.data_ptr(), Kq4.data_ptr(), Vq4.data_ptr(),
                                            out.data_ptr(), ctx_len, n_q, n_kv_heads, head_dim,
                                            M, stride, float(softmax_scale), _stream_ptr(stream))
    _check(st, "q4kv_attn_decode_noalloc")
    return out


def device_error(reset: bool = False) -> int:
    """Synchronise and read the device error word: 0 when clear, else the
    status it stands for (6: a bounded wait ran out, 7: an index check of the
    debug build failed)."""
    return lib().q4d_device_error(1 if reset else 0)


def device_error_record(reset: bool = False):
    """Synchronise and read the device error record: (status, bits, site,
    index) -- site and index of the first failed index check of a debug
    build (0, 0 when none failed)."""
    rec = (ctypes.c_uint * 4)()
    st = lib().q4d_device_error_record(rec, 1 if reset else 0)
    if st not in (0, 6, 7):
        _check(st, "q4d_device_error_record")
    index = rec[2] | (rec[3] << 32)
    return st, rec[0], rec[1], index - (1 << 64) if index >= 1 << 63 else index


def debug_build() -> bool:
    """Whether the loaded library is the debug (index-checked) build."""
    return lib().q4d_debug_build() == 1


def debug_limit_weights(nbytes: int) -> None:
    """Debug build only: declare the weight extent of GEMVs launched or
    batches prepared from now on as min(true extent, nbytes) (0: true)."""
    _check(lib().q4d_debug_limit_weights(int(nbytes)), "q4d_debug_limit_weights")
