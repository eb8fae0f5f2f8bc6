"""Thin ctypes binding of libkmip (the C ABI declared in include/kmip.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libkmip.so.  torch provides device memory and streams.  There is
no CPU fallback -- if the library is missing, or the tensors are not on a
CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# KMIP_DEBUG_BOUNDS=1 loads the build with device-side index checks
# (python -m graph_transformer_sparse_kmip_b200.build --debug-bounds).
LIB_PATH = os.path.join(_PKG, "libkmip_debug.so" if os.environ.get("KMIP_DEBUG_BOUNDS") == "1"
                        else "libkmip.so")
# KMIP_NVTX=1 wraps every library call in an NVTX range (for nsys/ncu timelines).
_NVTX = os.environ.get("KMIP_NVTX") == "1"

KMIP_BF16, KMIP_F32 = 0, 1
STATUS_NAMES = {0: "KMIP_OK", 1: "KMIP_ERR_INVALID_ARG", 2: "KMIP_ERR_UNSUPPORTED",
                3: "KMIP_ERR_CUDA", 4: "KMIP_ERR_BAD_OFFSETS", 5: "KMIP_ERR_TIMEOUT",
                6: "KMIP_ERR_BAD_INDEX", 7: "KMIP_ERR_SCRATCH_LIMIT"}
EXPORTED = ("kmip_attn_fwd", "kmip_attn_fwd_noalloc", "kmip_attn_fwd_diag", "kmip_attn_bwd",
            "kmip_attn_bwd_deterministic", "kmip_attn_gather", "kmip_get_status",
            "kmip_scratch_usage", "kmip_scratch_trim", "kmip_error_string",
            "kmip_fwd_path", "kmip_version")

_lib = None


class KmipError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


def load() -> ctypes.CDLL:
    """Load libkmip.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkmip.so not found at {LIB_PATH}; build it with "
                          "`python -m graph_transformer_sparse_kmip_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.kmip_attn_fwd.argtypes = [P, P, P, P, I64, I32, I32, I32, F32, P, P, P, P, I32, I32]
    lib.kmip_attn_fwd.restype = I32
    lib.kmip_attn_fwd_noalloc.argtypes = lib.kmip_attn_fwd.argtypes
    lib.kmip_attn_fwd_noalloc.restype = I32
    lib.kmip_attn_fwd_diag.argtypes = [P, P, P, P, I64, I32, I32, I32, F32, P, P, P, P, P, I32,
                                       I32]
    lib.kmip_attn_fwd_diag.restype = I32
    lib.kmip_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I64, I32, I32, I32, F32, I32]
    lib.kmip_attn_bwd.restype = I32
    lib.kmip_attn_bwd_deterministic.argtypes = lib.kmip_attn_bwd.argtypes
    lib.kmip_attn_bwd_deterministic.restype = I32
    lib.kmip_attn_gather.argtypes = [P, P, P, P, I64, I32, I32, I32, F32, P, P, P, I32]
    lib.kmip_attn_gather.restype = I32
    lib.kmip_get_status.argtypes = [P]
    lib.kmip_get_status.restype = I32
    lib.kmip_scratch_usage.argtypes = [P, P, I32]
    lib.kmip_scratch_usage.restype = I32
    lib.kmip_scratch_trim.argtypes = []
    lib.kmip_scratch_trim.restype = I32
    lib.kmip_error_string.argtypes = [I32]
    lib.kmip_error_string.restype = ctypes.c_char_p
    lib.kmip_test_wait_timeout.argtypes = [P, I32]
    lib.kmip_test_wait_timeout.restype = I32
    lib.kmip_fwd_path.argtypes = [I32, I32, I32]
    lib.kmip_fwd_path.restype = I32
    lib.kmip_version.argtypes = []
    lib.kmip_version.restype = I32
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(name, *args):
    """Calls the C entry point `name` (inside an NVTX range when KMIP_NVTX=1)."""
    fn = getattr(load(), name)
    if not _NVTX:
        return fn(*args)
    torch.cuda.nvtx.range_push(name)
    try:
        return fn(*args)
    finally:
        torch.cuda.nvtx.range_pop()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return KMIP_BF16
    if t == torch.float32:
        return KMIP_F32
    raise TypeError(f"unsupported dtype {t} (bf16 or fp32)")


def _check_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libkmip takes contiguous CUDA tensors")


# --- the C entry points, same names, torch tensors in place of pointers ---

def kmip_attn_fwd(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, stream=None,
                  num_graphs=None, dtype=None) -> int:
    _check_cuda(Q, K, V, graph_offsets, out, idx, lse)
    G = (graph_offsets.numel() - 1) if graph_offsets is not None else 1
    if num_graphs is None:
        num_graphs = G
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call("kmip_attn_fwd", _ptr(Q), _ptr(K), _ptr(V), _ptr(graph_offsets), int(N), int(H),
                                int(d), int(k), float(scale), _ptr(out), _ptr(idx), _ptr(lse),
                                _stream(stream), int(num_graphs), int(dtype))


def kmip_attn_fwd_noalloc(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse,
                          stream=None, num_graphs=None, dtype=None) -> int:
    """kmip_attn_fwd without any device allocation inside the library: the
    work list lives in a fixed device array of the library (for callers whose
    memory is fully owned by their own pool, or who must not allocate after
    start-up).  Calls on one device must not overlap on the GPU."""
    _check_cuda(Q, K, V, graph_offsets, out, idx, lse)
    G = (graph_offsets.numel() - 1) if graph_offsets is not None else 1
    if num_graphs is None:
        num_graphs = G
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call("kmip_attn_fwd_noalloc", _ptr(Q), _ptr(K), _ptr(V), _ptr(graph_offsets), int(N),
                                        int(H), int(d), int(k), float(scale), _ptr(out),
                                        _ptr(idx), _ptr(lse), _stream(stream), int(num_graphs),
                                        int(dtype))


def kmip_attn_fwd_diag(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, lse_all,
                       stream=None, num_graphs=None, dtype=None) -> int:
    """kmip_attn_fwd plus lse_all [N, H]: the log-sum-exp over every key of
    the query's graph (the normaliser of full softmax attention)."""
    _check_cuda(Q, K, V, graph_offsets, out, idx, lse, lse_all)
    G = (graph_offsets.numel() - 1) if graph_offsets is not None else 1
    if num_graphs is None:
        num_graphs = G
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call("kmip_attn_fwd_diag", _ptr(Q), _ptr(K), _ptr(V), _ptr(graph_offsets), int(N),
                                     int(H), int(d), int(k), float(scale), _ptr(out), _ptr(idx),
                                     _ptr(lse), _ptr(lse_all), _stream(stream), int(num_graphs),
                                     int(dtype))


def kmip_attn_bwd(dOut, Q, K, V, idx, lse, dQ, dK, dV, stream=None, N=None, H=None, d=None,
                  k=None, scale=None, dtype=None) -> int:
    _check_cuda(dOut, Q, K, V, idx, lse, dQ, dK, dV)
    N_, H_, d_ = Q.shape
    N = N_ if N is None else N
    H = H_ if H is None else H
    d = d_ if d is None else d
    k = idx.shape[-1] if k is None else k
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call("kmip_attn_bwd", _ptr(dOut), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(lse),
                                _ptr(dQ), _ptr(dK), _ptr(dV), _stream(stream), int(N), int(H),
                                int(d), int(k), float(scale), int(dtype))


def kmip_attn_bwd_deterministic(dOut, Q, K, V, idx, lse, dQ, dK, dV, stream=None, N=None,
                                H=None, d=None, k=None, scale=None, dtype=None) -> int:
    """kmip_attn_bwd with bitwise reproducible dK/dV (sorted gather, no
    atomics)."""
    _check_cuda(dOut, Q, K, V, idx, lse, dQ, dK, dV)
    N_, H_, d_ = Q.shape
    N = N_ if N is None else N
    H = H_ if H is None else H
    d = d_ if d is None else d
    k = idx.shape[-1] if k is None else k
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call(
        "kmip_attn_bwd_deterministic", _ptr(dOut), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(lse), _ptr(dQ), _ptr(dK),
        _ptr(dV), _stream(stream), int(N), int(H), int(d), int(k), float(scale), int(dtype))


def kmip_attn_gather(Q, K, V, idx, N, H, d, k, scale, out, lse, stream=None, dtype=None) -> int:
    """Softmax and V gather over the given key sets (idx), scores recomputed."""
    _check_cuda(Q, K, V, idx, out, lse)
    if dtype is None:
        dtype = dtype_code(Q.dtype)
    return _call("kmip_attn_gather", _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), int(N), int(H),
                 int(d), int(k), float(scale), _ptr(out), _ptr(lse), _stream(stream), int(dtype))


def attn_gather(Q, K, V, idx, scale: float, stream=None):
    """Returns (out, lse) of attention over the given sets idx [N, H, k]."""
    N, H, d = Q.shape
    out = torch.empty_like(Q)
    lse = torch.empty((N, H), dtype=torch.float32, device=Q.device)
    rc = kmip_attn_gather(Q, K, V, idx, N, H, d, idx.shape[-1], scale, out, lse, stream)
    if rc:
        raise KmipError(rc, "kmip_attn_gather")
    return out, lse


def kmip_get_status(stream=None) -> int:
    return load().kmip_get_status(_stream(stream))


def kmip_error_string(code: int) -> str:
    return load().kmip_error_string(int(code)).decode()


def kmip_scratch_usage(reset_high: bool = False):
    """(reserved, used_high) bytes of the library's scratch pool on the
    current device."""
    r, h = ctypes.c_uint64(0), ctypes.c_uint64(0)
    rc = load().kmip_scratch_usage(ctypes.byref(r), ctypes.byref(h), int(bool(reset_high)))
    if rc:
        raise KmipError(rc, "kmip_scratch_usage")
    return int(r.value), int(h.value)


def kmip_scratch_trim():
    """Return the library's unused pool memory on the current device (after
    the streams that used the library have been synchronised)."""
    rc = load().kmip_scratch_trim()
    if rc:
        raise KmipError(rc, "kmip_scratch_trim")


def kmip_version() -> int:
    return load().kmip_version()


def kmip_fwd_path(d: int, k: int, dtype: int = KMIP_BF16) -> int:
    """1 = tcgen05 tensor-core forward, 0 = fp32-FMA forward, -1 = unsupported."""
    return load().kmip_fwd_path(int(d), int(k), int(dtype))


def kmip_test_wait_timeout(timeout_us: int, stream=None) -> int:
    """Test hook (include/kmip_testing.h): a bounded wait that must run out."""
    return load().kmip_test_wait_timeout(_stream(stream), int(timeout_us))


# --- convenience wrappers that allocate the outputs with torch ---

def attn_fwd(Q, K, V, k: int, scale: float, graph_offsets=None, stream=None):
    """Returns (out [N,H,d] like Q, idx [N,H,k] int32, lse [N,H] fp32)."""
    N, H, d = Q.shape
    out = torch.empty_like(Q)
    idx = torch.empty((N, H, k), dtype=torch.int32, device=Q.device)
    lse = torch.empty((N, H), dtype=torch.float32, device=Q.device)
    rc = kmip_attn_fwd(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, stream)
    if rc:
        raise KmipError(rc, "kmip_attn_fwd")
    return out, idx, lse


def attn_fwd_diag(Q, K, V, k: int, scale: float, graph_offsets=None, stream=None):
    """Returns (out, idx, lse, lse_all): kmip_attn_fwd's outputs and the
    log-sum-exp over every key of the query's graph."""
    N, H, d = Q.shape
    out = torch.empty_like(Q)
    idx = torch.empty((N, H, k), dtype=torch.int32, device=Q.device)
    lse = torch.empty((N, H), dtype=torch.float32, device=Q.device)
    lse_all = torch.empty((N, H), dtype=torch.float32, device=Q.device)
    rc = kmip_attn_fwd_diag(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, lse_all,
                            stream)
    if rc:
        raise KmipError(rc, "kmip_attn_fwd_diag")
    return out, idx, lse, lse_all


def attn_bwd(dOut, Q, K, V, idx, lse, scale: float, stream=None, deterministic=False):
    """Returns (dQ, dK, dV), fp32 [N,H,d]."""
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    dK = torch.empty_like(dQ)
    dV = torch.empty_like(dQ)
    fn = kmip_attn_bwd_deterministic if deterministic else kmip_attn_bwd
    rc = fn(dOut, Q, K, V, idx, lse, dQ, dK, dV, stream, scale=scale)
    if rc:
        raise KmipError(rc, fn.__name__)
    return dQ, dK, dV


def check_status(stream=None):
    rc = kmip_get_status(stream)
    if rc:
        raise KmipError(rc, "device status")
