"""fp64 CPU oracle for k-MIP attention (ctypes loader for ``kmip_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or runs anything in this directory, and this directory
imports nothing from the CUDA package.

What it computes is stated in ``kmip_oracle.c`` (k-Maximum Inner Product
Attention for Graph Transformers and the Expressive Power of GraphGPS,
Abstract: top-k selection by inner product, then attention over the kept
keys).  Every array is widened to fp64 before the call; bf16 and fp32 values
widen exactly, so the oracle sees the same numbers the GPU does.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kmip_oracle.c")
_LIB = os.path.join(_HERE, "libkmip_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: fp64 in program order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64, I32, F64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.kmip_oracle_fwd.argtypes = [P, P, P, P, I64, I64, I32, I32, I32, F64,
                                        P, P, P, P, P, I32]
        lib.kmip_oracle_fwd.restype = I32
        lib.kmip_oracle_fwd_pairs.argtypes = [P, P, P, P, I64, I64, I32, I32, I32, F64,
                                              P, P, I64, P, P, P, P, P, I32]
        lib.kmip_oracle_fwd_pairs.restype = I32
        lib.kmip_oracle_given_idx.argtypes = [P, P, P, P, P, P, I64, I64, I32, I32, I32,
                                              F64, P, P, P, P, P]
        lib.kmip_oracle_given_idx.restype = I32
        lib.kmip_oracle_full.argtypes = [P, P, P, P, I64, I64, I32, I32, F64, P, P, I64, P, P,
                                         I32]
        lib.kmip_oracle_full.restype = I32
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (any dtype): widen exactly on the CPU
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _offsets(offsets, N: int) -> np.ndarray:
    if offsets is None:
        return np.array([0, N], dtype=np.int64)
    if hasattr(offsets, "detach"):
        offsets = offsets.detach().cpu().numpy()
    return np.ascontiguousarray(offsets, dtype=np.int64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return os.cpu_count() or 1


def fwd(Q, K, V, offsets, k: int, scale: float, nthreads: int | None = None):
    """Forward for every (query, head).

    Q, K, V: [N, H, d].  offsets: G+1 node offsets (None = one graph).
    Returns dict(out [N,H,d] f64, idx [N,H,k] i32, lse [N,H], gap [N,H],
    kth [N,H]): gap = s_(k) - s_(k+1) (inf when the graph has <= k nodes),
    kth = s_(k_eff), both on unscaled scores.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    N, H, d = Q.shape
    off = _offsets(offsets, N)
    out = np.zeros((N, H, d)); idx = np.full((N, H, k), -1, dtype=np.int32)
    lse = np.zeros((N, H)); gap = np.zeros((N, H)); kth = np.zeros((N, H))
    rc = _load().kmip_oracle_fwd(_p(Q), _p(K), _p(V), _p(off), len(off) - 1, N, H, d, k,
                                 float(scale), _p(out), _p(idx), _p(lse), _p(gap), _p(kth),
                                 nthreads or default_threads())
    if rc:
        raise ValueError(f"kmip_oracle_fwd failed with code {rc}")
    return dict(out=out, idx=idx, lse=lse, gap=gap, kth=kth)


def fwd_pairs(Q, K, V, offsets, k: int, scale: float, pairs_q, pairs_h,
              nthreads: int | None = None):
    """Forward for a list of (query, head) pairs; row t of each output is pair t."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    N, H, d = Q.shape
    off = _offsets(offsets, N)
    pq = np.ascontiguousarray(pairs_q, dtype=np.int64)
    ph = np.ascontiguousarray(pairs_h, dtype=np.int32)
    n = len(pq)
    out = np.zeros((n, d)); idx = np.full((n, k), -1, dtype=np.int32)
    lse = np.zeros(n); gap = np.zeros(n); kth = np.zeros(n)
    rc = _load().kmip_oracle_fwd_pairs(_p(Q), _p(K), _p(V), _p(off), len(off) - 1, N, H, d, k,
                                       float(scale), _p(pq), _p(ph), n, _p(out), _p(idx),
                                       _p(lse), _p(gap), _p(kth), nthreads or default_threads())
    if rc:
        raise ValueError(f"kmip_oracle_fwd_pairs failed with code {rc}")
    return dict(out=out, idx=idx, lse=lse, gap=gap, kth=kth)


def given_idx(Q, K, V, idx, offsets, scale: float, dO=None):
    """Attention (and, with dO, its backward) over the given selected sets.

    idx: [N, H, k] int32, -1 = padding.  Returns dict(out, lse) and, with dO,
    also dQ, dK, dV (all fp64).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    N, H, d = Q.shape
    if hasattr(idx, "detach"):
        idx = idx.detach().cpu().numpy()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    k = idx.shape[-1]
    off = _offsets(offsets, N)
    out = np.zeros((N, H, d)); lse = np.zeros((N, H))
    res = dict(out=out, lse=lse)
    if dO is not None:
        dO = _f64(dO)
        dQ = np.zeros((N, H, d)); dK = np.zeros((N, H, d)); dV = np.zeros((N, H, d))
        res.update(dQ=dQ, dK=dK, dV=dV)
        args = (_p(dO), _p(idx), _p(off), len(off) - 1, N, H, d, k, float(scale),
                _p(out), _p(lse), _p(dQ), _p(dK), _p(dV))
    else:
        args = (None, _p(idx), _p(off), len(off) - 1, N, H, d, k, float(scale),
                _p(out), _p(lse), None, None, None)
    rc = _load().kmip_oracle_given_idx(_p(Q), _p(K), _p(V), *args)
    if rc:
        raise ValueError(f"kmip_oracle_given_idx failed with code {rc}")
    return res


def full_attention(Q, K, V, offsets, scale: float, pairs_q=None, pairs_h=None,
                   nthreads: int | None = None):
    """Full softmax attention over every key of each query's graph (the
    comparison of Figure 8).  Returns dict(out, lse): [N, H, d] / [N, H] for
    every pair, or [n, d] / [n] for the listed pairs."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    N, H, d = Q.shape
    off = _offsets(offsets, N)
    if pairs_q is None:
        out = np.zeros((N, H, d)); lse = np.zeros((N, H)); pq = ph = None; n = 0
    else:
        pq = np.ascontiguousarray(pairs_q, dtype=np.int64)
        ph = np.ascontiguousarray(pairs_h, dtype=np.int32)
        n = len(pq)
        out = np.zeros((n, d)); lse = np.zeros(n)
    rc = _load().kmip_oracle_full(_p(Q), _p(K), _p(V), _p(off), len(off) - 1, N, H, d,
                                  float(scale), None if pq is None else _p(pq),
                                  None if ph is None else _p(ph), n, _p(out), _p(lse),
                                  nthreads or default_threads())
    if rc:
        raise ValueError(f"kmip_oracle_full failed with code {rc}")
    return dict(out=out, lse=lse)


def decided(gap: np.ndarray, kth: np.ndarray, rel: float = 1e-3) -> np.ndarray:
    """A (query, head) is decided when its k-th/(k+1)-th score gap exceeds
    rel * |s_(k)|; only decided selections are unique enough to compare."""
    return gap > rel * np.abs(kth)
