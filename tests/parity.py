"""Comparison rules between the CUDA path and the fp64 oracle.

Selection (k-Maximum Inner Product Attention for Graph Transformers ...,
Abstract: the k keys of largest inner product).  For every (query, head)
whose oracle gap s_(k) - s_(k+1) exceeds 1e-3 |s_(k)| ("decided") the kept
key set must equal the oracle's.  For the other pairs several sets are
correct, because scores nearly tie; a set is accepted when it is a top-k up
to that margin: every kept key scores at least s_(k) - margin, and every
in-graph key left out scores at most s_(k) + margin.  Both halves are needed:
the first alone would accept a set that drops the best key.  Every row must
also hold k_eff distinct keys of the query's own graph, padded with -1, in
non-increasing score order (up to fp32 rounding).

Values.  ``north_star`` bounds the "max relative error" by 2e-2 for bf16
inputs and 1e-4 for fp32 inputs.  Three figures are computed per tensor:
  * normwise   max|gpu - ref| / max|ref| over the whole tensor;
  * per row    for every (node, head) row of out, dQ, dK, dV:
               max_c |gpu - ref| / max(max_c |ref|, f max|ref|), the floor
               keeping rows that are zero or nearly zero from dividing by ~0
               (f = 1e-3 for bf16 inputs, 1e-2 for fp32 inputs: see
               ROW_FLOOR);
  * elementwise |gpu - ref| / max(|ref|, 1e-3 max|ref|) (reported only).
The normwise and per-row figures must both be within the tolerance.  lse is
a logarithm, so its absolute error is the relative error of the softmax
normaliser exp(lse); it is checked element by element as
|gpu - ref| / max(|ref|, 1).  ref is the oracle's attention over the
GPU-selected sets (and, on decided pairs, the oracle's own result).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
GAP_REL = 1e-3
# Floor of the per-row check, relative to the tensor's largest entry.  fp32
# results are held to 1e-4 per row only for rows at least 1% of the largest:
# below that, fp32 rounding of the kept-key sums and of dS = p (dP - D),
# which cancels, is already a visible fraction of such a small row.
ROW_FLOOR = {torch.bfloat16: 1e-3, torch.float32: 1e-2}


def _np(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def normwise(gpu, ref) -> float:
    gpu, ref = _np(gpu), _np(ref)
    if ref.size == 0:
        return 0.0
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0))


def rowwise(gpu, ref, floor_rel: float = 1e-3) -> float:
    """Largest per-row relative error over the last axis (rows = (node, head))."""
    gpu, ref = _np(gpu), _np(ref)
    if ref.size == 0:
        return 0.0
    top = np.abs(ref).max()
    floor = floor_rel * top if top > 0 else 1.0
    err = np.abs(gpu - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), floor)
    return float((err / den).max())


def elementwise(gpu, ref, floor_rel: float = 1e-3) -> float:
    gpu, ref = _np(gpu), _np(ref)
    if ref.size == 0:
        return 0.0
    top = np.abs(ref).max()
    floor = floor_rel * top if top > 0 else 1.0
    return float((np.abs(gpu - ref) / np.maximum(np.abs(ref), floor)).max())


def lse_error(gpu, ref) -> float:
    gpu, ref = _np(gpu), _np(ref)
    if ref.size == 0:
        return 0.0
    return float((np.abs(gpu - ref) / np.maximum(np.abs(ref), 1.0)).max())


def _graph_of(off: np.ndarray, i: int) -> int:
    g = int(np.searchsorted(off, i, side="right")) - 1
    while g + 1 < len(off) - 1 and off[g + 1] <= i:
        g += 1
    return g


def score_slack(q: np.ndarray, Kg: np.ndarray) -> float:
    """Slack for comparing scores the GPU accumulated in fp32 with fp64 ones:
    one fp32 sum of d exact products is within about d 2^-24 sum_c |q_c k_c|
    of the exact value (twice that if the accumulator truncates); a
    difference of two such scores within twice that again; the bound below
    doubles it once more."""
    d = q.shape[-1]
    return 8.0 * d * 2.0 ** -24 * float((np.abs(Kg) @ np.abs(q)).max(initial=0.0)) + 1e-30


def check_selection(Q, K, offsets, idx_gpu, ref, pairs_q=None, pairs_h=None):
    """ref: oracle fwd result (full, or for the listed pairs).  Returns the
    number of decided and undecided pairs; raises AssertionError on a
    mismatch."""
    Qd, Kd = _np(Q), _np(K)
    off = (offsets.detach().cpu().numpy() if hasattr(offsets, "detach") else
           np.asarray(offsets)) if offsets is not None else np.array([0, Qd.shape[0]])
    off = off.astype(np.int64)
    gi = idx_gpu.detach().cpu().numpy() if hasattr(idx_gpu, "detach") else np.asarray(idx_gpu)
    if pairs_q is None:
        N, H = Qd.shape[:2]
        pq = np.repeat(np.arange(N), H)
        ph = np.tile(np.arange(H), N)
        ref_idx = ref["idx"].reshape(N * H, -1)
        gap, kth = ref["gap"].reshape(-1), ref["kth"].reshape(-1)
    else:
        pq, ph = np.asarray(pairs_q), np.asarray(pairs_h)
        ref_idx, gap, kth = ref["idx"], ref["gap"], ref["kth"]
    got = gi[pq, ph]
    dec = oracle.decided(gap, kth, GAP_REL)
    k = got.shape[1]
    n_und = 0
    for t in range(len(pq)):
        i, h = int(pq[t]), int(ph[t])
        g = _graph_of(off, i)
        j0, j1 = int(off[g]), int(off[g + 1])
        keff = min(k, j1 - j0)
        a, b = got[t], ref_idx[t]
        assert (a[keff:] == -1).all(), f"pair {(i, h)}: padding {a}"
        assert (a[:keff] >= j0).all() and (a[:keff] < j1).all(), \
            f"pair {(i, h)}: key outside graph {a}"
        assert len(set(a[:keff].tolist())) == keff, f"pair {(i, h)}: repeated key {a}"
        q = Qd[i, h]
        s_sel = Kd[a[:keff], h] @ q
        eps = score_slack(q, Kd[a[:keff], h])
        assert (np.diff(s_sel) <= eps).all(), f"pair {(i, h)}: idx not in score order"
        if dec[t]:
            assert set(a[:keff].tolist()) == set(b[:keff].tolist()), \
                f"pair {(i, h)}: gpu {sorted(a[:keff])} oracle {sorted(b[:keff])}"
        else:
            n_und += 1
            s_all = Kd[j0:j1, h] @ q
            margin = GAP_REL * abs(kth[t]) + score_slack(q, Kd[j0:j1, h])
            assert s_sel.min() >= kth[t] - margin, f"pair {(i, h)}: kept key below s_(k)"
            left = np.ones(j1 - j0, dtype=bool)
            left[a[:keff] - j0] = False
            if left.any():
                assert s_all[left].max() <= kth[t] + margin, \
                    f"pair {(i, h)}: a key above s_(k) was left out"
    return int(dec.sum()), n_und


def check_values(name, gpu, ref, dtype, mask=None):
    """Asserts the error figures of one output or gradient; returns them."""
    g, r = _np(gpu), _np(ref)
    if mask is not None:
        g, r = g[mask], r[mask]
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    tol = TOL[dtype]
    errs = {"normwise": normwise(g, r), "elementwise": elementwise(g, r)}
    if name.startswith("lse"):
        errs["lse"] = lse_error(g, r)
        assert errs["lse"] <= tol, f"{name}: error {errs['lse']:.3e} > {tol:.0e}"
    else:
        errs["rowwise"] = rowwise(g, r, ROW_FLOOR[dtype])
        assert errs["rowwise"] <= tol, \
            f"{name}: per-row relative error {errs['rowwise']:.3e} > {tol:.0e}"
    assert errs["normwise"] <= tol, \
        f"{name}: normwise relative error {errs['normwise']:.3e} > {tol:.0e}"
    return errs
