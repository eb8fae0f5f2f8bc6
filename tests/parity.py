"""Comparison rules between the CUDA path and the fp64 oracle.

Selection: for every (query, head) whose k-th/(k+1)-th oracle score gap is
larger than 1e-3 |s_(k)| ("decided"), the kept key set must match exactly;
for the other pairs any set whose every member scores within that margin of
s_(k) is accepted (several sets are correct when scores nearly tie).
Values: normwise relative error max|gpu - ref| / max|ref| per tensor, at most
2e-2 for bf16 inputs and 1e-4 for fp32 inputs, where ref is the oracle's
attention over the GPU-selected sets (and, on decided pairs, the oracle's own
result).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
GAP_REL = 1e-3


def normwise(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0))


def check_selection(Q, K, offsets, idx_gpu, ref, pairs_q=None, pairs_h=None):
    """ref: oracle fwd result (full, or for the listed pairs).  Returns the
    number of decided and undecided pairs; raises AssertionError on a
    mismatch."""
    Qd = Q.detach().cpu().double().numpy()
    Kd = K.detach().cpu().double().numpy()
    off = offsets.detach().cpu().numpy().astype(np.int64) if offsets is not None else \
        np.array([0, Qd.shape[0]], dtype=np.int64)
    gi = idx_gpu.detach().cpu().numpy()
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
        g = np.searchsorted(off, i, side="right") - 1
        while g + 1 < len(off) - 1 and off[g + 1] <= i:
            g += 1
        n = int(off[g + 1] - off[g])
        keff = min(k, n)
        a, b = got[t], ref_idx[t]
        assert (a[keff:] == -1).all(), f"pair {(i, h)}: padding {a}"
        assert (a[:keff] >= off[g]).all() and (a[:keff] < off[g + 1]).all(), \
            f"pair {(i, h)}: key outside graph {a}"
        assert len(set(a[:keff].tolist())) == keff, f"pair {(i, h)}: repeated key {a}"
        if dec[t]:
            assert set(a[:keff].tolist()) == set(b[:keff].tolist()), \
                f"pair {(i, h)}: gpu {sorted(a[:keff])} oracle {sorted(b[:keff])}"
        else:
            n_und += 1
            s = Kd[a[:keff], h] @ Qd[i, h]
            margin = GAP_REL * abs(kth[t]) + 1e-6 * np.abs(Kd[a[:keff], h]).sum() * np.abs(Qd[i, h]).max()
            assert s.min() >= kth[t] - margin, f"pair {(i, h)}: invalid near-tie set"
    return int(dec.sum()), n_und


def check_values(name, gpu, ref, dtype, mask=None):
    g = gpu.detach().cpu().double().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    r = np.asarray(ref)
    if mask is not None:
        g, r = g[mask], r[mask]
    err = normwise(g, r)
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    assert err <= TOL[dtype], f"{name}: normwise relative error {err:.3e} > {TOL[dtype]:.0e}"
    return err
