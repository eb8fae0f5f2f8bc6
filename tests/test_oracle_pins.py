"""Pins for the fp64 oracle: checks against things other than the oracle itself.

The pages (k-Maximum Inner Product Attention for Graph Transformers and the
Expressive Power of GraphGPS) print no worked example, so the oracle is
pinned by
  * hand-derived closed-form cases (tests/golden/handworked.json);
  * k >= n_g reducing to full softmax attention (the approximation claim of
    the Abstract and the full-attention comparison of Figure 8a), computed by
    torch's dense fp64 softmax and autograd -- a library routine;
  * k = 1 reducing to "return the V row of the arg-max key" (closed form);
  * brute-force enumeration of all k-subsets on tiny graphs and torch.topk;
  * central finite differences of the forward for the backward;
  * permutation equivariance f(PH, PAP^T) = P f(H, A) (the GNN background
    page, section 1) and block-diagonal batching.
Each check is chosen so that a plausible slip (a dropped scale, a wrong sign,
a transposed operand, a missing key, an off-by-one in the padding) fails.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from graph_transformer_sparse_kmip_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "handworked.json")


def _ev(expr) -> float:
    if isinstance(expr, (int, float)):
        return float(expr)
    return float(eval(expr, {"__builtins__": {}},
                      {"ln": math.log, "Fraction": Fraction, "inf": math.inf}))


def _arr(rows):
    return np.array([[_ev(x) for x in r] if isinstance(r, list) else _ev(r) for r in rows])


def _case_inputs(c):
    N = len(c["Q"])
    H, d = c["H"], c["d"]
    Q = np.array(c["Q"], dtype=np.float64).reshape(N, H, d)
    K = np.array(c["K"], dtype=np.float64).reshape(N, H, d)
    V = np.array(c["V"], dtype=np.float64).reshape(N, H, d)
    return N, H, d, Q, K, V


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_handworked(case):
    N, H, d, Q, K, V = _case_inputs(case)
    k, scale = case["k"], _ev(case["scale"])
    off = np.array(case["offsets"], dtype=np.int64)
    r = oracle.fwd(Q, K, V, off, k, scale, nthreads=2)
    np.testing.assert_array_equal(r["idx"].reshape(N, k), np.array(case["idx"]))
    np.testing.assert_allclose(r["lse"].reshape(N), _arr(case["lse"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(r["out"].reshape(N, d), _arr(case["out"]), rtol=0, atol=1e-13)
    # order statistics behind the parity rule: s_(k_eff), s_(k) - s_(k+1), decided
    np.testing.assert_array_equal(r["kth"].reshape(N), _arr(case["kth"]))
    np.testing.assert_array_equal(r["gap"].reshape(N), _arr(case["gap"]))
    np.testing.assert_array_equal(oracle.decided(r["gap"], r["kth"]).reshape(N),
                                  np.array(case["decided"]))
    if "dO" in case:
        dO = np.array(case["dO"], dtype=np.float64).reshape(N, H, d)
        g = oracle.given_idx(Q, K, V, r["idx"], off, scale, dO=dO)
        for name in ("dQ", "dK", "dV"):
            np.testing.assert_allclose(g[name].reshape(N, d), _arr(case[name]), rtol=0, atol=1e-13,
                                       err_msg=name)


def _dense_attention_fp64(Q, K, V, off, scale):
    """Full softmax attention inside each graph, by torch (library routine)."""
    Qt = torch.tensor(Q, dtype=torch.float64, requires_grad=True)
    Kt = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    Vt = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    N = Q.shape[0]
    gid = np.zeros(N, dtype=np.int64)
    for g in range(len(off) - 1):
        gid[off[g]:off[g + 1]] = g
    mask = torch.tensor(gid[:, None] != gid[None, :])
    logits = torch.einsum("ihc,jhc->hij", Qt, Kt) * scale
    logits = logits.masked_fill(mask[None], float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)               # [H, N]
    out = torch.einsum("hij,jhc->ihc", torch.softmax(logits, dim=-1), Vt)
    return Qt, Kt, Vt, out, lse.T


@pytest.mark.parametrize("seed", [0, 1])
def test_k_ge_graph_size_is_full_attention(seed):
    sizes = [5, 9, 1, 7]
    c = wl.random_case(sizes, H=2, d=6, dtype="f32", seed=seed)
    Q, K, V, dO = (c[n].double().numpy() for n in ("Q", "K", "V", "dO"))
    off = c["offsets"].numpy().astype(np.int64)
    scale = 0.37
    k = max(sizes) + 3
    r = oracle.fwd(Q, K, V, off, k, scale, nthreads=3)
    Qt, Kt, Vt, out, lse = _dense_attention_fp64(Q, K, V, off, scale)
    np.testing.assert_allclose(r["out"], out.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse.detach().numpy(), rtol=0, atol=1e-12)
    # padding: a graph of n nodes keeps exactly n keys
    for g in range(len(sizes)):
        rows = r["idx"][off[g]:off[g + 1]]
        assert (rows[..., :sizes[g]] >= off[g]).all() and (rows[..., :sizes[g]] < off[g + 1]).all()
        assert (rows[..., sizes[g]:] == -1).all()
    # backward against torch autograd of the dense attention
    (out * torch.tensor(dO)).sum().backward()
    g = oracle.given_idx(Q, K, V, r["idx"], off, scale, dO=dO)
    np.testing.assert_allclose(g["dQ"], Qt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dK"], Kt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dV"], Vt.grad.numpy(), rtol=0, atol=1e-12)


def test_k1_is_argmax_row():
    c = wl.random_case([40, 13], H=3, d=8, dtype="f32", seed=3)
    Q, K, V, dO = (c[n].double().numpy() for n in ("Q", "K", "V", "dO"))
    off = c["offsets"].numpy().astype(np.int64)
    scale = 0.5
    r = oracle.fwd(Q, K, V, off, 1, scale, nthreads=2)
    N, H, d = Q.shape
    g = oracle.given_idx(Q, K, V, r["idx"], off, scale, dO=dO)
    dV_expect = np.zeros_like(V)
    for i in range(N):
        gi = np.searchsorted(off, i, side="right") - 1
        for h in range(H):
            s = K[off[gi]:off[gi + 1], h] @ Q[i, h]
            j = off[gi] + int(np.argmax(s))
            assert r["idx"][i, h, 0] == j
            np.testing.assert_allclose(r["out"][i, h], V[j, h], rtol=0, atol=1e-14)
            assert abs(r["lse"][i, h] - scale * s.max()) < 1e-12
            dV_expect[j, h] += dO[i, h]
    assert np.abs(g["dQ"]).max() < 1e-13 and np.abs(g["dK"]).max() < 1e-13
    np.testing.assert_allclose(g["dV"], dV_expect, rtol=0, atol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_selection_brute_force_subsets(seed):
    sizes = [7, 4, 9]
    c = wl.random_case(sizes, H=2, d=3, dtype="f32", seed=10 + seed)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    off = c["offsets"].numpy().astype(np.int64)
    for k in (1, 2, 3, 5):
        r = oracle.fwd(Q, K, V, off, k, 1.0, nthreads=1)
        for i in range(Q.shape[0]):
            gi = np.searchsorted(off, i, side="right") - 1
            keys = list(range(off[gi], off[gi + 1]))
            for h in range(Q.shape[1]):
                sc = {j: float(Q[i, h] @ K[j, h]) for j in keys}
                keff = min(k, len(keys))
                best = max(itertools.combinations(keys, keff), key=lambda S: sum(sc[j] for j in S))
                assert set(r["idx"][i, h, :keff].tolist()) == set(best)
                assert (r["idx"][i, h, keff:] == -1).all()
                # order statistics by brute force: the smallest score of the
                # best subset, and the best score outside it
                kth = min(sc[j] for j in best)
                rest = [sc[j] for j in keys if j not in best]
                gap = kth - max(rest) if len(keys) > k else np.inf
                assert abs(r["kth"][i, h] - kth) <= 1e-12
                assert r["gap"][i, h] == gap if np.isinf(gap) else abs(r["gap"][i, h] - gap) <= 1e-12


def test_selection_matches_torch_topk():
    c = wl.random_case([300, 257], H=4, d=16, dtype="bf16", seed=5, with_grad_out=False)
    Q, K, V = (c[n].double() for n in ("Q", "K", "V"))
    off = c["offsets"].numpy().astype(np.int64)
    k = 15
    r = oracle.fwd(Q, K, V, off, k, 0.25)
    for g in range(len(off) - 1):
        sl = slice(off[g], off[g + 1])
        s = torch.einsum("ihc,jhc->hij", Q[sl], K[sl])          # [H, n, n]
        top = torch.topk(s, k, dim=-1).indices + off[g]        # [H, n, k]
        got = torch.tensor(r["idx"][sl]).permute(1, 0, 2)
        assert torch.equal(torch.sort(top, dim=-1).values, torch.sort(got.long(), dim=-1).values)


def test_idx_order_is_descending_score_then_index():
    c = wl.random_case([50], H=2, d=4, dtype="f32", seed=8, with_grad_out=False)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    off = c["offsets"].numpy().astype(np.int64)
    r = oracle.fwd(Q, K, V, off, 10, 1.0)
    for i in range(50):
        for h in range(2):
            s = [float(Q[i, h] @ K[j, h]) for j in r["idx"][i, h]]
            assert all(a >= b for a, b in zip(s, s[1:]))


def test_finite_difference_gradients():
    """Central differences of L = sum(out * dO) with the selection held by
    large score gaps (so the top-k sets do not move under the perturbation)."""
    rng = np.random.default_rng(7)
    N, H, d, k = 9, 2, 3, 3
    Q = rng.normal(size=(N, H, d))
    K = rng.normal(size=(N, H, d)) * 3.0
    V = rng.normal(size=(N, H, d))
    dO = rng.normal(size=(N, H, d))
    off = np.array([0, 5, 9], dtype=np.int64)
    scale = 0.8
    r = oracle.fwd(Q, K, V, off, k, scale, nthreads=1)
    finite = np.isfinite(r["gap"])
    assert (r["gap"][finite] > 1e-3).all(), "seed gives a near-tie; choose another"
    g = oracle.given_idx(Q, K, V, r["idx"], off, scale, dO=dO)
    h = 1e-6

    def loss(Qx, Kx, Vx):
        rr = oracle.fwd(Qx, Kx, Vx, off, k, scale, nthreads=1)
        assert np.array_equal(rr["idx"], r["idx"])
        return float((rr["out"] * dO).sum())

    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        fd = np.zeros_like(X)
        for pos in itertools.product(*(range(n) for n in X.shape)):
            Xp, Xm = X.copy(), X.copy()
            Xp[pos] += h
            Xm[pos] -= h
            args_p = [Xp if Y is X else Y for Y in (Q, K, V)]
            args_m = [Xm if Y is X else Y for Y in (Q, K, V)]
            fd[pos] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g[name], fd, rtol=0, atol=1e-7, err_msg=name)


def test_permutation_equivariance():
    sizes = [30, 11, 25]
    c = wl.random_case(sizes, H=2, d=8, dtype="f32", seed=21, with_grad_out=True)
    Q, K, V, dO = (c[n].double().numpy() for n in ("Q", "K", "V", "dO"))
    off = c["offsets"].numpy().astype(np.int64)
    k, scale = 6, 0.4
    r = oracle.fwd(Q, K, V, off, k, scale)
    g = oracle.given_idx(Q, K, V, r["idx"], off, scale, dO=dO)
    # relabel: reverse the graph order and shuffle nodes inside each graph
    rng = np.random.default_rng(0)
    perm, new_sizes = [], []
    for gi in reversed(range(len(sizes))):
        nodes = np.arange(off[gi], off[gi + 1])
        rng.shuffle(nodes)
        perm.extend(nodes.tolist())
        new_sizes.append(sizes[gi])
    perm = np.array(perm)                      # new node t is old node perm[t]
    inv = np.empty_like(perm); inv[perm] = np.arange(len(perm))
    off2 = np.concatenate([[0], np.cumsum(new_sizes)]).astype(np.int64)
    r2 = oracle.fwd(Q[perm], K[perm], V[perm], off2, k, scale)
    g2 = oracle.given_idx(Q[perm], K[perm], V[perm], r2["idx"], off2, scale, dO=dO[perm])
    np.testing.assert_allclose(r2["out"], r["out"][perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r2["lse"], r["lse"][perm], rtol=0, atol=1e-12)
    mapped = np.where(r2["idx"] >= 0, perm[np.maximum(r2["idx"], 0)], -1)
    np.testing.assert_array_equal(np.sort(mapped, -1), np.sort(r["idx"][perm], -1))
    for name in ("dQ", "dK", "dV"):
        np.testing.assert_allclose(g2[name], g[name][perm], rtol=0, atol=1e-12, err_msg=name)


def test_block_diagonal_equals_separate_graphs():
    sizes = [20, 0, 33, 3]
    c = wl.random_case(sizes, H=2, d=4, dtype="f32", seed=4, with_grad_out=False)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    off = c["offsets"].numpy().astype(np.int64)
    k = 5
    r = oracle.fwd(Q, K, V, off, k, 0.9)
    for g in range(len(sizes)):
        a, b = off[g], off[g + 1]
        if a == b:
            continue
        rg = oracle.fwd(Q[a:b], K[a:b], V[a:b], None, k, 0.9)
        np.testing.assert_allclose(r["out"][a:b], rg["out"], rtol=0, atol=0)
        np.testing.assert_array_equal(r["idx"][a:b], np.where(rg["idx"] >= 0, rg["idx"] + a, -1))


def test_positive_key_rescaling_keeps_selection():
    c = wl.random_case([120], H=3, d=8, dtype="f32", seed=9, with_grad_out=False)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    r1 = oracle.fwd(Q, K, V, None, 7, 1.0)
    r2 = oracle.fwd(Q, K * 3.5, V, None, 7, 1.0)
    np.testing.assert_array_equal(r1["idx"], r2["idx"])
    # and the softmax does see the scale: lse changes
    assert np.abs(r1["lse"] - r2["lse"]).max() > 1e-3


def test_pairs_match_full_run_and_given_idx():
    c = wl.random_case([200, 150], H=2, d=16, dtype="bf16", seed=2, with_grad_out=False)
    off = c["offsets"]
    r = oracle.fwd(c["Q"], c["K"], c["V"], off, 9, 0.25)
    pq, ph = wl.sample_pairs(350, 2, 64, seed=1)
    rp = oracle.fwd_pairs(c["Q"], c["K"], c["V"], off, 9, 0.25, pq.numpy(), ph.numpy())
    np.testing.assert_array_equal(rp["idx"], r["idx"][pq.numpy(), ph.numpy()])
    np.testing.assert_array_equal(rp["out"], r["out"][pq.numpy(), ph.numpy()])
    g = oracle.given_idx(c["Q"], c["K"], c["V"], r["idx"], off, 0.25)
    np.testing.assert_allclose(g["out"], r["out"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["lse"], r["lse"], rtol=0, atol=1e-13)


def test_rejects_malformed_offsets():
    c = wl.random_case([10], H=1, d=4, dtype="f32", seed=0, with_grad_out=False)
    with pytest.raises(ValueError):
        oracle.fwd(c["Q"], c["K"], c["V"], np.array([0, 6, 4, 10]), 3, 1.0)
    with pytest.raises(ValueError):
        oracle.fwd(c["Q"], c["K"], c["V"], np.array([0, 9]), 3, 1.0)


def test_workload_generators_are_seeded():
    w = wl.WORKLOADS["batched64_n300to600"]
    a = wl.make_inputs(w)
    b = wl.make_inputs(w)
    assert torch.equal(a["Q"], b["Q"]) and torch.equal(a["offsets"], b["offsets"])
    sizes = np.diff(a["offsets"].numpy())
    assert len(sizes) == 64 and sizes.min() >= 300 and sizes.max() <= 600
    assert a["Q"].dtype == torch.bfloat16 and a["Q"].shape == (int(sizes.sum()), 4, 32)


# --- full softmax attention (the comparison of Figure 8) ---

@pytest.mark.parametrize("seed", [0, 3])
def test_full_attention_matches_torch_dense(seed):
    sizes = [6, 11, 0, 4]
    c = wl.random_case(sizes, H=2, d=5, dtype="f32", seed=seed, with_grad_out=False)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    off = c["offsets"].numpy().astype(np.int64)
    r = oracle.full_attention(Q, K, V, off, 0.6, nthreads=2)
    _, _, _, out, lse = _dense_attention_fp64(Q, K, V, off, 0.6)
    np.testing.assert_allclose(r["out"], out.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse.detach().numpy(), rtol=0, atol=1e-12)
    pq = np.array([0, 7, 20]); ph = np.array([1, 0, 1], dtype=np.int32)
    rp = oracle.full_attention(Q, K, V, off, 0.6, pq, ph)
    np.testing.assert_array_equal(rp["out"], r["out"][pq, ph])


def test_topk_weight_share_rises_to_one():
    """exp(lse_k - lse_full) is the softmax weight the k kept keys carry:
    it grows with k and reaches 1 once k covers the graph."""
    c = wl.random_case([40], H=1, d=8, dtype="f32", seed=2, with_grad_out=False)
    Q, K, V = (c[n].double().numpy() for n in ("Q", "K", "V"))
    full = oracle.full_attention(Q, K, V, None, 0.5)
    prev = np.zeros(40)
    for k in (1, 3, 10, 39, 40, 45):
        r = oracle.fwd(Q, K, V, None, k, 0.5)
        share = np.exp(r["lse"] - full["lse"]).reshape(-1)
        assert (share <= 1 + 1e-12).all() and (share >= prev - 1e-12).all()
        prev = share
    np.testing.assert_allclose(prev, 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["out"], full["out"], rtol=0, atol=1e-12)
