"""The parity rules themselves (tests/parity.py), checked on the CPU.

The selection rule must reject every wrong answer a GPU kernel could give
-- a dropped best key, a key of another graph, a repeated key, bad padding,
a scrambled order, a differing set on a decided pair -- and must accept the
other valid answer of a near tie.  The value rules must catch a single bad
row that a tensor-wide (normwise) figure hides.  Everything here is built by
hand, so no GPU and no kernel output is involved.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (TOL, check_selection, check_values, elementwise, lse_error, normwise,
                    rowwise)


def _case():
    # d = 1, H = 1.  Graph 0 = nodes 0..5, graph 1 = nodes 6..9.
    #   node 0 (q = 1):  scores 10, 9, 5, 4.999, 1, 0 -> k = 3: s_(3) = 5,
    #                    gap = 0.001 < 1e-3 * 5, undecided; {0,1,2} or {0,1,3}.
    #   node 6 (q = 1):  scores 3, 2, 1, 0 -> s_(3) = 1, gap = 1, decided: {6,7,8}.
    K = np.array([10, 9, 5, 4.999, 1, 0, 3, 2, 1, 0], dtype=np.float64).reshape(10, 1, 1)
    Q = np.array([1, -1, 2, 0.5, -2, 3, 1, -1, 0.25, 2], dtype=np.float64).reshape(10, 1, 1)
    V = np.arange(10, dtype=np.float64).reshape(10, 1, 1)
    off = np.array([0, 6, 10], dtype=np.int64)
    k = 3
    ref = oracle.fwd(Q, K, V, off, k, 1.0, nthreads=1)
    return Q, K, off, ref


def _check(idx, Q, K, off, ref):
    return check_selection(torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(off),
                           torch.from_numpy(idx), ref)


def test_case_has_the_intended_decided_pattern():
    Q, K, off, ref = _case()
    dec = oracle.decided(ref["gap"], ref["kth"])
    assert not dec[0, 0] and dec[6, 0]
    assert sorted(ref["idx"][0, 0].tolist()) == [0, 1, 2]


def test_oracle_sets_pass():
    Q, K, off, ref = _case()
    n_dec, n_und = _check(ref["idx"].copy(), Q, K, off, ref)
    assert n_dec + n_und == 10 and n_und >= 1


def test_near_tie_alternative_passes():
    Q, K, off, ref = _case()
    idx = ref["idx"].copy()
    idx[0, 0] = [0, 1, 3]          # key 3 (4.999) instead of key 2 (5): a valid top-3
    _check(idx, Q, K, off, ref)


@pytest.mark.parametrize("row,bad", [
    (0, [1, 2, 3]),     # undecided pair: drops the best key (10) for near-tie keys
    (6, [6, 7, 9]),     # decided pair: a different set
    (6, [6, 7, 2]),     # a key of another graph
    (6, [6, 7, 7]),     # a repeated key
    (6, [7, 6, 8]),     # not in descending score order
    (0, [0, 1, 5]),     # undecided pair: a key far below s_(k)
])
def test_wrong_sets_fail(row, bad):
    Q, K, off, ref = _case()
    idx = ref["idx"].copy()
    idx[row, 0] = bad
    with pytest.raises(AssertionError):
        _check(idx, Q, K, off, ref)


def test_bad_padding_fails():
    # a 2-node graph with k = 3 keeps 2 keys and one -1
    Q = np.array([1.0, 2.0, 1.0]).reshape(3, 1, 1)
    K = np.array([1.0, 0.0, 5.0]).reshape(3, 1, 1)
    V = np.zeros((3, 1, 1))
    off = np.array([0, 2, 3], dtype=np.int64)
    ref = oracle.fwd(Q, K, V, off, 3, 1.0, nthreads=1)
    idx = ref["idx"].copy()
    _check(idx, Q, K, off, ref)
    idx[0, 0] = [0, 1, 2]
    with pytest.raises(AssertionError):
        _check(idx, Q, K, off, ref)


def test_rowwise_catches_a_bad_row_normwise_misses():
    rng = np.random.default_rng(0)
    ref = rng.normal(size=(50, 2, 8))
    ref[7, 1] *= 1e-2                     # a small-magnitude row
    gpu = ref.copy()
    gpu[7, 1] *= 1.5                      # entirely wrong by 50%
    assert normwise(gpu, ref) < TOL[torch.bfloat16]
    assert rowwise(gpu, ref) > 0.4
    with pytest.raises(AssertionError):
        check_values("dK", gpu, ref, torch.bfloat16)


def test_rowwise_floor_keeps_zero_rows_finite():
    ref = np.zeros((4, 1, 8)); ref[0] = 1.0
    gpu = ref.copy(); gpu[3, 0, 0] = 1e-9   # a zero row off by far less than the floor
    assert rowwise(gpu, ref) <= 1e-6
    assert elementwise(gpu, ref) <= 1e-6


def test_lse_rule_is_elementwise():
    ref = np.array([[5.0, 3.0], [0.5, 100.0]])
    gpu = ref.copy()
    gpu[1, 0] += 0.05                     # 5% off in the normaliser of one pair
    assert normwise(gpu, ref) < TOL[torch.bfloat16]
    assert abs(lse_error(gpu, ref) - 0.05) < 1e-12
    with pytest.raises(AssertionError):
        check_values("lse", gpu, ref, torch.bfloat16)
    gpu[1, 0] = ref[1, 0] + 1e-3
    check_values("lse", gpu, ref, torch.bfloat16)
