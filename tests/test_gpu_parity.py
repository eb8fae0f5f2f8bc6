"""CUDA path vs the fp64 oracle, through the C ABI (ctypes binding).

Small cases compare every (query, head) and every gradient element; the
full-size workloads compare the selection on a seeded sample of pairs (the
oracle fully sorts each sampled query's scores against all keys) and every
output and gradient against the oracle's attention over the GPU-selected
sets.
"""
import numpy as np
import pytest
import torch

import oracle
from graph_transformer_sparse_kmip_b200 import binding
from graph_transformer_sparse_kmip_b200 import workloads as wl
from parity import TOL, check_selection, check_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    binding.load()
    return torch.device("cuda:0")


def _to(dev, inp):
    return {n: (t.to(dev) if t is not None else None) for n, t in inp.items()}


def _run(dev, inp, k, scale, bwd=True, use_offsets=True):
    g = _to(dev, inp)
    off = g["offsets"] if use_offsets else None
    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], k, scale, off)
    res = dict(out=out, idx=idx, lse=lse)
    if bwd:
        dQ, dK, dV = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, scale)
        res.update(dQ=dQ, dK=dK, dV=dV)
    torch.cuda.synchronize()
    binding.check_status()
    return res


def _full_compare(inp, res, k, scale, bwd=True):
    dt = inp["Q"].dtype
    ref = oracle.fwd(inp["Q"], inp["K"], inp["V"], inp["offsets"], k, scale)
    n_dec, n_und = check_selection(inp["Q"], inp["K"], inp["offsets"], res["idx"], ref)
    dec = oracle.decided(ref["gap"], ref["kth"])
    check_values("out(decided)", res["out"], ref["out"], dt, mask=dec)
    check_values("lse(decided)", res["lse"], ref["lse"], dt, mask=dec)
    dO = inp.get("dO") if bwd else None
    given = oracle.given_idx(inp["Q"], inp["K"], inp["V"], res["idx"].cpu(), inp["offsets"],
                             scale, dO=dO)
    check_values("out", res["out"], given["out"], dt)
    check_values("lse", res["lse"], given["lse"], dt)
    if bwd:
        for n in ("dQ", "dK", "dV"):
            check_values(n, res[n], given[n], dt)
    return n_dec, n_und


def test_tiny_f32_workload(dev):
    w = wl.WORKLOADS["tiny_n1024_f32"]
    inp = wl.make_inputs(w)
    res = _run(dev, inp, w.k, w.scale, bwd=False)
    n_dec, _ = _full_compare(inp, res, w.k, w.scale, bwd=False)
    assert n_dec > 0.8 * 1024


def test_batched_workload_fwd_bwd(dev):
    w = wl.WORKLOADS["batched64_n300to600"]
    inp = wl.make_inputs(w)
    res = _run(dev, inp, w.k, w.scale)
    _full_compare(inp, res, w.k, w.scale)


SIZES = [1, 0, 37, 300, 129, 513, 7]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("k", [1, 5, 15, 45, 64])
def test_small_shapes(dev, dtype, d, k):
    inp = wl.random_case(SIZES, H=2, d=d, dtype=dtype, seed=d * 100 + k)
    scale = 1.0 / np.sqrt(d)
    res = _run(dev, inp, k, scale)
    _full_compare(inp, res, k, scale)


@pytest.mark.parametrize("d,k", [(32, 15), (128, 16), (16, 64), (64, 45)])
def test_max_heads(dev, d, k):
    # 64 heads: rows of H * d * 2 bytes (up to 16 KiB) in the tensor maps and
    # 64 work items per graph slice.
    inp = wl.random_case([300, 5, 171], H=64, d=d, dtype="bf16", seed=900 + d + k)
    res = _run(dev, inp, k, 1.0 / np.sqrt(d))
    _full_compare(inp, res, k, 1.0 / np.sqrt(d))


def test_single_graph_null_offsets(dev):
    inp = wl.random_case([777], H=3, d=32, dtype="bf16", seed=4)
    a = _run(dev, inp, 15, 0.2, bwd=False, use_offsets=True)
    b = _run(dev, inp, 15, 0.2, bwd=False, use_offsets=False)
    assert torch.equal(a["idx"], b["idx"]) and torch.equal(a["out"], b["out"])


def test_forward_is_deterministic(dev):
    inp = wl.random_case([1000, 333], H=4, d=32, dtype="bf16", seed=6)
    a = _run(dev, inp, 15, 0.2)
    b = _run(dev, inp, 15, 0.2)
    for n in ("out", "idx", "lse", "dQ"):
        assert torch.equal(a[n], b[n]), n


def test_side_stream(dev):
    inp = wl.random_case([600], H=2, d=32, dtype="bf16", seed=8)
    g = _to(dev, inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], 15, 0.2, g["offsets"], stream=s)
    s.synchronize()
    ref = _run(dev, inp, 15, 0.2, bwd=False)
    assert torch.equal(idx, ref["idx"]) and torch.equal(out, ref["out"])


def test_malformed_offsets_reported_and_outputs_untouched(dev):
    inp = wl.random_case([50, 50], H=1, d=32, dtype="bf16", seed=1)
    g = _to(dev, inp)
    bad = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=dev)
    out = torch.full_like(g["Q"], 7.0)
    idx = torch.full((100, 1, 5), -7, dtype=torch.int32, device=dev)
    lse = torch.full((100, 1), 7.0, device=dev)
    rc = binding.kmip_attn_fwd(g["Q"], g["K"], g["V"], bad, 100, 1, 32, 5, 0.2, out, idx, lse)
    assert rc == 0
    assert binding.kmip_get_status() == 4  # KMIP_ERR_BAD_OFFSETS
    assert binding.kmip_get_status() == 0  # cleared
    assert (out == 7.0).all() and (idx == -7).all() and (lse == 7.0).all()
    bad_end = torch.tensor([0, 50, 99], dtype=torch.int32, device=dev)
    rc = binding.kmip_attn_fwd(g["Q"], g["K"], g["V"], bad_end, 100, 1, 32, 5, 0.2, out, idx, lse)
    assert rc == 0 and binding.kmip_get_status() == 4


def test_bad_index_reported(dev):
    inp = wl.random_case([64], H=1, d=32, dtype="bf16", seed=2)
    g = _to(dev, inp)
    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], 4, 0.2)
    idx[3, 0, 1] = 64  # out of range
    binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, 0.2)
    assert binding.kmip_get_status() == 6  # KMIP_ERR_BAD_INDEX
    assert binding.kmip_get_status() == 0


def test_bounded_wait_times_out_and_context_survives(dev):
    import time
    t0 = time.time()
    assert binding.kmip_test_wait_timeout(20000) == 0   # 20 ms limit
    assert binding.kmip_get_status() == 5               # KMIP_ERR_TIMEOUT
    assert time.time() - t0 < 10
    assert binding.kmip_get_status() == 0
    inp = wl.random_case([300], H=2, d=32, dtype="bf16", seed=3)
    res = _run(dev, inp, 15, 0.2)                       # the context still works
    _full_compare(inp, res, 15, 0.2)


# --- full-size workloads, in the configuration the benchmark runs ---

def _large(dev, name, k=None, n_pairs=512, bwd=None):
    w = wl.WORKLOADS[name]
    k = k or w.k
    inp = wl.make_inputs(w)
    bwd = ("bwd" in w.phases) if bwd is None else bwd
    res = _run(dev, inp, k, w.scale, bwd=bwd)
    N, H = inp["Q"].shape[:2]
    pq, ph = wl.sample_pairs(N, H, n_pairs, seed=k)
    ref = oracle.fwd_pairs(inp["Q"], inp["K"], inp["V"], inp["offsets"], k, w.scale,
                           pq.numpy(), ph.numpy())
    n_dec, n_und = check_selection(inp["Q"], inp["K"], inp["offsets"], res["idx"], ref,
                                   pq.numpy(), ph.numpy())
    dt = inp["Q"].dtype
    dec = oracle.decided(ref["gap"], ref["kth"])
    sel = (pq.numpy(), ph.numpy())
    check_values("out(sample)", res["out"].cpu()[sel], ref["out"], dt, mask=dec)
    check_values("lse(sample)", res["lse"].cpu()[sel], ref["lse"], dt, mask=dec)
    given = oracle.given_idx(inp["Q"], inp["K"], inp["V"], res["idx"].cpu(), inp["offsets"],
                             w.scale, dO=inp.get("dO") if bwd else None)
    check_values("out", res["out"], given["out"], dt)
    check_values("lse", res["lse"], given["lse"], dt)
    if bwd:
        for n in ("dQ", "dK", "dV"):
            check_values(n, res[n], given[n], dt)
    assert n_dec >= 0.2 * len(pq)


def test_graph_n31623(dev):
    _large(dev, "graph_n31623")


@pytest.mark.parametrize("k", [5, 15, 45])
def test_gmm_n100000(dev, k):
    _large(dev, "gmm_n100000", k=k)


def test_pointcloud_n524288(dev):
    _large(dev, "pointcloud_n524288", n_pairs=128)
