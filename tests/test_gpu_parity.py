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


# --- all-key diagnostics (kmip_attn_fwd_diag) ---

def _diag_compare(dev, inp, k, scale, pairs=None):
    g = _to(dev, inp)
    out, idx, lse, lse_all = binding.attn_fwd_diag(g["Q"], g["K"], g["V"], k, scale, g["offsets"])
    torch.cuda.synchronize()
    binding.check_status()
    # same selection and outputs as the plain forward
    o2, i2, l2 = binding.attn_fwd(g["Q"], g["K"], g["V"], k, scale, g["offsets"])
    assert torch.equal(idx, i2) and torch.equal(out, o2) and torch.equal(lse, l2)
    dt = inp["Q"].dtype
    if pairs is None:
        full = oracle.full_attention(inp["Q"], inp["K"], inp["V"], inp["offsets"], scale)
        check_values("lse_all", lse_all, full["lse"], dt)
        got = lse_all.cpu().double().numpy()
    else:
        pq, ph = pairs
        full = oracle.full_attention(inp["Q"], inp["K"], inp["V"], inp["offsets"], scale, pq, ph)
        got = lse_all.cpu().double().numpy()[pq, ph]
        check_values("lse_all(sample)", got, full["lse"], dt)
    # the kept keys' share of the full softmax weight lies in (0, 1]
    share = np.exp(lse.cpu().double().numpy() - lse_all.cpu().double().numpy())
    assert (share > 0).all() and (share <= 1 + 2 * TOL[dt]).all()
    return share


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,k", [(16, 5), (32, 15), (64, 45), (128, 16)])
def test_diag_lse_all_small(dev, dtype, d, k):
    inp = wl.random_case(SIZES, H=2, d=d, dtype=dtype, seed=7 * d + k)
    _diag_compare(dev, inp, k, 1.0 / np.sqrt(d))


def test_diag_k_covering_the_graph_is_full_attention(dev):
    inp = wl.random_case([30, 5, 0, 64], H=2, d=32, dtype="bf16", seed=5)
    share = _diag_compare(dev, inp, 64, 0.2)
    np.testing.assert_allclose(share, 1.0, rtol=0, atol=1e-4)


def test_diag_graph_n31623(dev):
    w = wl.WORKLOADS["graph_n31623"]
    inp = wl.make_inputs(w, with_grad_out=False)
    N, H = inp["Q"].shape[:2]
    pq, ph = wl.sample_pairs(N, H, 256, seed=3)
    _diag_compare(dev, inp, w.k, w.scale, (pq.numpy(), ph.numpy()))


# --- deterministic backward (kmip_attn_bwd_deterministic) ---

def _det_compare(dev, inp, k, scale):
    g = _to(dev, inp)
    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], k, scale, g["offsets"])
    a = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, scale, deterministic=True)
    b = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, scale, deterministic=True)
    atomic = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, scale)
    torch.cuda.synchronize()
    binding.check_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y), "deterministic backward differs between two runs"
    assert torch.equal(a[0], atomic[0])  # dQ is the same computation in both
    dt = inp["Q"].dtype
    given = oracle.given_idx(inp["Q"], inp["K"], inp["V"], idx.cpu(), inp["offsets"], scale,
                             dO=inp["dO"])
    for name, x in zip(("dQ", "dK", "dV"), a):
        check_values(name, x, given[name], dt)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,k", [(16, 64), (32, 15), (64, 45), (128, 5)])
def test_deterministic_bwd_small(dev, dtype, d, k):
    inp = wl.random_case(SIZES, H=2, d=d, dtype=dtype, seed=3 * d + k)
    _det_compare(dev, inp, k, 1.0 / np.sqrt(d))


def test_deterministic_bwd_gmm_n100000(dev):
    w = wl.WORKLOADS["gmm_n100000"]
    _det_compare(dev, wl.make_inputs(w), w.k, w.scale)


# --- exact ties: the smaller key index wins ---

@pytest.mark.parametrize("dtype,d,k", [("bf16", 32, 15), ("bf16", 16, 45), ("f32", 32, 15),
                                       ("bf16", 64, 5)])
def test_exact_ties_go_to_the_smaller_index(dev, dtype, d, k):
    """Many keys are exact copies of one strong key, so their scores tie
    bit for bit (the same products summed in the same order) and the k-th and
    (k+1)-th best are equal.  The pages give no tie rule; the library's (and
    the oracle's) is larger score first, then the smaller node index, so on
    every exactly tied pair the kept set must be the oracle's."""
    sizes = [700, 300]
    inp = wl.random_case(sizes, H=2, d=d, dtype=dtype, seed=77 + d)
    K = inp["K"].clone()
    for h in range(2):
        strong = K[5, h] * 3                      # one key far above the rest
        for j in list(range(100, 160)) + list(range(720, 740)):
            K[j, h] = strong
        K[650, h] = strong
    inp["K"] = K
    res = _run(dev, inp, k, 1.0 / np.sqrt(d), bwd=False)
    ref = oracle.fwd(inp["Q"], inp["K"], inp["V"], inp["offsets"], k, 1.0 / np.sqrt(d))
    got = res["idx"].cpu().numpy()
    # where the oracle's k-th and (k+1)-th scores tie exactly, the kept set
    # must still be the oracle's (ties to the smaller index)
    tied = ref["gap"] == 0
    assert tied.sum() > 100
    same = (np.sort(got, -1) == np.sort(ref["idx"], -1)).all(-1)
    assert same[tied].all(), f"{(~same[tied]).sum()} tied pairs keep other keys"


# --- attention over given sets (kmip_attn_gather) ---

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,k", [(16, 5), (32, 15), (64, 45), (128, 64)])
def test_gather_given_sets(dev, dtype, d, k):
    inp = wl.random_case(SIZES, H=2, d=d, dtype=dtype, seed=11 * d + k)
    g = _to(dev, inp)
    scale = 1.0 / np.sqrt(d)
    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], k, scale, g["offsets"])
    o2, l2 = binding.attn_gather(g["Q"], g["K"], g["V"], idx, scale)
    torch.cuda.synchronize()
    binding.check_status()
    dt = inp["Q"].dtype
    given = oracle.given_idx(inp["Q"], inp["K"], inp["V"], idx.cpu(), inp["offsets"], scale)
    check_values("out", o2, given["out"], dt)
    check_values("lse", l2, given["lse"], dt)


def test_gather_gmm_n100000(dev):
    w = wl.WORKLOADS["gmm_n100000"]
    inp = wl.make_inputs(w, with_grad_out=False)
    g = _to(dev, inp)
    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], w.k, w.scale, g["offsets"])
    o2, l2 = binding.attn_gather(g["Q"], g["K"], g["V"], idx, w.scale)
    torch.cuda.synchronize()
    binding.check_status()
    dt = inp["Q"].dtype
    # the same attention as the fused forward's, over the same sets
    check_values("out", o2, out, dt)
    check_values("lse", l2, lse, dt)
