"""kmip_attn_fwd_noalloc: the forward entry point that allocates nothing.

It exists for callers that cannot let the library allocate device memory
(their own pool holds the GPU, their device has no stream-ordered pools, or
they must not allocate once running).  It must give the same results as
kmip_attn_fwd, and -- checked on its own, so that a fault shared by both
entry points cannot hide -- the same results as the fp64 oracle under the
parity rules of tests/parity.py.  Two calls in a row with different inputs
also show that the fixed work-list array, which keeps the previous call's
contents, is fully rewritten by each call.
"""
import numpy as np
import pytest
import torch

import oracle
from graph_transformer_sparse_kmip_b200 import binding
from graph_transformer_sparse_kmip_b200 import workloads as wl
from parity import TOL, check_selection, check_values, normwise

pytestmark = pytest.mark.gpu


def _outputs(Q, k):
    N, H, d = Q.shape
    return (torch.empty_like(Q), torch.empty((N, H, k), dtype=torch.int32, device=Q.device),
            torch.empty((N, H), dtype=torch.float32, device=Q.device))


def _both(g, k, scale, offsets):
    N, H, d = g["Q"].shape
    ref = _outputs(g["Q"], k)
    new = _outputs(g["Q"], k)
    rc = binding.kmip_attn_fwd(g["Q"], g["K"], g["V"], offsets, N, H, d, k, scale, *ref)
    assert rc == 0
    rc = binding.kmip_attn_fwd_noalloc(g["Q"], g["K"], g["V"], offsets, N, H, d, k, scale, *new)
    assert rc == 0, binding.kmip_error_string(rc)
    torch.cuda.synchronize()
    assert binding.kmip_get_status() == 0
    return ref, new


def test_noalloc_forward_matches_allocating_forward():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    cases = [
        (wl.random_case([300, 45, 0, 517, 129], H=2, d=32, dtype="bf16", seed=21), 15),
        (wl.random_case([1000], H=4, d=64, dtype="f32", seed=22), 7),
    ]
    for inp, k in cases:  # two calls in a row, different work lists
        g = {n: t.to(dev) for n, t in inp.items()}
        scale = 1.0 / np.sqrt(g["Q"].shape[-1])
        offsets = g["offsets"] if g["offsets"].numel() > 2 else None
        (o1, i1, l1), (o2, i2, l2) = _both(g, k, scale, offsets)
        tol = TOL[g["Q"].dtype]
        assert torch.equal(i1, i2)
        assert normwise(o2.double().cpu().numpy(), o1.double().cpu().numpy()) <= tol
        assert normwise(l2.double().cpu().numpy(), l1.double().cpu().numpy()) <= tol
        # and against the oracle, on the no-allocation call's own outputs
        dt = inp["Q"].dtype
        ref = oracle.fwd(inp["Q"], inp["K"], inp["V"], inp["offsets"], k, scale)
        check_selection(inp["Q"], inp["K"], inp["offsets"], i2, ref)
        given = oracle.given_idx(inp["Q"], inp["K"], inp["V"], i2.cpu(), inp["offsets"], scale)
        check_values("out", o2, given["out"], dt)
        check_values("lse", l2, given["lse"], dt)


def test_noalloc_rejects_work_lists_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    x = torch.zeros((1, 1, 32), dtype=torch.bfloat16, device=dev)
    o, i, l = _outputs(x, 4)
    # 2^31 - 1 nodes need far more than 65536 items; rejected before any launch
    rc = binding.kmip_attn_fwd_noalloc(x, x, x, None, 2**31 - 1, 1, 32, 4, 0.5, o, i, l)
    assert rc == 7  # KMIP_ERR_SCRATCH_LIMIT
    assert "fixed array" in binding.kmip_error_string(rc)
