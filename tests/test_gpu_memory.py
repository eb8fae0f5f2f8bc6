"""Memory stays linear in N (k-Maximum Inner Product Attention for Graph
Transformers ..., Abstract: the attention score computation's memory is
linear in the number of nodes).

At N = 100,000 (H = 4, d = 32, k = 15) a dense score matrix would be
N^2 * H * 4 bytes = 160 GB.  The library's own device allocations (the
stream-ordered work list, from the device's default memory pool) must stay
far below even N^2 / 64 bytes, and the outputs and gradients the binding
allocates are O(N H d).
"""
import numpy as np
import pytest
import torch

from graph_transformer_sparse_kmip_b200 import binding
from graph_transformer_sparse_kmip_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _pool_used_high(rt, drv, pool, reset=False):
    attr = rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh
    if reset:
        err, = rt.cudaMemPoolSetAttribute(pool, attr, drv.cuuint64_t(0))
        assert err == rt.cudaError_t.cudaSuccess
        return 0
    err, v = rt.cudaMemPoolGetAttribute(pool, attr)
    assert err == rt.cudaError_t.cudaSuccess
    return int(v)


def test_memory_is_linear_in_n():
    rt = pytest.importorskip("cuda.bindings.runtime")
    drv = pytest.importorskip("cuda.bindings.driver")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS["gmm_n100000"]
    inp = wl.make_inputs(w, with_grad_out=True)
    g = {n: t.to(dev) for n, t in inp.items()}
    N, H, d = inp["Q"].shape
    # warm-up call (loads the library, creates the pool's first block)
    binding.attn_fwd(g["Q"], g["K"], g["V"], w.k, w.scale, g["offsets"])
    torch.cuda.synchronize()

    err, pool = rt.cudaDeviceGetDefaultMemPool(0)
    assert err == rt.cudaError_t.cudaSuccess
    _pool_used_high(rt, drv, pool, reset=True)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)

    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], w.k, w.scale, g["offsets"])
    dQ, dK, dV = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, w.scale)
    torch.cuda.synchronize()
    binding.check_status()

    lib_high = _pool_used_high(rt, drv, pool)
    torch_peak = torch.cuda.max_memory_allocated(dev) - base
    # The library: only the work list (16 B per item, about N/256 + 1 items per head slice).
    assert lib_high <= 1 << 20, lib_high
    assert lib_high < N * N // 64
    # The binding's outputs and gradients: out, idx, lse, dQ, dK, dV.
    linear = N * H * (2 * d + 4 * w.k + 4 + 3 * 4 * d)
    assert torch_peak <= 2 * linear, (torch_peak, linear)
    assert torch.isfinite(out.float()).all() and (idx >= 0).all()
