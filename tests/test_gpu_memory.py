"""Memory stays linear in N (k-Maximum Inner Product Attention for Graph
Transformers ..., Abstract: the attention score computation's memory is
linear in the number of nodes).

At N = 100,000 (H = 4, d = 32, k = 15) a dense score matrix would be
N^2 * H * 4 bytes = 160 GB.  The library's own device allocations (the
work list, from the library's scratch pool) must stay far below even
N^2 / 64 bytes, and the outputs and gradients the binding allocates are
O(N H d).  The deterministic backward's sort scratch is O(N H k).
"""
import pytest
import torch

from graph_transformer_sparse_kmip_b200 import binding
from graph_transformer_sparse_kmip_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_memory_is_linear_in_n():
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS["gmm_n100000"]
    inp = wl.make_inputs(w, with_grad_out=True)
    g = {n: t.to(dev) for n, t in inp.items()}
    N, H, d = inp["Q"].shape
    # warm-up call (loads the library, creates its pool)
    binding.attn_fwd(g["Q"], g["K"], g["V"], w.k, w.scale, g["offsets"])
    torch.cuda.synchronize()

    binding.kmip_scratch_usage(reset_high=True)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)

    out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], w.k, w.scale, g["offsets"])
    dQ, dK, dV = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, w.scale)
    torch.cuda.synchronize()
    binding.check_status()

    reserved, lib_high = binding.kmip_scratch_usage()
    torch_peak = torch.cuda.max_memory_allocated(dev) - base
    # The library: only the work list (16 B per item, about N/256 + 1 items).
    assert 0 < lib_high <= 1 << 20, lib_high
    assert lib_high < N * N // 64
    assert reserved < N * N // 64, reserved
    # The binding's outputs and gradients: out, idx, lse, dQ, dK, dV.
    linear = N * H * (2 * d + 4 * w.k + 4 + 3 * 4 * d)
    assert torch_peak <= 2 * linear, (torch_peak, linear)
    assert torch.isfinite(out.float()).all() and (idx >= 0).all()

    # The deterministic backward's scratch: about 28 bytes per kept key plus
    # 4 per (node, head), kept by the pool for the next call.
    binding.kmip_scratch_usage(reset_high=True)
    binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, w.scale, deterministic=True)
    torch.cuda.synchronize()
    binding.check_status()
    reserved2, high2 = binding.kmip_scratch_usage()
    kept = N * H * w.k
    assert 20 * kept <= high2 <= 40 * kept + 8 * N * H + (4 << 20), (high2, kept)
    assert reserved2 >= high2

    # trimming returns the kept memory once the work is done
    torch.cuda.synchronize()
    binding.kmip_scratch_trim()
    reserved3, _ = binding.kmip_scratch_usage()
    assert reserved3 < reserved2, (reserved3, reserved2)
    assert reserved3 <= 64 << 20, reserved3
