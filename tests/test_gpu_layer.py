"""GraphGPS global-attention block (projection, k-MIP attention, output
projection, residual) against an fp64 reference on the CPU.

The reference applies the same parameters in fp64 with torch and takes the
attention over the GPU-selected key sets from the oracle (forward and
backward, ``oracle.given_idx``), so every gradient -- of the input, of both
projections' weights and biases -- is compared through the whole block.
The GPU's selection itself is checked against the oracle's on the GPU's own
projected queries and keys.
"""
import numpy as np
import pytest
import torch

import oracle
from graph_transformer_sparse_kmip_b200 import binding
from graph_transformer_sparse_kmip_b200 import workloads as wl
from graph_transformer_sparse_kmip_b200.layer import KmipGlobalAttention, kmip_attention
from parity import TOL, check_selection, check_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    binding.load()
    return torch.device("cuda:0")


class _OracleAttention(torch.autograd.Function):
    """fp64 attention over fixed key sets, forward and backward by the oracle."""

    @staticmethod
    def forward(ctx, Q, K, V, idx, offsets, scale):
        r = oracle.given_idx(Q, K, V, idx, offsets, scale)
        ctx.save_for_backward(Q, K, V)
        ctx.idx, ctx.offsets, ctx.scale = idx, offsets, scale
        return torch.from_numpy(r["out"])

    @staticmethod
    def backward(ctx, dout):
        Q, K, V = ctx.saved_tensors
        r = oracle.given_idx(Q, K, V, ctx.idx, ctx.offsets, ctx.scale, dO=dout.contiguous())
        return (torch.from_numpy(r["dQ"]), torch.from_numpy(r["dK"]), torch.from_numpy(r["dV"]),
                None, None, None)


def test_global_attention_block_matches_fp64_reference(dev):
    sizes = [300, 45, 0, 517, 129]
    hidden, heads, k = 128, 4, 15
    gen = torch.Generator().manual_seed(31)
    N = sum(sizes)
    offsets = wl.offsets_from_sizes(sizes)
    torch.manual_seed(7)
    blk = KmipGlobalAttention(hidden, heads, k, dtype=torch.bfloat16, device=dev)
    x = torch.randn((N, hidden), generator=gen).to(torch.bfloat16).to(dev).requires_grad_(True)
    gy = torch.randn((N, hidden), generator=gen).to(torch.bfloat16).to(dev)
    y = blk(x, offsets.to(dev))
    y.backward(gy)
    torch.cuda.synchronize()
    binding.check_status()
    idx = blk.last_idx.cpu()

    # the selection on the GPU's own projected queries and keys
    with torch.no_grad():
        qkv = blk.qkv(x).view(N, 3, heads, hidden // heads).cpu()
    ref = oracle.fwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], offsets, k, blk.scale)
    check_selection(qkv[:, 0], qkv[:, 1], offsets, idx, ref)

    # fp64 reference of the whole block over the GPU-selected sets
    P = {n: p.detach().cpu().double().requires_grad_(True) for n, p in blk.named_parameters()}
    x64 = x.detach().cpu().double().requires_grad_(True)
    q64 = (x64 @ P["qkv.weight"].T + P["qkv.bias"]).view(N, 3, heads, hidden // heads)
    a64 = _OracleAttention.apply(q64[:, 0].contiguous(), q64[:, 1].contiguous(),
                                 q64[:, 2].contiguous(), idx.numpy(), offsets.numpy(), blk.scale)
    y64 = x64 + a64.reshape(N, hidden) @ P["proj.weight"].T + P["proj.bias"]
    y64.backward(gy.cpu().double())

    bf = torch.bfloat16
    check_values("y", y, y64.detach(), bf)
    check_values("dx", x.grad, x64.grad, bf)
    for n, p in blk.named_parameters():
        g, r = p.grad, P[n].grad
        if g.dim() == 1:
            g, r = g[None], r[None]
        check_values("d" + n, g, r, bf)


def test_kmip_attention_autograd_matches_c_abi(dev):
    inp = wl.random_case([400, 77], H=2, d=32, dtype="bf16", seed=12)
    g = {n: t.to(dev) for n, t in inp.items()}
    Q, K, V = (g[n].clone().requires_grad_(True) for n in ("Q", "K", "V"))
    out, idx = kmip_attention(Q, K, V, 15, 0.2, g["offsets"])
    out.backward(g["dO"])
    o2, i2, l2 = binding.attn_fwd(g["Q"], g["K"], g["V"], 15, 0.2, g["offsets"])
    dQ, dK, dV = binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], i2, l2, 0.2)
    assert torch.equal(idx, i2) and torch.equal(out, o2)
    # dK and dV are fp32 atomic sums (last bits vary run to run), then bf16
    for a, b in ((Q.grad, dQ), (K.grad, dK), (V.grad, dV)):
        assert a.dtype == torch.bfloat16
        np.testing.assert_allclose(a.float().cpu().numpy(), b.float().cpu().numpy(),
                                   rtol=1e-2, atol=1e-6)
