"""The global-attention block of a GraphGPS layer with k-MIP attention.

k-Maximum Inner Product Attention for Graph Transformers and the Expressive
Power of GraphGPS (Figure 1: one GraphGPS layer, whose global-attention
branch is where k-MIP attention replaces full attention): node features x
[N, hidden] are projected to queries, keys and values of H heads of width d
(hidden = H d), every query attends over its k best keys of its own graph,
and the heads are projected back and added to the input:

    [Q | K | V] = x W_qkv + b_qkv            one GEMM, [N, 3 H d]
    A           = kmip_attention(Q, K, V)    libkmip (C ABI), [N, H, d]
    y           = x + A W_o + b_o

The projections are plain GEMMs (torch / cuBLAS); the attention forward and
backward run in libkmip's kernels through the ctypes binding, and the block
is trainable through torch autograd.  The MPNN branch and the feed-forward
part of a GraphGPS layer are not part of this block.
"""
from __future__ import annotations

import math

import torch

from . import binding


class KmipAttentionFunction(torch.autograd.Function):
    """Autograd wrapper of kmip_attn_fwd / kmip_attn_bwd.

    Q, K, V: [N, H, d] CUDA tensors (bf16 or fp32); offsets: int32 [G+1]
    CUDA tensor or None.  Returns out [N, H, d] in the input dtype; the
    selection (idx) gets no gradient.  Gradients come back in the input
    dtype (the library computes them in fp32)."""

    @staticmethod
    def forward(ctx, Q, K, V, offsets, k: int, scale: float):
        Q, K, V = Q.contiguous(), K.contiguous(), V.contiguous()
        out, idx, lse = binding.attn_fwd(Q, K, V, k, scale, offsets)
        ctx.save_for_backward(Q, K, V, idx, lse)
        ctx.scale = scale
        ctx.mark_non_differentiable(idx)
        return out, idx

    @staticmethod
    def backward(ctx, dout, _didx):
        Q, K, V, idx, lse = ctx.saved_tensors
        dQ, dK, dV = binding.attn_bwd(dout.contiguous().to(Q.dtype), Q, K, V, idx, lse,
                                      ctx.scale)
        return dQ.to(Q.dtype), dK.to(K.dtype), dV.to(V.dtype), None, None, None


def kmip_attention(Q, K, V, k: int, scale: float | None = None, offsets=None):
    """k-MIP attention with autograd; returns (out [N, H, d], idx [N, H, k])."""
    if scale is None:
        scale = 1.0 / math.sqrt(Q.shape[-1])
    return KmipAttentionFunction.apply(Q, K, V, offsets, int(k), float(scale))


class KmipGlobalAttention(torch.nn.Module):
    """GraphGPS global-attention block: fused QKV projection, k-MIP
    attention, output projection and residual (see the module docstring)."""

    def __init__(self, hidden: int, heads: int, k: int, dtype=torch.bfloat16, device=None):
        super().__init__()
        if hidden % heads:
            raise ValueError("hidden must be a multiple of heads")
        self.hidden, self.heads, self.d, self.k = hidden, heads, hidden // heads, k
        self.scale = 1.0 / math.sqrt(self.d)
        self.qkv = torch.nn.Linear(hidden, 3 * hidden, dtype=dtype, device=device)
        self.proj = torch.nn.Linear(hidden, hidden, dtype=dtype, device=device)

    def forward(self, x, offsets=None):
        N = x.shape[0]
        qkv = self.qkv(x).view(N, 3, self.heads, self.d)
        a, idx = kmip_attention(qkv[:, 0], qkv[:, 1], qkv[:, 2], self.k, self.scale, offsets)
        self.last_idx = idx
        return x + self.proj(a.reshape(N, self.hidden))
