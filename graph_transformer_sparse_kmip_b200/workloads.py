"""Seeded synthetic inputs shaped like the workloads the k-MIP pages measure.

Only random-number generation and shape bookkeeping live here -- none of the
method's arithmetic -- so the CUDA path and the fp64 oracle can both be fed
from it.  Everything is drawn on the CPU with ``torch.Generator`` in fp32 and
then rounded to the working dtype (round-to-nearest-even for bf16), so a
given seed always yields the same bits.

The pages' datasets (LRGB superpixels, City-Networks, ShapeNet-Part, S3DIS;
k-Maximum Inner Product Attention for Graph Transformers and the Expressive
Power of GraphGPS, Tables 2, 3, 8, 13) are not available; these inputs stand
in for them with the node counts, batching structure and head shapes the
pages describe.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    d: int
    k: int
    dtype: str                      # "bf16" | "f32"
    phases: str                     # "fwd" | "fwd+bwd"
    N: int = 0                      # single graph size (when sizes_range is None)
    sizes_range: tuple | None = None  # per-graph node counts drawn uniformly from this range
    G: int = 1
    values: str = "normal"          # "normal" | "gmm_keys" | "pointcloud"
    seed: int = 0
    k_sweep: tuple = field(default=())

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# Workloads, named for what they are.  The node counts and batching follow the
# pages: one graph of 10^3 nodes class (tiny check case), batched
# superpixel-like graphs of a few hundred nodes (Tables 8/9, LRGB), a single
# graph at N = 10^4.5 (the training-setting timings of Tables 10-12, 16),
# N = 10^5 where full attention runs out of memory (Figure 2), with the k
# range of the hyper-parameter tables (Tables 5/6: k in {5, 15, 45}), and a
# point-cloud-scale graph of over 500k nodes (Abstract).
WORKLOADS = {
    "tiny_n1024_f32": Workload("tiny_n1024_f32", H=1, d=32, k=15, dtype="f32", phases="fwd",
                               N=1024),
    "batched64_n300to600": Workload("batched64_n300to600", H=4, d=32, k=15, dtype="bf16",
                                    phases="fwd+bwd", G=64, sizes_range=(300, 600)),
    "graph_n31623": Workload("graph_n31623", H=4, d=32, k=15, dtype="bf16", phases="fwd+bwd",
                             N=31623),
    "gmm_n100000": Workload("gmm_n100000", H=4, d=32, k=15, dtype="bf16", phases="fwd+bwd",
                            N=100000, values="gmm_keys", k_sweep=(5, 15, 45)),
    "pointcloud_n524288": Workload("pointcloud_n524288", H=4, d=16, k=15, dtype="bf16",
                                   phases="fwd", N=524288, values="pointcloud"),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def graph_sizes(w: Workload) -> list[int]:
    """Per-graph node counts (uniform integers in sizes_range, inclusive)."""
    if w.sizes_range is None:
        return [w.N]
    g = torch.Generator().manual_seed(w.seed)
    lo, hi = w.sizes_range
    return torch.randint(lo, hi + 1, (w.G,), generator=g).tolist()


def offsets_from_sizes(sizes) -> torch.Tensor:
    off = [0]
    for s in sizes:
        off.append(off[-1] + int(s))
    return torch.tensor(off, dtype=torch.int32)


def _normal(shape, gen) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def make_inputs(w: Workload, with_grad_out: bool | None = None, seed: int | None = None):
    """Return dict(Q, K, V, offsets, [dO]) as CPU tensors of the workload dtype.

    Q, K, V, dO are [N, H, d]; offsets is int32 [G+1].  dO is drawn from
    seed + 1.  Value recipes:
      normal     -- Q, K, V i.i.d. N(0, 1);
      gmm_keys   -- Q, V ~ N(0, 1); key of node j in head h is
                    c[h, m_j] + 0.3 * eps, centres c ~ N(0, I_d) (64 per head),
                    m_j uniform over the 64 components (shared by all heads);
      pointcloud -- P ~ U[0, 1]^3 per node; for X in (Q, K, V) and head h,
                    X[:, h] = P @ W_{X,h} + 0.1 * eps with W ~ N(0, 1) of
                    shape 3 x d (a random linear projection plus noise).
    """
    seed = w.seed if seed is None else seed
    sizes = graph_sizes(w)
    N = sum(sizes)
    H, d = w.H, w.d
    gen = torch.Generator().manual_seed(seed + 1000)
    if w.values == "normal":
        Q = _normal((N, H, d), gen)
        K = _normal((N, H, d), gen)
        V = _normal((N, H, d), gen)
    elif w.values == "gmm_keys":
        Q = _normal((N, H, d), gen)
        V = _normal((N, H, d), gen)
        centres = _normal((H, 64, d), gen)
        comp = torch.randint(0, 64, (N,), generator=gen)
        K = centres[:, comp, :].permute(1, 0, 2).contiguous() + 0.3 * _normal((N, H, d), gen)
    elif w.values == "pointcloud":
        P = torch.rand((N, 3), generator=gen, dtype=torch.float32)
        mats = []
        for _ in range(3):
            W = _normal((H, 3, d), gen)
            X = torch.einsum("nc,hcd->nhd", P, W) + 0.1 * _normal((N, H, d), gen)
            mats.append(X.contiguous())
        Q, K, V = mats
    else:
        raise ValueError(w.values)
    dt = torch_dtype(w.dtype)
    res = dict(Q=Q.to(dt), K=K.to(dt), V=V.to(dt), offsets=offsets_from_sizes(sizes))
    if with_grad_out is None:
        with_grad_out = "bwd" in w.phases
    if with_grad_out:
        g2 = torch.Generator().manual_seed(seed + 1)
        res["dO"] = _normal((N, H, d), g2).to(dt)
    return res


def random_case(N_sizes, H: int, d: int, dtype: str = "bf16", seed: int = 0,
                values: str = "normal", with_grad_out: bool = True):
    """Small ad-hoc case: graphs of the given node counts, N(0,1) values."""
    if values != "normal":
        raise ValueError(values)
    sizes = list(N_sizes)
    N = sum(sizes)
    gen = torch.Generator().manual_seed(seed + 1000)
    Q = _normal((N, H, d), gen)
    K = _normal((N, H, d), gen)
    V = _normal((N, H, d), gen)
    dt = torch_dtype(dtype)
    res = dict(Q=Q.to(dt), K=K.to(dt), V=V.to(dt), offsets=offsets_from_sizes(sizes))
    if with_grad_out:
        g2 = torch.Generator().manual_seed(seed + 1)
        res["dO"] = _normal((N, H, d), g2).to(dt)
    return res


def sample_pairs(N: int, H: int, n: int, seed: int = 12345):
    """Seeded sample of (query, head) pairs without replacement."""
    g = torch.Generator().manual_seed(seed)
    total = N * H
    n = min(n, total)
    flat = torch.randperm(total, generator=g)[:n].sort().values
    return (flat // H).to(torch.int64), (flat % H).to(torch.int32)
