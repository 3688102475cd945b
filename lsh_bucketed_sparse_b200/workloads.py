"""Seeded synthetic inputs for the LSH attention forward pass.

This module only draws random numbers and names workload shapes.  It holds
none of the method's arithmetic (no hashing, sorting, masking or softmax), so
both the CUDA path and the fp64 oracle can be fed from it without sharing any
part of the computation.

Recipe (same for every workload): a CPU ``torch.Generator`` seeded with
``1000 + index`` draws, in this order, ``qk`` then ``v`` then the rotations,
each as float32 N(0, 1), and the result is cast to the workload's dtype.
The rotations have shape ``[n_hashes, d_k, n_buckets // 2]``: one random
projection matrix per hashing round, shared by every (batch, head), as in the
random-projection hash h(x) = argmax([xR; -xR]) ("Reformer: The Efficient
Transformer", section 2).

The clustered workload replaces the N(0, 1) ``qk`` with points around 256
centres so that the buckets are highly skewed (see ``clustered_qk``).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    seq_len: int
    d_k: int
    n_hashes: int
    n_buckets: int
    chunk_len: int
    causal: bool
    dtype: torch.dtype
    seed: int
    clustered: bool = False
    n_clusters: int = 256
    cluster_sigma: float = 0.05
    zipf_s: float = 1.2

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "batch": self.batch,
            "heads": self.heads,
            "seq_len": self.seq_len,
            "d_k": self.d_k,
            "n_hashes": self.n_hashes,
            "n_buckets": self.n_buckets,
            "chunk_len": self.chunk_len,
            "causal": self.causal,
            "dtype": "f32" if self.dtype == torch.float32 else "bf16",
            "inputs": "clustered" if self.clustered else "normal",
        }


# The five workloads, in order.  Index i (0-based) is seeded with 1000 + i + 1.
WORKLOADS = (
    Workload("small-fp32-L1024", 1, 1, 1024, 64, 1, 32, 64, False, torch.float32, 1001),
    Workload("causal-bf16-4x8-L4096", 4, 8, 4096, 64, 4, 64, 64, True, torch.bfloat16, 1002),
    Workload("image-bf16-1x8-L12288", 1, 8, 12288, 64, 8, 192, 64, True, torch.bfloat16, 1003),
    Workload("longtext-bf16-1x8-L65536", 1, 8, 65536, 64, 8, 1024, 64, True, torch.bfloat16, 1004),
    Workload("clustered-bf16-2x16-L16384-d128", 2, 16, 16384, 128, 4, 256, 128, False,
             torch.bfloat16, 1005, clustered=True),
)

BY_NAME = {w.name: w for w in WORKLOADS}

# The long-text shape (L = 65536, 8 hashes) is the headline workload.
HEADLINE = WORKLOADS[3]


def zipf_sizes(total: int, n: int, s: float) -> list:
    """Split ``total`` into ``n`` sizes proportional to k^-s (k = 1..n),
    rounding by largest remainder so that the sizes sum to ``total``."""
    w = [k ** (-s) for k in range(1, n + 1)]
    tot_w = sum(w)
    raw = [total * x / tot_w for x in w]
    base = [int(r) for r in raw]
    rem = total - sum(base)
    order = sorted(range(n), key=lambda k: (-(raw[k] - base[k]), k))
    for k in order[:rem]:
        base[k] += 1
    return base


def clustered_qk(wl: Workload, gen: torch.Generator) -> torch.Tensor:
    """qk drawn as ``n_clusters`` Gaussian clusters per (batch, head):
    centres ~ N(0, 1), members = centre + sigma * N(0, 1), cluster sizes
    Zipf(s) normalised to L by largest remainder, then the positions are
    shuffled with the same generator."""
    B, H, L, d = wl.batch, wl.heads, wl.seq_len, wl.d_k
    sizes = zipf_sizes(L, wl.n_clusters, wl.zipf_s)
    label = torch.repeat_interleave(torch.arange(wl.n_clusters), torch.tensor(sizes))
    out = torch.empty(B, H, L, d, dtype=torch.float32)
    for b in range(B):
        for h in range(H):
            centres = torch.randn(wl.n_clusters, d, generator=gen, dtype=torch.float32)
            noise = torch.randn(L, d, generator=gen, dtype=torch.float32)
            shuffle = torch.randperm(L, generator=gen)
            out[b, h] = (centres[label] + wl.cluster_sigma * noise)[shuffle]
    return out


def make_inputs(wl: Workload, seed: Optional[int] = None):
    """Return host tensors (qk, v, rotations) for a workload.

    qk, v: [batch, heads, seq_len, d_k]; rotations: [n_hashes, d_k, n_buckets // 2]
    (``None`` when n_buckets == 1, the one-bucket case that needs no hash).
    All are contiguous CPU tensors in ``wl.dtype``.
    """
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    shape = (wl.batch, wl.heads, wl.seq_len, wl.d_k)
    if wl.clustered:
        qk = clustered_qk(wl, gen)
    else:
        qk = torch.randn(*shape, generator=gen, dtype=torch.float32)
    v = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if wl.n_buckets >= 2:
        rot = torch.randn(wl.n_hashes, wl.d_k, wl.n_buckets // 2, generator=gen,
                          dtype=torch.float32)
        rot = rot.to(wl.dtype).contiguous()
    else:
        rot = None
    return qk.to(wl.dtype).contiguous(), v.to(wl.dtype).contiguous(), rot


def make_centroids(wl: Workload, seed: Optional[int] = None):
    """Centroids [n_hashes, d_k, n_buckets] for the routing-style assignment:
    float32 N(0, 1) from their own generator (seed + 10000, so qk, v and the
    rotations of make_inputs are unchanged), cast to ``wl.dtype``."""
    gen = torch.Generator().manual_seed((wl.seed if seed is None else seed) + 10000)
    c = torch.randn(wl.n_hashes, wl.d_k, wl.n_buckets, generator=gen, dtype=torch.float32)
    return c.to(wl.dtype).contiguous()


def make_upstream(wl: Workload, seed: Optional[int] = None):
    """An upstream gradient dout [batch, heads, seq_len, d_k] for the backward
    pass: float32 N(0, 1) from its own generator (seed + 20000), cast to
    ``wl.dtype``."""
    gen = torch.Generator().manual_seed((wl.seed if seed is None else seed) + 20000)
    g = torch.randn(wl.batch, wl.heads, wl.seq_len, wl.d_k, generator=gen, dtype=torch.float32)
    return g.to(wl.dtype).contiguous()


def small(name="tiny", batch=1, heads=2, seq_len=256, d_k=64, n_hashes=2, n_buckets=16,
          chunk_len=64, causal=True, dtype=torch.bfloat16, seed=7, clustered=False,
          n_clusters=16) -> Workload:
    """A small workload for parity tests (oracle finishes in well under a second)."""
    return Workload(name, batch, heads, seq_len, d_k, n_hashes, n_buckets, chunk_len, causal,
                    dtype, seed, clustered=clustered, n_clusters=n_clusters)
