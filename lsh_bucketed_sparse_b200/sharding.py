"""Splitting the forward pass over ranks (one process per GPU).

Hashing, sorting, the chunk windows and the combine never cross (batch, head)
pairs, so the pairs are independent problems: each rank takes a contiguous
range of the flattened B*H pairs and runs the unchanged single-GPU pass on
it.  No collective is needed on the data path; outputs stay on the rank that
owns the pairs.
"""

from __future__ import annotations


def head_range(batch: int, heads: int, rank: int, world: int):
    """[start, stop) of the flattened (batch, head) pairs owned by `rank`.

    The first (B*H) % world ranks take one pair more; every pair belongs to
    exactly one rank.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    total = batch * heads
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def local_slice(t, batch: int, heads: int, rank: int, world: int):
    """The rank's pairs of a [B, H, ...] tensor, as a [1, n, ...] view."""
    start, stop = head_range(batch, heads, rank, world)
    flat = t.reshape(batch * heads, *t.shape[2:])
    return flat[start:stop].unsqueeze(0)


def forward_local(qk, v, rotations, n_hashes, n_buckets, chunk_len, causal, rank, world, **kw):
    """Run lsh_attn_forward on this rank's (batch, head) pairs of full
    [B, H, L, d] tensors (present on every rank); returns that slice's
    (out, lse) as [1, n, L, d] and [1, n, L]."""
    from . import lsh_attn_forward
    B, H = qk.shape[:2]
    q = local_slice(qk, B, H, rank, world).contiguous()
    vv = local_slice(v, B, H, rank, world).contiguous()
    return lsh_attn_forward(q, vv, rotations, n_hashes, n_buckets, chunk_len, causal, **kw)
