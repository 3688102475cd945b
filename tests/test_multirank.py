"""The multi-rank path on CPU: world-size-2 gloo ranks.

(batch, head) pairs are independent, so each rank runs the unchanged pass on
its own range of pairs and no data-path collective exists.  Here each rank
runs the fp64 oracle on its range (standing in for the GPU pass) and the
pieces, gathered only to check them, must equal a single-process run; the
max-over-ranks timing reduction of the benchmark is checked too.
"""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lsh_bucketed_sparse_b200 import sharding
from lsh_bucketed_sparse_b200 import workloads as W


def test_head_range_partitions():
    for total_b, total_h in [(1, 8), (2, 16), (3, 5), (1, 1)]:
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = sharding.head_range(total_b, total_h, r, world)
                assert 0 <= a <= b <= total_b * total_h
                seen.extend(range(a, b))
            assert seen == list(range(total_b * total_h))
    with pytest.raises(ValueError):
        sharding.head_range(1, 8, 2, 2)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import lsh_oracle as O
        wl = W.small("mr", batch=2, heads=3, seq_len=256, n_hashes=2, n_buckets=16)
        qk, v, rot = W.make_inputs(wl)
        lq = sharding.local_slice(qk, wl.batch, wl.heads, rank, world)
        lv = sharding.local_slice(v, wl.batch, wl.heads, rank, world)
        res = O.forward(lq, lv, rot, wl.n_buckets, wl.chunk_len, wl.causal)
        out = torch.from_numpy(res["out"][0])
        # gather only to check (the pass itself needs no collective)
        sizes = [sharding.head_range(wl.batch, wl.heads, r, world) for r in range(world)]
        n_max = max(b - a for a, b in sizes)
        pad = torch.zeros(n_max, *out.shape[1:], dtype=out.dtype)
        pad[: out.shape[0]] = out
        got = [torch.zeros_like(pad) for _ in range(world)]
        dist.all_gather(got, pad)
        # the benchmark's timing: max over ranks
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            pieces = [g[: b - a] for g, (a, b) in zip(got, sizes)]
            q.put((torch.cat(pieces).numpy(), float(t.item())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_one_process():
    from oracle import lsh_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    joined, tmax = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = W.small("mr", batch=2, heads=3, seq_len=256, n_hashes=2, n_buckets=16)
    qk, v, rot = W.make_inputs(wl)
    full = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal)["out"]
    np.testing.assert_allclose(joined, full.reshape(-1, *full.shape[2:]), rtol=0, atol=0)
    assert tmax == 2.0
