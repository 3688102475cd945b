"""The seeded input recipe (CPU): the five workloads' shapes, the clustered
generator's structure, and determinism of every draw."""

import math

import pytest
import torch

from lsh_bucketed_sparse_b200 import workloads as W


def test_five_workloads_have_the_stated_shapes_and_seeds():
    table = {
        # name: (B, H, L, d, dtype, n_h, n_b, c, causal, clustered)
        "small-fp32-L1024": (1, 1, 1024, 64, torch.float32, 1, 32, 64, False, False),
        "causal-bf16-4x8-L4096": (4, 8, 4096, 64, torch.bfloat16, 4, 64, 64, True, False),
        "image-bf16-1x8-L12288": (1, 8, 12288, 64, torch.bfloat16, 8, 192, 64, True, False),
        "longtext-bf16-1x8-L65536": (1, 8, 65536, 64, torch.bfloat16, 8, 1024, 64, True, False),
        "clustered-bf16-2x16-L16384-d128": (2, 16, 16384, 128, torch.bfloat16, 4, 256, 128,
                                            False, True),
    }
    assert [w.name for w in W.WORKLOADS] == list(table)
    for i, w in enumerate(W.WORKLOADS):
        got = (w.batch, w.heads, w.seq_len, w.d_k, w.dtype, w.n_hashes, w.n_buckets,
               w.chunk_len, w.causal, w.clustered)
        assert got == table[w.name], w.name
        assert w.seed == 1000 + i + 1
        assert w.seq_len % w.chunk_len == 0 and w.n_buckets % 2 == 0
    assert W.HEADLINE.name == "longtext-bf16-1x8-L65536"


@pytest.mark.parametrize("total,n,s", [(16384, 256, 1.2), (1000, 7, 1.0), (5, 8, 2.0)])
def test_zipf_sizes_sum_to_total_and_follow_the_power_law(total, n, s):
    sizes = W.zipf_sizes(total, n, s)
    assert len(sizes) == n and sum(sizes) == total and min(sizes) >= 0
    tot_w = sum(k ** (-s) for k in range(1, n + 1))
    for k, size in enumerate(sizes, start=1):
        assert abs(size - total * k ** (-s) / tot_w) < 1.0  # largest remainder: off by < 1
    assert sizes == sorted(sizes, reverse=True)


def test_largest_cluster_of_the_clustered_workload():
    wl = W.BY_NAME["clustered-bf16-2x16-L16384-d128"]
    sizes = W.zipf_sizes(wl.seq_len, wl.n_clusters, wl.zipf_s)
    assert 4000 <= sizes[0] <= 4200  # about a quarter of the tokens in one cluster


def test_clustered_members_sit_around_their_centres_and_are_shuffled():
    wl = W.BY_NAME["clustered-bf16-2x16-L16384-d128"].with_(
        batch=1, heads=2, seq_len=2048, n_clusters=16, dtype=torch.float32)
    gen = torch.Generator().manual_seed(5)
    qk = W.clustered_qk(wl, gen)
    sizes = W.zipf_sizes(wl.seq_len, wl.n_clusters, wl.zipf_s)
    for h in range(wl.heads):
        x = qk[0, h]
        # every point's nearest other point is within a few sigma (it has
        # cluster mates), and the distinct cluster centres are far apart
        d2 = torch.cdist(x, x)
        d2.fill_diagonal_(float("inf"))
        assert d2.min(dim=1).values.max() < 8 * wl.cluster_sigma * math.sqrt(wl.d_k)
        # grouping points by proximity recovers the Zipf sizes
        labels = torch.full((wl.seq_len,), -1)
        found = []
        for i in range(wl.seq_len):
            if labels[i] >= 0:
                continue
            near = (torch.cdist(x[i:i + 1], x)[0] < 12 * wl.cluster_sigma * math.sqrt(wl.d_k))
            labels[near] = len(found)
            found.append(int(near.sum()))
        assert sorted(found, reverse=True) == sizes
        # positions are shuffled: members of the largest cluster are spread out
        big = (labels == labels[torch.argmax(torch.bincount(labels))]).nonzero()[:, 0]
        assert big.max() - big.min() > wl.seq_len // 2


def test_inputs_are_deterministic_and_well_formed():
    wl = W.small("det", batch=2, heads=3, seq_len=128, n_hashes=3, n_buckets=10)
    a = W.make_inputs(wl)
    b = W.make_inputs(wl)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and x.is_contiguous() and x.dtype == wl.dtype
    qk, v, rot = a
    assert qk.shape == v.shape == (2, 3, 128, 64) and rot.shape == (3, 64, 5)
    assert not torch.equal(qk, v)
    c = W.make_inputs(wl, seed=wl.seed + 1)
    assert not torch.equal(a[0], c[0])
    one = W.make_inputs(W.small("one", n_buckets=1))
    assert one[2] is None


def test_centroids_and_upstream_use_their_own_generators():
    wl = W.small("own", n_hashes=2, n_buckets=12)
    before = W.make_inputs(wl)
    cen = W.make_centroids(wl)
    g = W.make_upstream(wl)
    after = W.make_inputs(wl)
    for x, y in zip(before, after):
        assert torch.equal(x, y)
    assert cen.shape == (2, 64, 12) and g.shape == before[0].shape
    assert not torch.equal(cen[:, :, :6], before[2])
