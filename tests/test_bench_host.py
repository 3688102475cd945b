"""Host-side pieces of bench.py that need no GPU: the CPU baseline's sample
accounting and the window-pair count behind the backward's roofline."""

import pytest

import bench
from lsh_bucketed_sparse_b200 import workloads as W


def test_cpu_baseline_scales_its_sample_to_the_whole_workload():
    wl = W.small("sample", batch=2, heads=2, seq_len=256, n_hashes=4, n_buckets=16)
    # 3 of the 4 (batch, head) pairs, every round: three quarters of the work
    dt, toks = bench.oracle_sample(wl, rounds=8, heads=3)
    assert dt > 0 and toks == pytest.approx(0.75 * wl.batch * wl.seq_len)
    # one pair, one round: a sixteenth
    _, toks = bench.oracle_sample(wl, rounds=1, heads=1)
    assert toks == pytest.approx(wl.batch * wl.seq_len / 16)
    line = bench.cpu_baseline(wl, 2, 1)
    assert line["kind"] == "oracle" and line["cores"] >= 1 and line["value"] > 0
    assert "1 of 4 (batch, head) pairs" in line["sample"] and "2 of 4 hashing" in line["sample"]


@pytest.mark.parametrize("L,c", [(256, 64), (100, 64), (40, 64), (1000, 48)])
def test_window_pairs_counts_every_query_key_pair(L, c):
    wl = W.small("pairs", batch=1, heads=3, seq_len=L, n_hashes=2, chunk_len=c)
    brute = 0
    for s in range(L):          # query slot s in chunk k sees chunks k-1 and k
        k = s // c
        lo = (k - 1) * c if k > 0 else 0
        brute += min((k + 1) * c, L) - lo
    assert bench.window_pairs(wl) == brute * 3 * 2
