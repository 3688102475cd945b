"""The sort stage alone against the oracle's stable sort, bit for bit.

Bucket ids are drawn directly (no hash) so that the bucket count can range
from one bucket to 32768 (one to fifteen bits of bucket id for
the warp ranking, both scatter kernels), with ragged lengths (the last tile
of 2048 keys short) and skewed distributions (most keys in one bucket, as
clustered inputs give).
"""
import numpy as np
import pytest
import torch

import lsh_bucketed_sparse_b200 as lsh
from oracle import lsh_oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _buckets(n_b, L, n_h, skew, seed):
    rng = np.random.default_rng(seed)
    b = rng.integers(0, n_b, size=(1, 1, n_h, L))
    if skew:
        # 90% of the keys in one bucket, the rest spread
        hot = rng.random((1, 1, n_h, L)) < 0.9
        b = np.where(hot, n_b - 1, b)
    return b.astype(np.int16)


# bucket counts the shape allows: 1 or even, up to 32768
@pytest.mark.parametrize("n_b", [1, 2, 4, 62, 192, 194, 1024, 4096, 32768])
@pytest.mark.parametrize("L,skew", [(5000, False), (2049, True), (4096, False)],
                         ids=["ragged", "skewed-ragged", "whole-tiles"])
def test_sort_matches_stable_sort(n_b, L, skew):
    n_h = 3
    b = _buckets(n_b, L, n_h, skew, seed=n_b * 7 + L)
    perm, undo, counts = lsh.lsh_attn_sort(torch.from_numpy(b).to(DEV), n_b, want_counts=True)
    want_perm, want_undo = O.sort_head(b[0, 0].astype(np.int64))
    np.testing.assert_array_equal(perm.cpu().numpy()[0, 0], want_perm)
    np.testing.assert_array_equal(undo.cpu().numpy()[0, 0], want_undo)
    want_counts = np.stack([np.bincount(b[0, 0, r], minlength=n_b) for r in range(n_h)])
    np.testing.assert_array_equal(counts.cpu().numpy()[0, 0], want_counts)
