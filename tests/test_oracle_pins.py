"""Pins for the fp64 oracle against what the pages and mathematics fix.

None of these re-types the oracle's own formulas: each check comes from a
hand-worked example, a special case that reduces to a textbook routine
(torch's scaled_dot_product_attention in float64), a closed form computed a
different way (window membership counts instead of per-round softmax plus
combine), an invariant, or brute force written from the set definitions.
"""

import json
import math
import os
import random

import numpy as np
import pytest
import torch

from oracle import lsh_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- hash ----
def test_hash_golden_tiny():
    g = _load("hash_tiny.json")
    x = np.array(g["x"])
    R = np.array(g["rotations"])
    b, m = O.hash_head(x, R, g["n_buckets"])
    assert b.tolist() == g["buckets"]
    np.testing.assert_array_equal(m, np.array(g["margins"]))
    perm, undo = O.sort_head(b)
    assert perm.tolist() == g["perm"]
    assert undo.tolist() == g["undo"]


def test_hash_two_buckets_is_sign():
    # n_buckets = 2: z = [p, -p], so the bucket is 0 when x.R >= 0 and 1 otherwise.
    rng = np.random.default_rng(1)
    x = rng.standard_normal((200, 8))
    R = rng.standard_normal((3, 8, 1))
    b, _ = O.hash_head(x, R, 2)
    for r in range(3):
        for i in range(200):
            dot = sum(float(x[i, k]) * float(R[r, k, 0]) for k in range(8))
            assert b[r, i] == (0 if dot >= 0 else 1)


def test_hash_brute_force_loops():
    # Argmax over [xR; -xR] by explicit loops, lowest index on ties.
    rng = np.random.default_rng(2)
    d, half, n_h, L = 5, 6, 2, 40
    x = rng.standard_normal((L, d))
    R = rng.standard_normal((n_h, d, half))
    x[3] = 0.0  # all projections zero: every z entry ties, bucket 0
    b, _ = O.hash_head(x, R, 2 * half)
    for r in range(n_h):
        for i in range(L):
            z = []
            for j in range(half):
                z.append(sum(x[i, k] * R[r, k, j] for k in range(d)))
            z = z + [-t for t in z]
            best = 0
            for j in range(1, len(z)):
                if z[j] > z[best]:
                    best = j
            assert b[r, i] == best
    assert (b[:, 3] == 0).all()


def test_hash_tie_rule_duplicate_columns():
    # Two equal columns of R make p_0 == p_1 exactly: the lower index wins,
    # in the positive half and in the negative half.
    R = np.zeros((1, 2, 3))
    R[0, :, 0] = R[0, :, 1] = [1.0, 0.5]
    R[0, :, 2] = [0.1, 0.1]
    x = np.array([[2.0, 0.0], [-2.0, 0.0]])
    b, m = O.hash_head(x, R, 6)
    assert b[0].tolist() == [0, 3]
    assert m[0].tolist() == [0.0, 0.0]


@pytest.mark.parametrize("k", [-3, 1, 5])
def test_hash_power_of_two_rescale_is_exact(k):
    # A positive rescale changes no argmax; by 2**k it is exact in floating point.
    rng = np.random.default_rng(3)
    x = rng.standard_normal((500, 16))
    R = rng.standard_normal((4, 16, 8))
    b0, m0 = O.hash_head(x, R, 16)
    b1, m1 = O.hash_head(x * 2.0 ** k, R, 16)
    np.testing.assert_array_equal(b0, b1)
    np.testing.assert_array_equal(m0 * 2.0 ** k, m1)


def test_hash_general_rescale_away_from_ties():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2000, 16))
    R = rng.standard_normal((2, 16, 16))
    b0, m0 = O.hash_head(x, R, 32)
    b1, _ = O.hash_head(x * 3.7, R, 32)
    safe = m0 > 1e-9
    assert safe.mean() > 0.99
    np.testing.assert_array_equal(b0[safe], b1[safe])


def test_hash_bucket_frequencies_follow_symmetry():
    # N(0, 1) points are rotation invariant: with orthonormal columns of R all
    # n_b buckets are equally likely (chi^2 sanity, 15 dof); with any R the
    # map x -> -x swaps bucket j and j + n_b/2, so those pairs are equally likely.
    rng = np.random.default_rng(5)
    x = rng.standard_normal((40000, 32))
    q, _ = np.linalg.qr(rng.standard_normal((32, 8)))
    b, _ = O.hash_head(x, q[None], 16)
    counts = np.bincount(b[0], minlength=16)
    exp = 40000 / 16
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 45.0, (chi2, counts)
    b2, _ = O.hash_head(x, rng.standard_normal((1, 32, 8)), 16)
    c2 = np.bincount(b2[0], minlength=16)
    pair = (c2[:8] - c2[8:]) ** 2 / (c2[:8] + c2[8:])
    assert float(pair.sum()) < 30.0, c2
    bneg, _ = O.hash_head(-x, q[None], 16)
    np.testing.assert_array_equal((b[0] + 8) % 16, bneg[0])


def test_hash_one_bucket():
    b, m = O.hash_head(np.ones((10, 4)), None, 1)
    assert (b == 0).all() and np.isinf(m).all()


# ---------------------------------------------------------------- sort ----
def test_sort_matches_tuple_sort_and_invariants():
    rng = np.random.default_rng(6)
    b = rng.integers(0, 7, size=(3, 300))
    perm, undo = O.sort_head(b)
    for r in range(3):
        expect = sorted(range(300), key=lambda i: (int(b[r, i]), i))
        assert perm[r].tolist() == expect
        assert sorted(perm[r].tolist()) == list(range(300))
        keys = [(int(b[r, p]), int(p)) for p in perm[r]]
        assert keys == sorted(keys)
        assert (undo[r][perm[r]] == np.arange(300)).all()


# ------------------------------------------------------ attention tiny ----
def test_attention_golden_tiny():
    g = _load("attention_tiny.json")
    for case in g["cases"]:
        x = np.array(case["x"])[None, None]
        v = np.array(case["v"])[None, None]
        L = x.shape[2]
        buckets = np.zeros((1, 1, case["n_hashes"], L), np.int64)
        res = O.forward(x, v, None, 1, case["chunk_len"], case["causal"], buckets=buckets)
        np.testing.assert_allclose(res["out"][0, 0], np.array(case["out"]), rtol=1e-10, atol=1e-12,
                                   err_msg=case["name"])
        np.testing.assert_allclose(res["lse"][0, 0], np.array(case["lse"]), rtol=1e-15, atol=1e-12,
                                   err_msg=case["name"])


# -------------------------------------------- full attention limit (a) ----
def _sdpa_reference(x, v, causal):
    """Textbook shared-QK attention: torch SDPA (float64) with the self score
    set to -1e5 through the additive mask and the causal mask as -inf."""
    L, d = x.shape
    xt = torch.from_numpy(x)
    norms = torch.linalg.vector_norm(xt, dim=1)
    k = xt / norms[:, None]
    mask = torch.zeros(L, L, dtype=torch.float64)
    # the diagonal score x_i . x_i/||x_i|| / sqrt(d) = ||x_i|| / sqrt(d) becomes -1e5
    mask[range(L), range(L)] = O.SELF_SCORE - norms / math.sqrt(d)
    if causal:
        mask = mask.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    out = torch.nn.functional.scaled_dot_product_attention(
        xt[None], k[None], torch.from_numpy(v)[None], attn_mask=mask)[0]
    scores = (xt @ k.T) / math.sqrt(d) + mask
    lse = torch.logsumexp(scores, dim=1)
    return out.numpy(), lse.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_buckets,n_hashes", [(1, 1), (1, 3), (2, 2)])
def test_full_attention_limit(causal, n_buckets, n_hashes):
    rng = np.random.default_rng(7)
    L, d = 96, 16
    x = rng.standard_normal((1, 2, L, d))
    v = rng.standard_normal((1, 2, L, d))
    R = rng.standard_normal((n_hashes, d, 1)) if n_buckets == 2 else None
    if n_buckets == 1:
        buckets = np.zeros((1, 2, n_hashes, L), np.int64)
        res = O.forward(x, v, None, 1, L, causal, buckets=buckets)
    else:
        res = O.forward(x, v, R, 2, L, causal)
    for h in range(2):
        ref_out, ref_lse = _sdpa_reference(x[0, h], v[0, h], causal)
        np.testing.assert_allclose(res["out"][0, h], ref_out, rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(res["lse"][0, h], ref_lse + math.log(n_hashes), rtol=1e-12,
                                   atol=1e-9)


# ------------------------------------------------- brute force (c) --------
def _brute_force(x, v, buckets, c, causal):
    """Windows enumerated from the set definitions, per-round softmax by loops."""
    n_h, L = buckets.shape
    d = x.shape[1]
    khat = [x[j] / math.sqrt(sum(t * t for t in x[j])) for j in range(L)]
    out = np.zeros((L, d))
    lse = np.zeros(L)
    for i in range(L):
        lses, outs = [], []
        for r in range(n_h):
            order = sorted(range(L), key=lambda j: (buckets[r, j], j))
            slot = order.index(i)
            k = slot // c
            chunks = {k, k - 1} if k > 0 else {k}
            window = [order[s] for s in range(L) if s // c in chunks]
            sc = {}
            for j in window:
                if causal and j > i:
                    continue
                sc[j] = O.SELF_SCORE if j == i else \
                    sum(x[i, t] * khat[j][t] for t in range(d)) / math.sqrt(d)
            mx = max(sc.values())
            den = sum(math.exp(s - mx) for s in sc.values())
            lses.append(mx + math.log(den))
            outs.append(sum(math.exp(sc[j] - mx) / den * v[j] for j in sc))
        mx = max(lses)
        tot = mx + math.log(sum(math.exp(t - mx) for t in lses))
        lse[i] = tot
        out[i] = sum(math.exp(lses[r] - tot) * outs[r] for r in range(n_h))
    return out, lse


@pytest.mark.parametrize("L,c,n_b,n_h,causal", [
    (16, 4, 4, 2, True), (24, 8, 6, 3, False), (64, 8, 8, 2, True), (32, 32, 4, 1, False),
    (48, 8, 2, 4, True),
    # chunk_len not dividing L: the last chunk is short
    (20, 8, 4, 2, True), (30, 8, 6, 3, False), (50, 16, 8, 2, True), (7, 16, 4, 2, False)])
def test_brute_force_small(L, c, n_b, n_h, causal):
    rng = np.random.default_rng(L * 7 + n_b)
    d = 6
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    res = O.forward(x, v, R, n_b, c, causal)
    bo, bl = _brute_force(x[0, 0], v[0, 0], res["buckets"][0, 0], c, causal)
    np.testing.assert_allclose(res["out"][0, 0], bo, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(res["lse"][0, 0], bl, rtol=1e-12, atol=1e-9)


# -------------------------------------- multiset-union closed form --------
def _membership(undo, c):
    """m[i, j] = number of rounds in which j lies in i's window (from chunk ids)."""
    n_h, L = undo.shape
    ch = undo // c
    m = np.zeros((L, L), np.int64)
    for r in range(n_h):
        diff = ch[r][:, None] - ch[r][None, :]
        m += ((diff == 0) | (diff == 1)).astype(np.int64)
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_multiset_union_closed_form(causal):
    rng = np.random.default_rng(11)
    L, d, c, n_h, n_b = 128, 8, 16, 4, 8
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    res = O.forward(x, v, R, n_b, c, causal)
    m = _membership(res["undo"][0, 0], c).astype(float)
    xx = x[0, 0]
    kh = xx / np.linalg.norm(xx, axis=1, keepdims=True)
    s = xx @ kh.T / math.sqrt(d)
    np.fill_diagonal(s, O.SELF_SCORE)
    if causal:
        m = np.tril(m)
    shift = np.where(m > 0, s, -np.inf).max(axis=1, keepdims=True)
    w = np.where(m > 0, m * np.exp(np.minimum(s - shift, 0.0)), 0.0)
    out = (w @ v[0, 0]) / w.sum(axis=1, keepdims=True)
    lse = shift[:, 0] + np.log(w.sum(axis=1))
    np.testing.assert_allclose(res["out"][0, 0], out, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(res["lse"][0, 0], lse, rtol=1e-12, atol=1e-10)


def test_dedup_gives_set_union():
    # With the duplicate-count correction each key in the union counts once.
    rng = np.random.default_rng(12)
    L, d, c, n_h, n_b = 64, 8, 8, 3, 4
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    res = O.forward(x, v, R, n_b, c, True, dedup=True)
    m = (_membership(res["undo"][0, 0], c) > 0).astype(float)
    m = np.tril(m)
    xx = x[0, 0]
    kh = xx / np.linalg.norm(xx, axis=1, keepdims=True)
    s = xx @ kh.T / math.sqrt(d)
    np.fill_diagonal(s, O.SELF_SCORE)
    shift = np.where(m > 0, s, -np.inf).max(axis=1, keepdims=True)
    w = np.where(m > 0, m * np.exp(np.minimum(s - shift, 0.0)), 0.0)
    np.testing.assert_allclose(res["out"][0, 0], (w @ v[0, 0]) / w.sum(1, keepdims=True),
                               rtol=1e-10, atol=1e-11)


# ----------------------------------------------------- invariants --------
def test_first_causal_token_attends_only_itself():
    rng = np.random.default_rng(13)
    L, d = 64, 8
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    for n_h in (1, 4):
        R = rng.standard_normal((n_h, d, 4))
        res = O.forward(x, v, R, 8, 16, True)
        # exp(lse_r - LSE) at |lse| ~ 1e5 carries rounding of ~1e-11 relative
        np.testing.assert_allclose(res["out"][0, 0, 0], v[0, 0, 0], rtol=1e-10, atol=0)
        if n_h == 1:
            np.testing.assert_array_equal(res["out"][0, 0, 0], v[0, 0, 0])
        assert abs(res["lse"][0, 0, 0] - (O.SELF_SCORE + math.log(n_h))) < 1e-9
        assert (res["lse_rounds"][0, 0, :, 0] == O.SELF_SCORE).all()


def test_rounds_are_independent_and_order_free():
    rng = np.random.default_rng(14)
    L, d, c = 64, 8, 8
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((3, d, 4))
    one = O.forward(x, v, R[:1], 8, c, True)
    # n_hashes = 1: the combine returns round 0 unchanged
    np.testing.assert_array_equal(one["out"][0, 0], one["o_rounds"][0, 0, 0])
    np.testing.assert_array_equal(one["lse"][0, 0], one["lse_rounds"][0, 0, 0])
    # the same rotation twice gives the one-round output, lse + log 2
    two = O.forward(x, v, np.concatenate([R[:1], R[:1]]), 8, c, True)
    np.testing.assert_allclose(two["out"], one["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(two["lse"], one["lse"] + math.log(2), rtol=1e-14, atol=1e-10)
    # permuting the rounds leaves out and lse unchanged
    a = O.forward(x, v, R, 8, c, True)
    b = O.forward(x, v, R[[2, 0, 1]], 8, c, True)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-14, atol=1e-12)


def test_token_rounds_matches_whole_pass():
    rng = np.random.default_rng(15)
    L, d, c, n_h = 256, 16, 32, 3
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, 8))
    res = O.forward(x, v, R, 16, c, True)
    for i in random.Random(0).sample(range(L), 20):
        o, lse = O.token_rounds(x[0, 0], v[0, 0], res["perm"][0, 0], res["undo"][0, 0], c, True, i)
        np.testing.assert_allclose(o, res["o_rounds"][0, 0, :, i], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, res["lse_rounds"][0, 0, :, i], rtol=1e-13, atol=1e-10)


def test_zero_norm_key_reads_as_zero_vector():
    x = np.zeros((1, 1, 4, 2))
    x[0, 0, 1] = [3.0, 4.0]
    v = np.arange(8.0).reshape(1, 1, 4, 2)
    res = O.forward(x, v, None, 1, 4, False, buckets=np.zeros((1, 1, 1, 4), np.int64))
    assert np.isfinite(res["out"]).all() and np.isfinite(res["lse"]).all()


# ------------------------------------------------- bucket-equality mask --
def test_bucket_mask_brute_force():
    # The variant of section 2 "LSH attention" (a query attends only to keys
    # in its own bucket), written from the set definition: for each query,
    # loop over all positions and keep those in its window (same or previous
    # chunk of the sorted order), in its bucket, not in its future; the self
    # pair scores -1e5.
    rng = np.random.default_rng(21)
    L, d, c, n_h, n_b = 48, 8, 8, 2, 6
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    for causal in (False, True):
        res = O.forward(x, v, R, n_b, c, causal, bucket_mask=True)
        xx, vv = x[0, 0], v[0, 0]
        for r in range(n_h):
            bk = res["buckets"][0, 0, r]
            slot = res["undo"][0, 0, r]
            for i in range(L):
                keys, scores = [], []
                for j in range(L):
                    ci, cj = slot[i] // c, slot[j] // c
                    if ci - cj not in (0, 1) or bk[j] != bk[i] or (causal and j > i):
                        continue
                    s = O.SELF_SCORE if j == i else \
                        xx[i] @ (xx[j] / np.linalg.norm(xx[j])) / math.sqrt(d)
                    keys.append(j)
                    scores.append(s)
                scores = np.array(scores)
                m = scores.max()
                w = np.exp(scores - m)
                o = (w[:, None] * vv[keys]).sum(0) / w.sum()
                np.testing.assert_allclose(res["o_rounds"][0, 0, r, i], o, rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(res["lse_rounds"][0, 0, r, i], m + np.log(w.sum()),
                                           rtol=1e-12, atol=1e-10)


def test_bucket_mask_is_a_no_op_within_one_bucket():
    rng = np.random.default_rng(22)
    L, d, c, n_h = 64, 8, 16, 2
    x = rng.standard_normal((1, 2, L, d))
    v = rng.standard_normal((1, 2, L, d))
    zero = np.zeros((1, 2, n_h, L), np.int64)
    a = O.forward(x, v, None, 1, c, True, buckets=zero)
    b = O.forward(x, v, None, 1, c, True, buckets=zero, bucket_mask=True)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


# ------------------------------------------------ routing-style assignment --
def test_kmeans_with_plus_minus_rotation_is_the_lsh_hash():
    # Centroids [R, -R] give dot products [xR; -xR]: the assignment must equal
    # the random-rotation hash, bucket for bucket and margin for margin.
    rng = np.random.default_rng(31)
    x = rng.standard_normal((2, 3, 40, 8))
    R = rng.standard_normal((3, 8, 5))
    lb, lm = O.hash_all(x, R, 10)
    kb, km = O.hash_all(x, np.concatenate([R, -R], axis=2), 10, kmeans=True)
    np.testing.assert_array_equal(kb, lb)
    np.testing.assert_array_equal(km, lm)


def test_kmeans_picks_the_largest_coordinate_with_basis_centroids():
    # Centroids e_0..e_{d-1}: x . e_j = x_j, so the bucket is the index of the
    # largest coordinate (the first one on ties).
    x = np.array([[0.5, 2.0, -3.0, 2.0], [-1.0, -2.0, -0.5, -4.0], [1.0, 1.0, 1.0, 1.0]])
    C = np.eye(4)[None]                            # [1, d, n_b = d]
    b, m = O.kmeans_head(x, C, 4)
    np.testing.assert_array_equal(b[0], [1, 2, 0])
    np.testing.assert_allclose(m[0], [0.0, 0.5, 0.0])


# ------------------------------------------------------------- backward --
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    # d out . g w.r.t. qk and v by central differences, the buckets and their
    # sort held fixed (the hash does not move for steps this small)
    rng = np.random.default_rng(41)
    L, d, c, n_h, n_b = 20, 4, 4, 2, 4
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    g = rng.standard_normal((L, d))
    res = O.forward(x, v, R, n_b, c, causal)
    perm = res["perm"][0, 0]
    buckets = res["buckets"]
    dq, dv = O.backward_head(x[0, 0], v[0, 0], perm, c, causal, g)
    h = 1e-6

    def f(xx, vv):
        r = O.forward(xx, vv, R, n_b, c, causal, buckets=buckets)
        return float((r["out"][0, 0] * g).sum())

    for (i, t) in [(0, 0), (3, 1), (7, 2), (12, 3), (19, 0)]:
        xp, xm = x.copy(), x.copy()
        xp[0, 0, i, t] += h
        xm[0, 0, i, t] -= h
        np.testing.assert_allclose(dq[i, t], (f(xp, v) - f(xm, v)) / (2 * h), rtol=1e-5,
                                   atol=1e-7)
        vp, vm = v.copy(), v.copy()
        vp[0, 0, i, t] += h
        vm[0, 0, i, t] -= h
        np.testing.assert_allclose(dv[i, t], (f(x, vp) - f(x, vm)) / (2 * h), rtol=1e-5,
                                   atol=1e-7)


def test_backward_of_v_is_the_attention_transpose():
    # out is linear in v: d v_j = sum_i A_ij g_i with A the combined attention
    # weights, which the multiset form gives from the membership counts
    rng = np.random.default_rng(42)
    L, d, c, n_h, n_b = 32, 4, 8, 3, 4
    x = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((n_h, d, n_b // 2))
    g = rng.standard_normal((L, d))
    res = O.forward(x, v, R, n_b, c, True)
    _, dv = O.backward_head(x[0, 0], v[0, 0], res["perm"][0, 0], c, True, g)
    # A_ij from the same forward with v = e_j (linearity in v)
    A = np.empty((L, L))
    for j in range(L):
        e = np.zeros((1, 1, L, 1))
        e[0, 0, j, 0] = 1.0
        A[:, j] = O.forward(x, e, R, n_b, c, True, buckets=res["buckets"])["out"][0, 0, :, 0]
    np.testing.assert_allclose(dv, A.T @ g, rtol=1e-10, atol=1e-12)
