"""Oracle for the LSH attention forward pass: plain, slow, float64, CPU only.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module.  The CUDA library never calls it, and it
shares no code, table or helper with the CUDA path.

It states the method the way "Reformer: The Efficient Transformer" (arXiv
2001.04451v2) describes it, in the order given there:

  1. hash      -- section 2, "LSH attention": random projections,
                  h(x) = argmax([xR; -xR]), one independent rotation per
                  round (Appendix A, "Multi-round attention").
  2. sort      -- section 2: queries/keys are sorted by bucket (position is
                  the secondary key, carried through the same permutation,
                  section 2 "Causal masking").
  3. chunk     -- section 2 and Appendix A "Implementation": attention runs on
                  fixed-size chunks of the sorted sequence; each chunk attends
                  to itself and to the chunk before it.
  4. attend    -- shared-QK attention with normalised keys (section 5,
                  "Shared query-key space"); future positions masked when
                  causal; attention to oneself forbidden unless nothing else
                  is available (section 2 "Causal masking", Appendix A
                  "Masking").
  5. combine   -- Appendix A: each round gives an independently computable
                  output; the rounds are combined with weights
                  exp(lse_r - logsumexp_r lse_r) after unsorting.

Readings where the pages are silent (each is also listed in the design notes):
  * the hash sees raw qk (argmax is unchanged by a positive rescale, so this
    equals hashing the normalised key away from exact ties);
  * ties in the argmax go to the lowest index of [xR; -xR];
  * n_buckets == 1 puts every token in bucket 0 and needs no rotations;
  * the first chunk of a round has no look-back (no wrap to the last chunk,
    no crossing into another round);
  * when chunk_len does not divide L the last chunk holds the remaining
    L mod chunk_len slots (as if padded with slots that neither attend nor
    are attended);
  * no bucket-equality mask inside a window: the window is the attended set
    (``bucket_mask=True`` is the variant that also drops the window's keys
    whose bucket in that round differs from the query's, section 2 "LSH
    attention": a query attends only to targets in its own hash bucket);
  * scores are (q . k_hat) / sqrt(d_k);
  * the self-mask REPLACES the score of j == i by SELF_SCORE = -1e5, a finite
    penalty, so a token that sees only itself in every round outputs v_i;
  * a key of zero norm normalises to the zero vector;
  * the routing-style assignment (``kmeans=True``; the pages name online
    k-means for the Routing Transformer and give no more) puts token x in
    the bucket of the centroid with the largest dot product, argmax_j x . mu_j
    (lowest index on ties), with the centroids given ([n_h, d, n_b], one set
    per round) and not updated;
  * the duplicate-count correction of Appendix A is off unless asked for
    (``dedup=True`` subtracts log N_ij, N_ij = number of rounds whose window
    of query i contains key j).

Parity unpinned (by the pages): the self score -1e5, the 1/sqrt(d_k) scale,
the first chunk's missing look-back and the absence of a bucket mask are
readings, not facts the pages state; the tests fix them only through
hand-worked fixtures and brute forces that take the same readings.  Every
function here is otherwise pinned by tests that do not reuse its code
(closed forms, brute force, invariants, finite differences).
"""

from __future__ import annotations

import math

import numpy as np

SELF_SCORE = -1.0e5


# ---------------------------------------------------------------------------
# 1. Hash (section 2, "LSH attention"; Appendix A, multi-round hashing)
# ---------------------------------------------------------------------------
def hash_head(x: np.ndarray, rotations, n_buckets: int):
    """Bucket ids of every row of ``x`` for every hashing round.

    x: [L, d] float64.  rotations: [n_hashes, d, n_buckets // 2] float64, or
    None when n_buckets == 1.  Returns (buckets [n_h, L] int64,
    margins [n_h, L] float64), where the margin is the largest minus the
    second largest entry of z = [xR; -xR] (+inf for the one-bucket case).
    """
    L = x.shape[0]
    if n_buckets == 1:
        n_h = 1 if rotations is None else rotations.shape[0]
        return np.zeros((n_h, L), np.int64), np.full((n_h, L), np.inf)
    n_h, d, half = rotations.shape
    assert 2 * half == n_buckets and d == x.shape[1]
    buckets = np.empty((n_h, L), np.int64)
    margins = np.empty((n_h, L), np.float64)
    for r in range(n_h):
        p = x @ rotations[r]                       # projections xR, [L, n_b/2]
        z = np.concatenate([p, -p], axis=1)        # [xR; -xR], [L, n_b]
        buckets[r] = np.argmax(z, axis=1)          # first maximal index
        top2 = np.partition(z, n_buckets - 2, axis=1)[:, n_buckets - 2:]
        margins[r] = top2[:, 1] - top2[:, 0]
    return buckets, margins


# ---------------------------------------------------------------------------
# 2. Sort (section 2; Appendix A "Implementation")
# ---------------------------------------------------------------------------
def sort_head(buckets: np.ndarray):
    """Per round, the order of positions by the key (bucket, position).

    buckets: [n_h, L].  Returns (perm, undo), both [n_h, L] int64:
    perm[r, s] = position that sits at sorted slot s; undo[r, perm[r, s]] = s.
    A stable sort by bucket keeps positions increasing inside a bucket, which
    is the secondary key.
    """
    n_h, L = buckets.shape
    perm = np.empty((n_h, L), np.int64)
    undo = np.empty((n_h, L), np.int64)
    for r in range(n_h):
        perm[r] = np.argsort(buckets[r], kind="stable")
        undo[r, perm[r]] = np.arange(L)
    return perm, undo


# ---------------------------------------------------------------------------
# 3 + 4. Chunks and masked shared-QK attention (section 2; Appendix A)
# ---------------------------------------------------------------------------
def normalised_keys(x: np.ndarray) -> np.ndarray:
    """k_hat = x / ||x||_2 row by row; a zero row stays zero."""
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    return np.where(n[:, None] > 0, x / safe[:, None], 0.0)


def window_slots(k: int, chunk_len: int, L: int):
    """Sorted slots a query in chunk k attends: chunk k-1 (if k > 0) and chunk
    k; the last chunk ends at L when chunk_len does not divide L."""
    lo = (k - 1) * chunk_len if k > 0 else 0
    return lo, min((k + 1) * chunk_len, L)


def attend_round(x, v, perm_r, chunk_len: int, causal: bool, dedup_undo=None,
                 bucket_r=None):
    """One hashing round: chunked attention in sorted order, results unsorted.

    x, v: [L, d] float64; perm_r: [L] sorted order of this round.
    Returns (o [L, d], lse [L]) indexed by ORIGINAL position.
    ``dedup_undo`` ([n_h, L] undo of every round) turns on the duplicate-count
    correction of Appendix A.  ``bucket_r`` ([L] bucket of every position in
    this round) turns on the bucket-equality mask: a key whose bucket differs
    from the query's is not attended.
    """
    L, d = x.shape
    c = chunk_len
    n_c = -(-L // c)  # the last chunk holds the L mod c remaining slots
    khat = normalised_keys(x)
    xs, ks, vs, pos = x[perm_r], khat[perm_r], v[perm_r], perm_r
    o = np.empty((L, d))
    lse = np.empty(L)
    for k in range(n_c):
        q0, q1 = k * c, min((k + 1) * c, L)
        k0, k1 = window_slots(k, c, L)
        s = xs[q0:q1] @ ks[k0:k1].T / math.sqrt(d)
        qp = pos[q0:q1][:, None]
        kp = pos[k0:k1][None, :]
        if dedup_undo is not None:
            s = s - np.log(duplicate_counts(dedup_undo, pos[q0:q1], pos[k0:k1], c))
        if bucket_r is not None:
            s = np.where(bucket_r[kp] != bucket_r[qp], -np.inf, s)
        s = np.where(kp == qp, SELF_SCORE, s)
        if causal:
            s = np.where(kp > qp, -np.inf, s)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        l = np.sum(e, axis=1)
        o[pos[q0:q1]] = (e / l[:, None]) @ vs[k0:k1]
        lse[pos[q0:q1]] = m[:, 0] + np.log(l)
    return o, lse


def duplicate_counts(undo, q_pos, k_pos, chunk_len):
    """N_ij: in how many rounds key j lies in the window of query i.

    undo: [n_h, L]; q_pos: [m]; k_pos: [n].  Returns [m, n] int (>= 1 for a
    pair taken from a window of one of the rounds).
    """
    cq = undo[:, q_pos] // chunk_len                 # [n_h, m] chunk of i
    ck = undo[:, k_pos] // chunk_len                 # [n_h, n] chunk of j
    diff = cq[:, :, None] - ck[:, None, :]
    return np.sum((diff == 0) | (diff == 1), axis=0)


# ---------------------------------------------------------------------------
# 5. Combine (Appendix A)
# ---------------------------------------------------------------------------
def combine_head(o_rounds: np.ndarray, lse_rounds: np.ndarray):
    """out_i = sum_r exp(lse_r,i - LSE_i) o_r,i with LSE_i = logsumexp_r lse_r,i.

    o_rounds: [n_h, L, d]; lse_rounds: [n_h, L].  Returns (out [L, d], lse [L]).
    """
    m = np.max(lse_rounds, axis=0)
    lse = m + np.log(np.sum(np.exp(lse_rounds - m), axis=0))
    w = np.exp(lse_rounds - lse)                      # [n_h, L]
    out = np.sum(w[:, :, None] * o_rounds, axis=0)
    return out, lse


# ---------------------------------------------------------------------------
# Whole forward pass and batched helpers
# ---------------------------------------------------------------------------
def as_f64(t) -> np.ndarray:
    """Exact promotion of a torch tensor (f32 or bf16) or array to float64."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def kmeans_head(x: np.ndarray, centroids, n_buckets: int):
    """Routing-style assignment: bucket = argmax_j x . mu_j over the round's
    n_b centroids (first maximal index).  x: [L, d]; centroids: [n_h, d, n_b].
    Returns (buckets [n_h, L], margins [n_h, L]) like hash_head."""
    n_h, d, nb = centroids.shape
    assert nb == n_buckets and d == x.shape[1]
    L = x.shape[0]
    buckets = np.empty((n_h, L), np.int64)
    margins = np.empty((n_h, L), np.float64)
    for r in range(n_h):
        p = x @ centroids[r]                       # [L, n_b]
        buckets[r] = np.argmax(p, axis=1)
        if nb >= 2:
            top2 = np.partition(p, nb - 2, axis=1)[:, nb - 2:]
            margins[r] = top2[:, 1] - top2[:, 0]
        else:
            margins[r] = np.inf
    return buckets, margins


def hash_all(qk, rotations, n_buckets, kmeans=False):
    """[B, H, L, d] -> buckets, margins [B, H, n_h, L].  With ``kmeans`` the
    rotations are centroids [n_h, d, n_b] and kmeans_head assigns."""
    qk = as_f64(qk)
    rot = None if rotations is None else as_f64(rotations)
    B, H, L, _ = qk.shape
    n_h = 1 if rot is None else rot.shape[0]
    buckets = np.empty((B, H, n_h, L), np.int64)
    margins = np.empty((B, H, n_h, L))
    for b in range(B):
        for h in range(H):
            if kmeans:
                buckets[b, h], margins[b, h] = kmeans_head(qk[b, h], rot, n_buckets)
            else:
                buckets[b, h], margins[b, h] = hash_head(qk[b, h], rot, n_buckets)
    return buckets, margins


def sort_all(buckets):
    """[B, H, n_h, L] buckets -> perm, undo of the same shape."""
    buckets = np.asarray(buckets)
    perm = np.empty(buckets.shape, np.int64)
    undo = np.empty(buckets.shape, np.int64)
    for b in range(buckets.shape[0]):
        for h in range(buckets.shape[1]):
            perm[b, h], undo[b, h] = sort_head(buckets[b, h])
    return perm, undo


def attend_all(qk, v, perm, chunk_len, causal, dedup=False, buckets=None):
    """Per-round outputs at original positions: o [B,H,n_h,L,d], lse [B,H,n_h,L].
    ``buckets`` ([B,H,n_h,L]) turns on the bucket-equality mask."""
    qk, v = as_f64(qk), as_f64(v)
    perm = np.asarray(perm)
    B, H, n_h, L = perm.shape
    d = qk.shape[-1]
    o = np.empty((B, H, n_h, L, d))
    lse = np.empty((B, H, n_h, L))
    for b in range(B):
        for h in range(H):
            undo = None
            if dedup:
                undo = np.empty((n_h, L), np.int64)
                for r in range(n_h):
                    undo[r, perm[b, h, r]] = np.arange(L)
            for r in range(n_h):
                bk = None if buckets is None else np.asarray(buckets)[b, h, r]
                o[b, h, r], lse[b, h, r] = attend_round(qk[b, h], v[b, h], perm[b, h, r],
                                                        chunk_len, causal, undo, bk)
    return o, lse


def combine_all(o_rounds, lse_rounds):
    o_rounds, lse_rounds = np.asarray(o_rounds, np.float64), np.asarray(lse_rounds, np.float64)
    B, H, n_h, L, d = o_rounds.shape
    out = np.empty((B, H, L, d))
    lse = np.empty((B, H, L))
    for b in range(B):
        for h in range(H):
            out[b, h], lse[b, h] = combine_head(o_rounds[b, h], lse_rounds[b, h])
    return out, lse


def forward(qk, v, rotations, n_buckets, chunk_len, causal, buckets=None, dedup=False,
            bucket_mask=False, kmeans=False):
    """The whole pass.  If ``buckets`` is given, hashing is skipped and those
    ids are used (this is how GPU bucket ids are fed back so that the later
    stages can be compared exactly).  Returns a dict of every intermediate."""
    res = {}
    if buckets is None:
        buckets, margins = hash_all(qk, rotations, n_buckets, kmeans=kmeans)
        res["margins"] = margins
    buckets = np.asarray(buckets, np.int64)
    perm, undo = sort_all(buckets)
    o_r, lse_r = attend_all(qk, v, perm, chunk_len, causal, dedup=dedup,
                            buckets=buckets if bucket_mask else None)
    out, lse = combine_all(o_r, lse_r)
    res.update(buckets=buckets, perm=perm, undo=undo, o_rounds=o_r, lse_rounds=lse_r,
               out=out, lse=lse)
    return res


def token_rounds(x, v, perm, undo, chunk_len, causal, i):
    """Per-round output of ONE token i, computed from its windows alone.

    x, v: [L, d] float64 of one (batch, head); perm, undo: [n_h, L].
    Returns (o [n_h, d], lse [n_h]).  Used to check sampled outputs at sizes
    where the whole oracle would be too slow.
    """
    n_h = perm.shape[0]
    d = x.shape[1]
    o = np.empty((n_h, d))
    lse = np.empty(n_h)
    xi = x[i]
    for r in range(n_h):
        k = undo[r, i] // chunk_len
        k0, k1 = window_slots(k, chunk_len, x.shape[0])
        kp = perm[r, k0:k1]
        keys = normalised_keys(x[kp])
        s = keys @ xi / math.sqrt(d)
        s = np.where(kp == i, SELF_SCORE, s)
        if causal:
            s = np.where(kp > i, -np.inf, s)
        m = np.max(s)
        e = np.exp(s - m)
        l = np.sum(e)
        o[r] = (e / l) @ v[kp]
        lse[r] = m + np.log(l)
    return o, lse


# ---------------------------------------------------------------------------
# 6. Backward (hash and sort held fixed: no gradient through bucket ids)
# ---------------------------------------------------------------------------
def backward_head(x, v, perm, chunk_len: int, causal: bool, dout):
    """Gradients of out w.r.t. the shared qk and v of one (batch, head), with
    the buckets and their sort held fixed (the hash is piecewise constant).

    The forward is re-stated in float64 torch, step for step as attend_round
    and combine_head do it (windows of chunks k-1 and k in sorted order,
    normalised keys, 1/sqrt(d), self score -1e5 as a constant, causal mask,
    per-round logsumexp, combine over rounds); autograd then gives
    (d qk [L, d], d v [L, d]) for the upstream gradient dout [L, d].  The
    tests pin it against central finite differences and the numpy forward.
    """
    import torch
    X = torch.tensor(np.asarray(x, np.float64), requires_grad=True)
    V = torch.tensor(np.asarray(v, np.float64), requires_grad=True)
    n_h, L = np.asarray(perm).shape
    d = X.shape[1]
    c = chunk_len
    norm = torch.sqrt((X * X).sum(1))
    K = torch.where(norm[:, None] > 0, X / torch.where(norm > 0, norm, 1.0)[:, None],
                    torch.zeros_like(X))
    outs, lses = [], []
    for r in range(n_h):
        pr = torch.as_tensor(np.asarray(perm)[r], dtype=torch.long)
        o_r = torch.zeros(L, d, dtype=torch.float64)
        l_r = torch.zeros(L, dtype=torch.float64)
        for k in range(-(-L // c)):
            q0, q1 = k * c, min((k + 1) * c, L)
            k0, k1 = (k - 1) * c if k > 0 else 0, min((k + 1) * c, L)
            qi, kj = pr[q0:q1], pr[k0:k1]
            s = X[qi] @ K[kj].T / math.sqrt(d)
            same = qi[:, None] == kj[None, :]
            s = torch.where(same, torch.full_like(s, SELF_SCORE), s)
            if causal:
                s = torch.where(kj[None, :] > qi[:, None], torch.full_like(s, -math.inf), s)
            lse = torch.logsumexp(s, dim=1)
            p = torch.exp(s - lse[:, None])
            o_r = o_r.index_put((qi,), p @ V[kj])
            l_r = l_r.index_put((qi,), lse)
        outs.append(o_r)
        lses.append(l_r)
    O = torch.stack(outs)                       # [n_h, L, d]
    Lr = torch.stack(lses)                      # [n_h, L]
    w = torch.softmax(Lr, dim=0)                # exp(lse_r - LSE)
    out = (w[:, :, None] * O).sum(0)
    out.backward(torch.as_tensor(np.asarray(dout, np.float64)))
    return X.grad.numpy(), V.grad.numpy()


def backward_all(qk, v, perm, chunk_len, causal, dout):
    """[B, H, L, d] gradients of out for fixed perm [B, H, n_h, L]."""
    qk, v, dout = as_f64(qk), as_f64(v), as_f64(dout)
    perm = np.asarray(perm)
    dq = np.empty_like(qk)
    dv = np.empty_like(v)
    for b in range(qk.shape[0]):
        for h in range(qk.shape[1]):
            dq[b, h], dv[b, h] = backward_head(qk[b, h], v[b, h], perm[b, h], chunk_len, causal,
                                               dout[b, h])
    return dq, dv
