"""CUDA path against the fp64 oracle, through the C ABI (needs an sm_100a GPU).

Every stage is compared on seeded inputs: bucket ids exactly except near
ties (reported), sort outputs bit for bit from the GPU's bucket ids, and the
floating-point outputs within the tolerances in ``parity.py``.  The fused
``lsh_attn_forward`` must equal the four stage calls bit for bit.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import lsh_bucketed_sparse_b200 as lsh
from lsh_bucketed_sparse_b200 import workloads as W
from oracle import lsh_oracle as O

import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _stages(wl, qk, v, rot, portable=False):
    """Run the four stage calls and the fused call on the GPU."""
    qk_d, v_d = qk.to(DEV), v.to(DEV)
    rot_d = None if rot is None else rot.to(DEV)
    buckets, inv_norm = lsh.lsh_attn_hash(qk_d, rot_d, wl.n_buckets, wl.n_hashes,
                                          portable=portable)
    perm, undo, counts = lsh.lsh_attn_sort(buckets, wl.n_buckets, want_counts=True)
    o_r, lse_r = lsh.lsh_attn_chunked_fwd(qk_d, v_d, inv_norm, perm, wl.chunk_len, wl.causal,
                                          n_buckets=wl.n_buckets, portable=portable)
    out, lse = lsh.lsh_attn_combine(o_r, lse_r)
    f_out, f_lse = lsh.lsh_attn_forward(qk_d, v_d, rot_d, wl.n_hashes, wl.n_buckets,
                                        wl.chunk_len, wl.causal, portable=portable)
    lsh.lsh_attn_device_check()
    return dict(buckets=buckets, inv_norm=inv_norm, perm=perm, undo=undo, counts=counts,
                o_rounds=o_r, lse_rounds=lse_r, out=out, lse=lse, f_out=f_out, f_lse=f_lse)


def _full_check(wl, portable=False, qk_override=None):
    qk, v, rot = W.make_inputs(wl)
    if qk_override is not None:
        qk = qk_override(qk)
    g = _stages(wl, qk, v, rot, portable)
    bf16 = wl.dtype == torch.bfloat16
    report = {}
    # hash
    if wl.n_buckets > 1:
        ob, margins = O.hash_all(qk, rot, wl.n_buckets)
        report["buckets"] = P.check_buckets(g["buckets"], ob, margins)
    else:
        assert (g["buckets"] == 0).all()
    xn = P.np64(qk)
    norms = np.sqrt((xn * xn).sum(-1))
    inv = np.where(norms > 0, 1.0 / np.where(norms > 0, norms, 1.0), 0.0)
    np.testing.assert_allclose(P.np64(g["inv_norm"]), inv, rtol=2e-6, atol=0)
    # everything downstream from the GPU's own bucket ids
    res = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal,
                    buckets=g["buckets"].cpu().numpy().astype(np.int64))
    np.testing.assert_array_equal(g["perm"].cpu().numpy(), res["perm"])
    np.testing.assert_array_equal(g["undo"].cpu().numpy(), res["undo"])
    counts = np.stack([np.stack([np.stack([np.bincount(res["buckets"][b, h, r],
                                                       minlength=wl.n_buckets)
                                           for r in range(wl.n_hashes)])
                                 for h in range(wl.heads)]) for b in range(wl.batch)])
    np.testing.assert_array_equal(g["counts"].cpu().numpy(), counts)
    report["o_rounds"] = P.check_float(g["o_rounds"], res["o_rounds"], bf16, "o_rounds", 3)
    report["lse_rounds"] = P.check_lse(g["lse_rounds"], res["lse_rounds"], bf16, "lse_rounds")
    report["out"] = P.check_float(g["out"], res["out"], bf16, "out")
    report["lse"] = P.check_lse(g["lse"], res["lse"], bf16, "lse")
    # the fused pass is the same kernels in the same order
    assert torch.equal(g["f_out"], g["out"]) and torch.equal(g["f_lse"], g["lse"])
    return report, g


# Workloads small enough for the whole oracle, spanning several hash tiles
# (128 rows), several chunks, a ragged hash tile and the edge cases.
SMALL = [
    W.small("bf16-causal-ragged", heads=2, seq_len=1088, n_hashes=3, n_buckets=32),
    W.small("bf16-noncausal-d128", heads=2, seq_len=1024, d_k=128, n_hashes=2, n_buckets=64,
            chunk_len=128, causal=False),
    W.small("f32-causal", heads=2, seq_len=512, n_hashes=2, n_buckets=16, dtype=torch.float32),
    W.small("bf16-one-chunk", heads=1, seq_len=64, n_hashes=2, n_buckets=8),
    W.small("bf16-two-buckets", heads=2, seq_len=512, n_hashes=4, n_buckets=2),
    W.small("bf16-c32-d32", heads=3, seq_len=768, d_k=32, n_hashes=2, n_buckets=12,
            chunk_len=32),
    W.small("bf16-clustered", heads=2, seq_len=2048, n_hashes=2, n_buckets=64, clustered=True,
            n_clusters=16, causal=False),
    # shapes that take the tensor-core hash: several rounds per MMA piece and a
    # ragged last tile; one round split over two pieces; d = 128 with a
    # 384-column round; 96-column rounds packed two per piece
    W.small("tc-hash-ragged", heads=2, seq_len=1088, n_hashes=3, n_buckets=64),
    W.small("tc-hash-wide", heads=2, seq_len=1024, n_hashes=2, n_buckets=1024),
    W.small("tc-hash-d128-p384", heads=2, seq_len=512, d_k=128, n_hashes=2, n_buckets=768,
            chunk_len=128, causal=False),
    W.small("tc-hash-p96", heads=3, seq_len=768, n_hashes=4, n_buckets=192),
    # 64-column rounds, four per 256-column piece, and a ragged last tile
    W.small("tc-hash-p64", heads=2, seq_len=1088, n_hashes=4, n_buckets=128),
    # rounds of whole 128-column groups: one round per 256-column piece, and
    # 384-column rounds that end inside a piece
    W.small("tc-hash-p256", heads=2, seq_len=1088, n_hashes=3, n_buckets=512),
    W.small("tc-hash-p384", heads=2, seq_len=1088, n_hashes=2, n_buckets=768),
    # chunk_len not dividing L: the last chunk of the sorted order is short
    W.small("ragged-chunk-c64-L1000", heads=2, seq_len=1000, n_hashes=2, n_buckets=32),
    W.small("ragged-chunk-c128-d128-L1500", heads=1, seq_len=1500, d_k=128, n_hashes=2,
            n_buckets=64, chunk_len=128, causal=False),
    W.small("ragged-chunk-c64-tc-hash-L1100", heads=2, seq_len=1100, n_hashes=3,
            n_buckets=128),
    W.small("ragged-chunk-f32-c48-L500", heads=2, seq_len=500, n_hashes=2, n_buckets=16,
            chunk_len=48, dtype=torch.float32),
    # the four tensor-core attention specialisations (chunk, d_k)
    W.small("tc-attn-c64-d128", heads=2, seq_len=1472, d_k=128, n_hashes=2, n_buckets=64),
    W.small("tc-attn-c128-d64-causal", heads=2, seq_len=1408, n_hashes=3, n_buckets=64,
            chunk_len=128),
    W.small("tc-attn-c128-d128-causal", heads=1, seq_len=2048, d_k=128, n_hashes=2,
            n_buckets=128, chunk_len=128),
    W.small("tc-attn-c64-d64-noncausal", batch=2, heads=2, seq_len=1536, n_hashes=2,
            n_buckets=128, causal=False),
    # L not a multiple of 4: every segment after the first starts off a
    # 16-byte boundary of perm (position loads fall back to 4-byte loads)
    W.small("odd-L1001-c64-d64", batch=2, heads=2, seq_len=1001, n_hashes=3, n_buckets=64),
    W.small("odd-L999-c128-d64", heads=3, seq_len=999, n_hashes=2, n_buckets=64,
            chunk_len=128, causal=False),
    W.small("odd-L1003-c64-d128", heads=2, seq_len=1003, d_k=128, n_hashes=2,
            n_buckets=128),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
@pytest.mark.parametrize("portable", [False, True], ids=["fast", "portable"])
def test_small_workloads(wl, portable):
    report, _ = _full_check(wl, portable)
    print(wl.name, report)


@pytest.mark.parametrize("idx", [0, 1, 2, 4])
def test_named_workloads_full_size(idx):
    wl = W.WORKLOADS[idx]
    report, _ = _full_check(wl)
    print(wl.name, report)


@pytest.mark.parametrize("causal", [False, True])
def test_full_attention_limit_on_gpu(causal):
    # one bucket, one chunk over the whole sequence: plain shared-QK attention
    wl = W.small("one-bucket", heads=2, seq_len=256, n_hashes=2, n_buckets=1, chunk_len=256,
                 causal=causal, dtype=torch.float32)
    report, g = _full_check(wl)
    qk, v, _ = W.make_inputs(wl)
    for h in range(2):
        x = P.np64(qk[0, h])
        kh = O.normalised_keys(x)
        s = x @ kh.T / math.sqrt(wl.d_k)
        np.fill_diagonal(s, O.SELF_SCORE)
        if causal:
            s = np.where(np.triu(np.ones_like(s, bool), 1), -np.inf, s)
        p = np.exp(s - s.max(1, keepdims=True))
        ref = (p / p.sum(1, keepdims=True)) @ P.np64(v[0, h])
        assert np.abs(P.np64(g["out"][0, h]) - ref).max() < 1e-4


def test_first_causal_token_outputs_its_value():
    wl = W.small("first-token", heads=2, seq_len=512, n_hashes=4, n_buckets=64)
    qk, v, rot = W.make_inputs(wl)
    g = _stages(wl, qk, v, rot)
    assert torch.equal(g["out"][:, :, 0].cpu(), v[:, :, 0])
    assert (g["lse_rounds"][:, :, :, 0] == -1e5).all()


def test_zero_rows_and_scaled_rows():
    wl = W.small("zero-rows", heads=1, seq_len=256, n_hashes=2, n_buckets=64, causal=False)

    def plant(qk):
        qk = qk.clone()
        qk[0, 0, 5] = 0
        qk[0, 0, 77] = 0
        qk[0, 0, 100] = qk[0, 0, 99] * 4  # exact rescale: same bucket in every round
        return qk

    report, g = _full_check(wl, qk_override=plant)
    b = g["buckets"][0, 0]
    assert (b[:, 5] == 0).all() and (b[:, 77] == 0).all()
    assert torch.equal(b[:, 100], b[:, 99])
    assert g["inv_norm"][0, 0, 5] == 0


def _planted_tie_rotations(wl, rot):
    """Rotations whose column j1 = 3 (scaled by 4, so it usually holds the
    largest |p|) is repeated in a chunk of the same epilogue half, repeated in
    a chunk of the other half, and negated in a later chunk: every token then
    has exact |p| ties, which the argmax breaks by the lowest index of
    [xR; -xR] (a positive entry before any negative one, then the smaller j)."""
    P_ = wl.n_buckets // 2
    j1 = 3
    same = j1 + 64 if P_ > j1 + 64 else 7
    other = j1 + 32 if P_ > j1 + 32 else 11
    neg = j1 + 96 if P_ > j1 + 96 else P_ - 5
    assert len({j1, same, other, neg}) == 4 and max(same, other, neg) < P_
    rot = rot.clone()
    rot[:, :, j1] *= 4
    rot[:, :, same] = rot[:, :, j1]
    rot[:, :, other] = rot[:, :, j1]
    rot[:, :, neg] = -rot[:, :, j1]
    return rot


@pytest.mark.parametrize("portable", [False, True], ids=["fast", "portable"])
@pytest.mark.parametrize("n_buckets", [64, 192, 256, 1024])
def test_hash_breaks_exact_ties_by_lowest_index(n_buckets, portable):
    wl = W.small(f"ties-{n_buckets}", heads=2, seq_len=640, n_hashes=2, n_buckets=n_buckets)
    qk, _, rot = W.make_inputs(wl)
    rot = _planted_tie_rotations(wl, rot)
    b, _ = lsh.lsh_attn_hash(qk.to(DEV), rot.to(DEV), wl.n_buckets, wl.n_hashes,
                             portable=portable)
    b = b.cpu().numpy().astype(np.int64)
    x, R = P.np64(qk), P.np64(rot)
    checked = 0
    for h in range(wl.heads):
        for r in range(wl.n_hashes):
            p = x[0, h] @ R[r]
            z = np.concatenate([p, -p], axis=1)
            top = z.max(1, keepdims=True)
            below = np.where(z < top, z, -np.inf).max(1)
            clear = (top[:, 0] - below) >= 1e-5      # a clear gap below the tied group
            want = np.argmax(z, axis=1)               # first maximal index
            ok = b[0, h, r] == want
            assert ok[clear].all(), np.nonzero(~ok & clear)[0][:10]
            checked += int(clear.sum())
    assert checked > 0.9 * wl.heads * wl.n_hashes * wl.seq_len


@pytest.mark.parametrize("chunk,d", [(64, 64), (128, 128)])
def test_large_norms_take_the_exact_max_path(chunk, d):
    # qk x 256 (exact in bf16): ||q|| / sqrt(d) is far above every actual
    # score, so exponents measured from that bound underflow and the kernel
    # must redo those rows with their exact maximum.
    wl = W.small(f"large-norm-{chunk}-{d}", heads=2, seq_len=1024, d_k=d, n_hashes=2,
                 n_buckets=64, chunk_len=chunk, causal=True)
    report, g = _full_check(wl, qk_override=lambda qk: qk * 256)
    assert torch.isfinite(g["out"].float()).all()
    print(wl.name, report)


@pytest.mark.parametrize("chunk,d", [(64, 64), (128, 128)])
@pytest.mark.parametrize("causal", [True, False])
def test_mixed_norms_in_one_warp(chunk, d, causal):
    # Every third token scaled by 256 (exact in bf16): in most warps some rows
    # take their exact maximum as the exponent reference and the rest keep
    # the bound, inside the same pass (and a large-norm query's keys are
    # mostly ordinary ones, and the reverse).
    wl = W.small(f"mixed-norm-{chunk}-{d}-{int(causal)}", heads=2, seq_len=1536, d_k=d,
                 n_hashes=2, n_buckets=64, chunk_len=chunk, causal=causal)

    def scale(qk):
        f = torch.ones(qk.shape[-2], 1, dtype=qk.dtype)
        f[::3] = 256
        return qk * f

    report, g = _full_check(wl, qk_override=scale)
    assert torch.isfinite(g["out"].float()).all()
    print(wl.name, report)


def test_deterministic():
    wl = W.small("det", heads=2, seq_len=1024, n_hashes=2, n_buckets=64)
    qk, v, rot = [t.to(DEV) if t is not None else None for t in W.make_inputs(wl)]
    a = lsh.lsh_attn_forward(qk, v, rot, wl.n_hashes, wl.n_buckets, wl.chunk_len, wl.causal)
    b = lsh.lsh_attn_forward(qk, v, rot, wl.n_hashes, wl.n_buckets, wl.chunk_len, wl.causal)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_host_buffer_entry_point_matches():
    wl = W.small("host", heads=2, seq_len=512, n_hashes=2, n_buckets=16)
    qk, v, rot = W.make_inputs(wl)
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype)
    dev = torch.empty(lsh.lsh_attn_forward_host_device_bytes(shp), dtype=torch.uint8,
                      device=DEV)
    qk_h, v_h, rot_h = qk.pin_memory(), v.pin_memory(), rot.pin_memory()
    out_h = torch.empty_like(qk_h).pin_memory()
    lse_h = torch.empty(wl.batch, wl.heads, wl.seq_len, dtype=torch.float32).pin_memory()
    lsh.lsh_attn_forward_host(shp, qk_h, v_h, rot_h, out_h, lse_h, dev)
    torch.cuda.current_stream().synchronize()
    ref_out, ref_lse = lsh.lsh_attn_forward(qk.to(DEV), v.to(DEV), rot.to(DEV), wl.n_hashes,
                                            wl.n_buckets, wl.chunk_len, wl.causal)
    assert torch.equal(out_h, ref_out.cpu()) and torch.equal(lse_h, ref_lse.cpu())


def test_headline_workload_sampled():
    """L = 65536, 8 hashes, 1024 buckets (the long-text shape) at full size, in the
    configuration the benchmark times: buckets of one head in full and sampled
    rows of the others against the oracle, the sort bit for bit everywhere,
    head 0's per-round and combined outputs element by element, and sampled
    tokens of the other heads recomputed one by one."""
    wl = W.HEADLINE
    qk, v, rot = W.make_inputs(wl)
    g = _stages(wl, qk, v, rot)
    bf16 = True
    gb = g["buckets"].cpu().numpy().astype(np.int64)
    x64, v64, rot64 = P.np64(qk), P.np64(v), P.np64(rot)
    rng = np.random.default_rng(0)
    # hash: head 0 in full, 512 random rows of every other head
    ob, om = O.hash_head(x64[0, 0], rot64, wl.n_buckets)
    rep = P.check_buckets(gb[0, 0], ob, om)
    for h in range(1, wl.heads):
        rows = rng.choice(wl.seq_len, 512, replace=False)
        ob, om = O.hash_head(x64[0, h, rows], rot64, wl.n_buckets)
        P.check_buckets(gb[0, h][:, rows], ob, om)
    print("headline buckets head 0:", rep)
    # sort: every segment, bit for bit from the GPU's buckets
    gp, gu = g["perm"].cpu().numpy(), g["undo"].cpu().numpy()
    for h in range(wl.heads):
        perm, undo = O.sort_head(gb[0, h])
        np.testing.assert_array_equal(gp[0, h], perm)
        np.testing.assert_array_equal(gu[0, h], undo)
    # attention + combine: head 0 in full, element by element (all 8 rounds,
    # every token), and the median elementwise relative error of its output
    go_r, gl_r = g["o_rounds"], g["lse_rounds"]
    o_r0 = np.empty((wl.n_hashes, wl.seq_len, wl.d_k))
    l_r0 = np.empty((wl.n_hashes, wl.seq_len))
    for r in range(wl.n_hashes):
        o_r0[r], l_r0[r] = O.attend_round(x64[0, 0], v64[0, 0], gp[0, 0, r], wl.chunk_len,
                                          wl.causal)
    out0, lse0 = O.combine_head(o_r0, l_r0)
    P.check_float(go_r[0, 0].cpu()[None], o_r0[None], bf16, "o_rounds(head 0)")
    P.check_lse(gl_r[0, 0].cpu(), l_r0, bf16, "lse_rounds(head 0)")
    P.check_float(g["f_out"][0, 0].cpu()[None, None], out0[None, None], bf16, "out(head 0)")
    P.check_lse(g["f_lse"][0, 0].cpu(), lse0, bf16, "lse(head 0)")
    go0 = P.np64(g["f_out"][0, 0])
    big = np.abs(out0) > 1e-3 * np.abs(out0).max()
    med = float(np.median(np.abs(go0 - out0)[big] / np.abs(out0)[big]))
    print(f"headline out head 0: median elementwise relative error {med:.2e}")
    assert med <= 5e-3, med  # bf16 rounding of the output alone is up to 2^-9 relative
    # heads 1-7: sampled tokens (including the first, causal edge), each
    # recomputed one by one through every round and the combine
    for h in range(1, wl.heads):
        toks = np.concatenate([[0, 1, wl.seq_len - 1], rng.choice(wl.seq_len, 61, replace=False)])
        o_or, o_lr, o_out, o_lse = [], [], [], []
        for i in toks:
            o, l = O.token_rounds(x64[0, h], v64[0, h], gp[0, h], gu[0, h], wl.chunk_len,
                                  wl.causal, int(i))
            out_i, lse_i = O.combine_head(o[:, None], l[:, None])
            o_or.append(o); o_lr.append(l); o_out.append(out_i[0]); o_lse.append(lse_i[0])
        t = torch.as_tensor(toks, device=DEV)
        P.check_float(go_r[0, h][:, t].transpose(0, 1)[None, None].cpu(),
                      np.array(o_or)[None, None], bf16, "o_rounds(sampled)")
        P.check_lse(gl_r[0, h][:, t].transpose(0, 1).cpu(), np.array(o_lr), bf16,
                    "lse_rounds(sampled)")
        P.check_float(g["f_out"][0, h][t][None, None].cpu(), np.array(o_out)[None, None], bf16,
                      "out(sampled)")
        P.check_lse(g["f_lse"][0, h][t].cpu(), np.array(o_lse), bf16, "lse(sampled)")
    assert torch.equal(g["f_out"], g["out"]) and torch.equal(g["f_lse"], g["lse"])


def test_sharded_ranks_concatenate_to_the_full_pass():
    # Each "rank" runs the unchanged pass on its own (batch, head) pairs; run
    # one after another here, they must reproduce the one-call result.
    from lsh_bucketed_sparse_b200 import sharding
    wl = W.small("shards", batch=2, heads=3, seq_len=1024, n_hashes=2, n_buckets=64)
    qk, v, rot = [t.to(DEV) for t in W.make_inputs(wl)]
    full_out, full_lse = lsh.lsh_attn_forward(qk, v, rot, wl.n_hashes, wl.n_buckets,
                                              wl.chunk_len, wl.causal)
    outs, lses = [], []
    for r in range(4):
        o, l = sharding.forward_local(qk, v, rot, wl.n_hashes, wl.n_buckets, wl.chunk_len,
                                      wl.causal, r, 4)
        outs.append(o[0])
        lses.append(l[0])
    assert torch.equal(torch.cat(outs), full_out.reshape(6, *full_out.shape[2:]))
    assert torch.equal(torch.cat(lses), full_lse.reshape(6, -1))


# ---------------------------------------------------------------------------
# Duplicate-count correction (LSH_FLAG_DEDUP): few buckets, so pairs share a
# window in several rounds and N_ij > 1 is common.
DEDUP = [
    W.small("dedup-bf16-causal", heads=2, seq_len=512, n_hashes=4, n_buckets=8),
    W.small("dedup-bf16-noncausal-d128", heads=2, seq_len=256, d_k=128, n_hashes=3,
            n_buckets=4, chunk_len=32, causal=False),
    W.small("dedup-f32-causal", heads=1, seq_len=256, n_hashes=3, n_buckets=8,
            dtype=torch.float32),
    # the tensor-core attention's correction: (c, d) = (128, 64), and (64, 128)
    # non-causal with a short last chunk; more than 8 rounds fall back
    W.small("dedup-tc-c128-d64", heads=2, seq_len=1024, n_hashes=4, n_buckets=8,
            chunk_len=128),
    W.small("dedup-tc-c64-d128-noncausal", heads=2, seq_len=1000, d_k=128, n_hashes=3,
            n_buckets=8, causal=False),
    W.small("dedup-nine-rounds", heads=1, seq_len=512, n_hashes=9, n_buckets=8),
]


@pytest.mark.parametrize("wl", DEDUP, ids=[w.name for w in DEDUP])
def test_dedup_matches_oracle(wl):
    qk, v, rot = W.make_inputs(wl)
    qk_d, v_d = qk.to(DEV), v.to(DEV)
    rot_d = rot.to(DEV)
    b, inv = lsh.lsh_attn_hash(qk_d, rot_d, wl.n_buckets, wl.n_hashes)
    perm, undo, _ = lsh.lsh_attn_sort(b, wl.n_buckets)
    o_r, lse_r = lsh.lsh_attn_chunked_fwd_ex(qk_d, v_d, inv, perm, wl.chunk_len, wl.causal,
                                            undo=undo, n_buckets=wl.n_buckets)
    out, lse = lsh.lsh_attn_combine(o_r, lse_r)
    f_out, f_lse = lsh.lsh_attn_forward(qk_d, v_d, rot_d, wl.n_hashes, wl.n_buckets,
                                        wl.chunk_len, wl.causal, dedup=True)
    lsh.lsh_attn_device_check()
    # the fused pass runs the same kernels in the same order
    assert torch.equal(f_out, out) and torch.equal(f_lse, lse)
    # the correction is on: some pair shares a window in more than one round
    res0 = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal,
                     buckets=b.cpu().numpy().astype(np.int64))
    res = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal,
                    buckets=b.cpu().numpy().astype(np.int64), dedup=True)
    assert np.abs(res["lse"] - res0["lse"]).max() > 1e-3
    bf16 = wl.dtype == torch.bfloat16
    P.check_float(o_r, res["o_rounds"], bf16, "o_rounds", 3)
    P.check_lse(lse_r, res["lse_rounds"], bf16, "lse_rounds")
    P.check_float(out, res["out"], bf16, "out")
    P.check_lse(lse, res["lse"], bf16, "lse")


def test_dedup_stage_call_needs_undo():
    wl = DEDUP[0]
    qk, v, rot = [t.to(DEV) for t in W.make_inputs(wl)]
    b, inv = lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes)
    perm, _, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False)
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype, dedup=True)
    o_r = torch.empty(1, wl.heads, wl.n_hashes, wl.seq_len, wl.d_k, dtype=qk.dtype, device=DEV)
    l_r = torch.empty(1, wl.heads, wl.n_hashes, wl.seq_len, dtype=torch.float32, device=DEV)
    st = lsh.lib().lsh_attn_chunked_fwd(ctypes.byref(shp), lsh._ptr(qk), lsh._ptr(v),
                                        lsh._ptr(inv), lsh._ptr(perm), lsh._ptr(o_r),
                                        lsh._ptr(l_r), None)
    assert st == 1  # LSH_ERR_INVALID_ARG: the flag needs every round's undo
    shp.flags = lsh.FLAG_BUCKET_MASK
    st = lsh.lib().lsh_attn_chunked_fwd(ctypes.byref(shp), lsh._ptr(qk), lsh._ptr(v),
                                        lsh._ptr(inv), lsh._ptr(perm), lsh._ptr(o_r),
                                        lsh._ptr(l_r), None)
    assert st == 1  # and the bucket mask the bucket ids


def test_host_pipeline_uneven_groups():
    # 10 (batch, head) pairs go through 8 groups of one or two pairs each
    wl = W.small("host-groups", batch=2, heads=5, seq_len=256, n_hashes=2, n_buckets=16)
    qk, v, rot = W.make_inputs(wl)
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype)
    dev = torch.empty(lsh.lsh_attn_forward_host_device_bytes(shp), dtype=torch.uint8,
                      device=DEV)
    out_h = torch.empty_like(qk).pin_memory()
    lse_h = torch.empty(wl.batch, wl.heads, wl.seq_len, dtype=torch.float32).pin_memory()
    lsh.lsh_attn_forward_host(shp, qk.pin_memory(), v.pin_memory(), rot.pin_memory(), out_h,
                              lse_h, dev)
    torch.cuda.current_stream().synchronize()
    ref_out, ref_lse = lsh.lsh_attn_forward(qk.to(DEV), v.to(DEV), rot.to(DEV), wl.n_hashes,
                                            wl.n_buckets, wl.chunk_len, wl.causal)
    assert torch.equal(out_h, ref_out.cpu()) and torch.equal(lse_h, ref_lse.cpu())


# ---------------------------------------------------------------------------
# Bucket-equality mask (LSH_FLAG_BUCKET_MASK), alone and with the correction.
MASKED = [
    (W.small("bmask-bf16-causal", heads=2, seq_len=512, n_hashes=3, n_buckets=16), False),
    (W.small("bmask-f32-noncausal", heads=1, seq_len=256, n_hashes=2, n_buckets=8,
             causal=False, dtype=torch.float32), False),
    (W.small("bmask-dedup-bf16-d128", heads=2, seq_len=256, d_k=128, n_hashes=3, n_buckets=4,
             chunk_len=32, causal=True), True),
    # tensor-core attention with the mask: (c, d) = (128, 64) causal, (64, 128)
    # non-causal with a short last chunk
    (W.small("bmask-tc-c128-d64", heads=2, seq_len=1408, n_hashes=2, n_buckets=32,
             chunk_len=128), False),
    (W.small("bmask-tc-c64-d128-noncausal", heads=2, seq_len=1000, d_k=128, n_hashes=2,
             n_buckets=16, causal=False), False),
]


@pytest.mark.parametrize("wl,dedup", MASKED, ids=[w.name for w, _ in MASKED])
def test_bucket_mask_matches_oracle(wl, dedup):
    qk, v, rot = W.make_inputs(wl)
    qk_d, v_d, rot_d = qk.to(DEV), v.to(DEV), rot.to(DEV)
    b, inv = lsh.lsh_attn_hash(qk_d, rot_d, wl.n_buckets, wl.n_hashes)
    perm, undo, _ = lsh.lsh_attn_sort(b, wl.n_buckets)
    o_r, lse_r = lsh.lsh_attn_chunked_fwd_ex(qk_d, v_d, inv, perm, wl.chunk_len, wl.causal,
                                            undo=undo if dedup else None, buckets=b,
                                            n_buckets=wl.n_buckets)
    out, lse = lsh.lsh_attn_combine(o_r, lse_r)
    f_out, f_lse = lsh.lsh_attn_forward(qk_d, v_d, rot_d, wl.n_hashes, wl.n_buckets,
                                        wl.chunk_len, wl.causal, dedup=dedup, bucket_mask=True)
    lsh.lsh_attn_device_check()
    assert torch.equal(f_out, out) and torch.equal(f_lse, lse)
    gb = b.cpu().numpy().astype(np.int64)
    res0 = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal, buckets=gb, dedup=dedup)
    res = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal, buckets=gb, dedup=dedup,
                    bucket_mask=True)
    assert np.abs(res["lse"] - res0["lse"]).max() > 1e-3  # the mask drops some keys
    bf16 = wl.dtype == torch.bfloat16
    P.check_float(o_r, res["o_rounds"], bf16, "o_rounds", 3)
    P.check_lse(lse_r, res["lse_rounds"], bf16, "lse_rounds")
    P.check_float(out, res["out"], bf16, "out")
    P.check_lse(lse, res["lse"], bf16, "lse")


# ---------------------------------------------------------------------------
# Routing-style assignment (LSH_FLAG_KMEANS): argmax over given centroids.
KMEANS = [
    W.small("kmeans-bf16-causal", heads=2, seq_len=512, n_hashes=3, n_buckets=24),
    W.small("kmeans-f32-noncausal-odd", heads=1, seq_len=256, n_hashes=2, n_buckets=7,
            causal=False, dtype=torch.float32, chunk_len=32),
    W.small("kmeans-bf16-d128-wide", heads=2, seq_len=256, d_k=128, n_hashes=2, n_buckets=300),
    # multiples of 32 centroids take the tensor-core hash: 64-column rounds and
    # a ragged tile, 96-column rounds with d = 128, 512-column rounds
    W.small("kmeans-tc-p64", heads=2, seq_len=1088, n_hashes=3, n_buckets=64),
    W.small("kmeans-tc-p96-d128", heads=2, seq_len=512, d_k=128, n_hashes=2, n_buckets=96,
            chunk_len=128, causal=False),
    W.small("kmeans-tc-p512", heads=2, seq_len=640, n_hashes=2, n_buckets=512),
]


@pytest.mark.parametrize("wl", KMEANS, ids=[w.name for w in KMEANS])
def test_kmeans_assignment_matches_oracle(wl):
    qk, v, _ = W.make_inputs(wl)
    cen = W.make_centroids(wl)
    qk_d, v_d, cen_d = qk.to(DEV), v.to(DEV), cen.to(DEV)
    b, inv = lsh.lsh_attn_hash(qk_d, cen_d, wl.n_buckets, wl.n_hashes, kmeans=True)
    ob, margins = O.hash_all(qk, cen, wl.n_buckets, kmeans=True)
    report = P.check_buckets(b, ob, margins)
    assert len(np.unique(ob)) > 1
    out, lse = lsh.lsh_attn_forward(qk_d, v_d, cen_d, wl.n_hashes, wl.n_buckets, wl.chunk_len,
                                    wl.causal, kmeans=True)
    lsh.lsh_attn_device_check()
    res = O.forward(qk, v, cen, wl.n_buckets, wl.chunk_len, wl.causal,
                    buckets=b.cpu().numpy().astype(np.int64))
    bf16 = wl.dtype == torch.bfloat16
    P.check_float(out, res["out"], bf16, "out")
    P.check_lse(lse, res["lse"], bf16, "lse")
    print(wl.name, report)


@pytest.mark.parametrize("n_buckets", [64, 96, 512])
def test_kmeans_breaks_exact_ties_by_lowest_index(n_buckets):
    # centroid 3 (scaled by 4, so it usually wins) repeated at a later column
    # of the same and of another 32-column chunk: the lowest column must win
    wl = W.small(f"kmeans-ties-{n_buckets}", heads=2, seq_len=640, n_hashes=2,
                 n_buckets=n_buckets)
    qk, _, _ = W.make_inputs(wl)
    cen = W.make_centroids(wl).clone()
    cen[:, :, 3] *= 4
    for j in (7, 35, min(70, n_buckets - 1)):
        cen[:, :, j] = cen[:, :, 3]
    b, _ = lsh.lsh_attn_hash(qk.to(DEV), cen.to(DEV), wl.n_buckets, wl.n_hashes, kmeans=True)
    b = b.cpu().numpy().astype(np.int64)
    x, C = P.np64(qk), P.np64(cen)
    checked = 0
    for h in range(wl.heads):
        for r in range(wl.n_hashes):
            pr = x[0, h] @ C[r]
            top = pr.max(1, keepdims=True)
            below = np.where(pr < top, pr, -np.inf).max(1)
            clear = (top[:, 0] - below) >= 1e-5
            want = np.argmax(pr, axis=1)
            ok = b[0, h, r] == want
            assert ok[clear].all(), np.nonzero(~ok & clear)[0][:10]
            checked += int(clear.sum())
    assert checked > 0.9 * wl.heads * wl.n_hashes * wl.seq_len


# ---------------------------------------------------------------------------
# Backward with the hash and sort held fixed (the oracle differentiates its
# float64 re-statement of the forward with autograd).
BWD = [
    W.small("bwd-f32-causal", heads=2, seq_len=256, n_hashes=2, n_buckets=8,
            dtype=torch.float32),
    W.small("bwd-bf16-noncausal-d128", heads=1, seq_len=256, d_k=128, n_hashes=3,
            n_buckets=16, chunk_len=32, causal=False),
    W.small("bwd-bf16-causal-short-chunk", heads=2, seq_len=300, n_hashes=2, n_buckets=16),
    # c = 64, d = 64 take the register-tiled kernel: several (batch, head)
    # pairs without the causal mask, and one short chunk alone
    W.small("bwd-bf16-noncausal-tiled", batch=2, heads=2, seq_len=512, n_hashes=4,
            n_buckets=16, causal=False),
    W.small("bwd-bf16-one-short-chunk", heads=1, seq_len=40, n_hashes=2, n_buckets=4),
    # windows too large to stage: sums in shared memory (c = 128, d = 64), and
    # straight float32 atomics (c = 128, d = 128)
    W.small("bwd-bf16-c128-d64", heads=1, seq_len=512, n_hashes=2, n_buckets=8,
            chunk_len=128),
    W.small("bwd-bf16-c128-d128", heads=1, seq_len=512, d_k=128, n_hashes=2, n_buckets=8,
            chunk_len=128, causal=False),
]


@pytest.mark.parametrize("wl", BWD, ids=[w.name for w in BWD])
def test_backward_matches_oracle(wl):
    qk, v, rot = W.make_inputs(wl)
    g = W.make_upstream(wl)
    qk_d, v_d, rot_d, g_d = qk.to(DEV), v.to(DEV), rot.to(DEV), g.to(DEV)
    b, inv = lsh.lsh_attn_hash(qk_d, rot_d, wl.n_buckets, wl.n_hashes)
    perm, _, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False)
    o_r, l_r = lsh.lsh_attn_chunked_fwd(qk_d, v_d, inv, perm, wl.chunk_len, wl.causal,
                                        n_buckets=wl.n_buckets)
    out, lse = lsh.lsh_attn_combine(o_r, l_r)
    dqk, dv = lsh.lsh_attn_backward(qk_d, v_d, inv, perm, out, lse, g_d, wl.chunk_len,
                                    wl.causal, n_buckets=wl.n_buckets)
    lsh.lsh_attn_device_check()
    odq, odv = O.backward_all(qk, v, perm.cpu().numpy(), wl.chunk_len, wl.causal, g)
    # A row that saw only itself (lse near -1e5) weighs its own v with
    # exp(-1e5 - LSE), and float32 holds LSE there only to |LSE| 2^-24 ~ 6e-3
    # (the forward's lse carries the same rounding): those rows get 1e-2.
    ref_lse = O.forward(qk, v, rot, wl.n_buckets, wl.chunk_len, wl.causal,
                        buckets=b.cpu().numpy().astype(np.int64))["lse"]
    tol = 2e-2 if wl.dtype == torch.bfloat16 else 1e-4
    for name, gpu, ref in (("dqk", dqk, odq), ("dv", dv, odv)):
        gg = gpu.cpu().numpy().astype(np.float64)
        assert np.isfinite(gg).all(), name
        for h in range(wl.heads):
            scale = np.abs(ref[0, h]).max()
            err = np.abs(gg[0, h] - ref[0, h]).max(axis=1) / scale
            alone = ref_lse[0, h] < -1e4
            assert err[~alone].max() <= tol, f"{name} head {h}: {err[~alone].max():.3e}"
            if alone.any():
                assert err[alone].max() <= max(tol, 1e-2), f"{name} head {h} (alone)"


def test_binding_rejects_mismatched_device_tensors():
    # The library sees only pointers; the binding must refuse every tensor
    # whose extent disagrees with qk's before a pointer reaches a kernel.
    wl = W.small("shapes", heads=2, seq_len=256, n_hashes=2, n_buckets=16)
    qk, v, rot = [t.to(DEV) for t in W.make_inputs(wl)]
    B, H, L, d = qk.shape
    bad_calls = [
        lambda: lsh.lsh_attn_forward(qk, v[:, :1].contiguous(), rot, 2, 16, 64, True),
        lambda: lsh.lsh_attn_forward(qk, v, rot[:1].contiguous(), 2, 16, 64, True),
        lambda: lsh.lsh_attn_forward(qk, v, rot, 2, 32, 64, True),  # rot is n_b/2 = 8 wide
        lambda: lsh.lsh_attn_forward(qk, v, None, 2, 16, 64, True),
        lambda: lsh.lsh_attn_forward(qk, v, rot, 2, 16, 64, True,
                                     out=torch.empty(B, H, L // 2, d, dtype=qk.dtype, device=DEV)),
        lambda: lsh.lsh_attn_forward(qk, v, rot, 2, 16, 64, True,
                                     lse=torch.empty(B, H, L, dtype=torch.bfloat16, device=DEV)),
        lambda: lsh.lsh_attn_hash(qk, rot, 16, 2, kmeans=True),  # centroids are n_b wide
        lambda: lsh.lsh_attn_forward_noalloc(qk, v[..., :32].contiguous(), rot, 2, 16, 64, True),
    ]
    b, inv = lsh.lsh_attn_hash(qk, rot, 16, 2)
    perm, undo, _ = lsh.lsh_attn_sort(b, 16)
    bad_calls += [
        lambda: lsh.lsh_attn_chunked_fwd(qk, v, inv, perm[..., :128].contiguous(), 64, True),
        lambda: lsh.lsh_attn_chunked_fwd(qk, v, inv[:, :1].contiguous(), perm, 64, True),
        lambda: lsh.lsh_attn_chunked_fwd_ex(qk, v, inv, perm, 64, True,
                                            undo=undo[:, :, :1].contiguous()),
        lambda: lsh.lsh_attn_combine(torch.empty(B, H, 2, L, d, dtype=qk.dtype, device=DEV),
                                     torch.empty(B, H, 2, L // 2, device=DEV)),
    ]
    for i, call in enumerate(bad_calls):
        with pytest.raises((ValueError, TypeError)):
            call()
    lsh.lsh_attn_device_check()


def test_o_rounds_only_16_byte_aligned_gives_the_same_result():
    # The chunk-64 kernel stores o_rounds in 32-byte pieces; an o_rounds that
    # is 16-byte aligned but not 32 (allowed by the boundary) takes the
    # general kernel instead, with the same result up to its own rounding.
    wl = W.small("align16", heads=2, seq_len=1024, n_hashes=2, n_buckets=64)
    qk, v, rot = [t.to(DEV) for t in W.make_inputs(wl)]
    b, inv = lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes)
    perm, _, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False)
    o_ref, l_ref = lsh.lsh_attn_chunked_fwd(qk, v, inv, perm, wl.chunk_len, wl.causal,
                                            n_buckets=wl.n_buckets)
    n = o_ref.numel()
    raw = torch.empty(n + 64, dtype=qk.dtype, device=DEV)
    shift = (-(raw.data_ptr() // 2) % 16) + 8   # 16 bytes past a 32-byte boundary
    o_mis = raw[shift:shift + n].view_as(o_ref)
    assert o_mis.data_ptr() % 32 == 16
    l_mis = torch.empty_like(l_ref)
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype)
    lsh._check(lsh.lib().lsh_attn_chunked_fwd(
        ctypes.byref(shp), lsh._ptr(qk), lsh._ptr(v), lsh._ptr(inv), lsh._ptr(perm),
        lsh._ptr(o_mis), lsh._ptr(l_mis), lsh._stream(None)))
    torch.cuda.synchronize()
    P.check_float(o_mis.cpu(), o_ref.cpu(), True, "o_rounds (16-byte aligned)", 3)
    P.check_lse(l_mis.cpu(), l_ref.cpu(), True, "lse_rounds (16-byte aligned)")
