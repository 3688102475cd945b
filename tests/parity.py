"""Comparison rules between the CUDA path and the fp64 oracle.

* Bucket ids: equal everywhere except positions whose fp64 margin (largest
  minus second largest entry of [xR; -xR]) is below NEAR_TIE; those are
  counted and reported.
* Sort (perm, undo, counts): the oracle is re-run from the GPU's bucket ids
  and must match bit for bit.
* Floating-point outputs, compared after feeding the GPU buckets back:
  float32 inputs  -> max |diff| <= 1e-4 on out/o_rounds and on lse;
  bfloat16 inputs -> per (b, h) slab, max |diff| / max |oracle| <= 2e-2 on
                     out/o_rounds; |diff lse| <= 2e-2 * max(1, |lse|).
"""

import numpy as np
import torch

NEAR_TIE = 1e-5
F32_ATOL = 1e-4
BF16_REL = 2e-2


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy() if isinstance(t, torch.Tensor) \
        else np.asarray(t, np.float64)


def check_buckets(gpu, oracle, margins):
    gpu = np.asarray(gpu.cpu().numpy() if isinstance(gpu, torch.Tensor) else gpu, np.int64)
    bad = gpu != oracle
    near = margins < NEAR_TIE
    hard = bad & ~near
    assert not hard.any(), (
        f"{int(hard.sum())} bucket mismatches with margin >= {NEAR_TIE}; "
        f"first at {np.argwhere(hard)[:5].tolist()}, margins {margins[hard][:5]}")
    return {"mismatch": int(bad.sum()), "near_ties": int(near.sum()), "total": int(bad.size)}


def check_float(gpu, oracle, bf16, what, slab_axes=2):
    """gpu/oracle: arrays [B, H, ...]; tolerance per (b, h) slab for bf16."""
    g, o = np64(gpu), np64(oracle)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    diff = np.abs(g - o)
    if not bf16:
        worst = float(diff.max()) if diff.size else 0.0
        assert worst <= F32_ATOL, f"{what}: max abs diff {worst:.3e} > {F32_ATOL}"
        return worst
    lead = g.shape[:slab_axes]
    d2 = diff.reshape(*lead, -1).max(axis=-1)
    o2 = np.abs(o).reshape(*lead, -1).max(axis=-1)
    rel = d2 / np.maximum(o2, 1e-30)
    worst = float(rel.max())
    assert worst <= BF16_REL, f"{what}: slab max|diff|/max|oracle| {worst:.3e} > {BF16_REL}"
    return worst


def check_lse(gpu, oracle, bf16, what):
    g, o = np64(gpu), np64(oracle)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    diff = np.abs(g - o)
    if not bf16:
        worst = float(diff.max())
        # fp32 rounding of a value near -1e5 (a token that saw only itself) is 4e-3 absolute
        tol = np.maximum(F32_ATOL, 1e-7 * np.abs(o))
        assert (diff <= tol).all(), f"{what}: max abs diff {worst:.3e}"
        return worst
    tol = BF16_REL * np.maximum(1.0, np.abs(o))
    assert (diff <= tol).all(), f"{what}: max abs diff {float(diff.max()):.3e}"
    return float((diff / np.maximum(1.0, np.abs(o))).max())
