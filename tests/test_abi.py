"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host (no GPU needed: validation runs before
any CUDA call, and nothing here launches a kernel)."""

import ctypes

import pytest

import lsh_bucketed_sparse_b200 as lsh
from lsh_bucketed_sparse_b200 import build as B


@pytest.fixture(scope="module")
def L():
    B.build()
    return lsh.lib()


def test_exports_every_declared_symbol(L):
    names = lsh.declared_symbols()
    assert {"lsh_attn_hash", "lsh_attn_sort", "lsh_attn_chunked_fwd", "lsh_attn_combine",
            "lsh_attn_forward", "lsh_attn_forward_workspace_size"} <= set(names), names
    for n in names:
        assert hasattr(L, n), n
    assert L.lsh_attn_version() == 1


def test_status_strings(L):
    for code, text in [(0, b"ok"), (1, b"invalid argument"), (3, b"workspace too small"),
                       (5, b"device wait timed out")]:
        assert L.lsh_attn_status_string(code) == text


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)
STREAM = ctypes.c_void_p(0)


def shape(**kw):
    base = dict(batch=1, heads=2, seq_len=256, d_k=64, n_hashes=2, n_buckets=16, chunk_len=64,
                causal=1, dtype=lsh.BF16, portable=False)
    base.update(kw)
    return lsh.make_shape(base["batch"], base["heads"], base["seq_len"], base["d_k"],
                          base["n_hashes"], base["n_buckets"], base["chunk_len"], base["causal"],
                          base["dtype"], base["portable"])


def fwd(L, shp, ws_bytes=1 << 40, rot=FAKE, ws=FAKE, qk=FAKE):
    return L.lsh_attn_forward(ctypes.byref(shp), qk, FAKE, rot, FAKE, FAKE, ws, ws_bytes, STREAM)


@pytest.mark.parametrize("kw", [
    dict(seq_len=0), dict(chunk_len=-1),
    dict(d_k=60), dict(d_k=264), dict(d_k=0),
    dict(n_buckets=7), dict(n_buckets=0), dict(n_buckets=65536),
    dict(n_hashes=0), dict(batch=0), dict(chunk_len=0),
    dict(dtype=7),
])
def test_bad_shape_is_rejected(L, kw):
    assert fwd(L, shape(**kw)) == 1
    assert L.lsh_attn_last_error()


def test_chunk_len_need_not_divide_seq_len(L):
    # the last chunk of the sorted order is short; the workspace covers it
    shp = shape(seq_len=250)
    n = ctypes.c_size_t()
    assert L.lsh_attn_forward_workspace_size(ctypes.byref(shp), ctypes.byref(n)) == 0
    assert n.value > 0


def test_bad_causal_flag_is_rejected(L):
    shp = shape()
    shp.causal = 2
    assert fwd(L, shp) == 1


def test_bad_pointers_are_rejected(L):
    assert fwd(L, shape(), qk=None) == 1
    assert fwd(L, shape(), qk=MISALIGNED) == 1
    assert fwd(L, shape(), rot=None) == 1                       # n_b > 1 needs rotations
    assert fwd(L, shape(n_buckets=1), rot=FAKE) == 1            # n_b == 1 forbids them
    assert fwd(L, shape(), ws=ctypes.c_void_p((1 << 20) + 16)) == 1  # not 256-aligned
    assert b"aligned" in L.lsh_attn_last_error()


def test_workspace_size_and_too_small(L):
    shp = shape()
    need = lsh.lsh_attn_forward_workspace_size(shp)
    slots = 1 * 2 * 2 * 256
    assert need >= slots * (2 + 4 + 64 * 2 + 4) + 2 * 256 * 4
    assert fwd(L, shp, ws_bytes=need - 1) == 3
    assert lsh.lsh_attn_forward_host_device_bytes(shp) > need


def test_unknown_flag_rejected(L):
    shp = shape()
    shp.flags = 16  # bits 0-3 are LSH_FLAG_PORTABLE, _DEDUP, _BUCKET_MASK, _KMEANS
    assert fwd(L, shp) == 1


def test_stage_calls_validate(L):
    shp = shape()
    assert L.lsh_attn_hash(ctypes.byref(shp), FAKE, FAKE, None, FAKE, STREAM) == 1
    assert L.lsh_attn_sort(ctypes.byref(shp), FAKE, None, None, None, FAKE, 1 << 30, STREAM) == 1
    # no workspace, or one that is too small
    assert L.lsh_attn_sort(ctypes.byref(shp), FAKE, FAKE, None, None, None, 1 << 30, STREAM) == 1
    need = ctypes.c_size_t()
    assert L.lsh_attn_sort_workspace_size(ctypes.byref(shp), ctypes.byref(need)) == 0
    assert need.value > 0
    assert L.lsh_attn_sort(ctypes.byref(shp), FAKE, FAKE, None, None, FAKE, need.value - 16,
                           STREAM) == 3  # LSH_ERR_WORKSPACE
    assert b"sort workspace" in L.lsh_attn_last_error()
    assert L.lsh_attn_chunked_fwd(ctypes.byref(shp), FAKE, FAKE, FAKE, MISALIGNED, FAKE, FAKE,
                                  STREAM) == 1
    assert L.lsh_attn_combine(ctypes.byref(shp), FAKE, FAKE, FAKE, None, STREAM) == 1
    assert L.lsh_attn_hash(None, FAKE, FAKE, FAKE, FAKE, STREAM) == 1


def test_binding_fails_loudly_without_gpu_tensors():
    import torch
    with pytest.raises(ValueError):
        lsh.lsh_attn_forward(torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16),
                             torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16), None, 1, 1, 64, True)


def test_binding_checks_host_tensor_shapes_before_any_copy():
    # The library sees only pointers, so the binding checks every extent: a
    # host tensor of the wrong shape, dtype or a missing rotation table raises
    # before the device buffer is even looked at (here it is not a CUDA tensor).
    import torch
    shp = lsh.make_shape(1, 2, 128, 64, 2, 16, 64, True, torch.bfloat16)
    x = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    rot = torch.zeros(2, 64, 8, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 128, dtype=torch.float32)
    cases = [
        (x, x, rot, x, torch.zeros(1, 2, 64, dtype=torch.float32)),    # lse too short
        (x, x[:, :1].contiguous(), rot, x, lse),                       # v has one head
        (x, x, torch.zeros(2, 64, 16, dtype=torch.bfloat16), x, lse),  # rotations n_b wide
        (x, x, None, x, lse),                                          # rotations missing
        (x, x, rot, torch.zeros(1, 2, 128, 64), lse),                  # out in float32
    ]
    for qk_h, v_h, rot_h, out_h, lse_h in cases:
        with pytest.raises((ValueError, TypeError)) as ei:
            lsh.lsh_attn_forward_host(shp, qk_h, v_h, rot_h, out_h, lse_h, "not a tensor")
        assert "device_buffer" not in str(ei.value)
    km = lsh.make_shape(1, 2, 128, 64, 2, 16, 64, True, torch.bfloat16, kmeans=True)
    with pytest.raises(ValueError, match="rot_host"):  # centroids are [n_h, d, n_b]
        lsh.lsh_attn_forward_host(km, x, x, rot, x, lse, "not a tensor")


def _flags(shp, flags):
    shp.flags = flags
    return shp


def test_backward_validates_before_launching(L):
    shp = shape()
    need = lsh.lsh_attn_backward_workspace_size(shp)
    assert need >= 2 * 256 * (4 + 64 * 4)  # delta and dk_hat, float32

    def bwd(s=shp, ws=FAKE, ws_bytes=need, dout=FAKE):
        return L.lsh_attn_backward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, dout,
                                   FAKE, FAKE, ws, ws_bytes, STREAM)
    assert bwd(s=_flags(shape(), lsh.FLAG_DEDUP)) == 2          # variants: unsupported
    assert bwd(dout=None) == 1
    assert bwd(ws=ctypes.c_void_p((1 << 20) + 16)) == 1          # not 256-aligned
    assert bwd(ws_bytes=need - 1) == 3


def test_variant_stage_call_needs_its_inputs(L):
    ded = _flags(shape(), lsh.FLAG_DEDUP)
    msk = _flags(shape(), lsh.FLAG_BUCKET_MASK)
    # the plain stage call refuses variant flags
    assert L.lsh_attn_chunked_fwd(ctypes.byref(ded), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  STREAM) == 1
    assert b"_ex" in L.lsh_attn_last_error()
    # the _ex call needs undo for the correction and buckets for the mask
    assert L.lsh_attn_chunked_fwd_ex(ctypes.byref(ded), FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                                     FAKE, STREAM) == 1
    assert L.lsh_attn_chunked_fwd_ex(ctypes.byref(msk), FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                                     FAKE, STREAM) == 1


def test_host_entry_point_validates_before_any_copy(L):
    shp = shape()
    need = lsh.lsh_attn_forward_host_device_bytes(shp)

    def host(qk=FAKE, rot=FAKE, dev=FAKE, n=need, s=shp):
        return L.lsh_attn_forward_host(ctypes.byref(s), qk, FAKE, rot, FAKE, FAKE, dev, n, STREAM)
    assert host(qk=None) == 1
    assert host(rot=None) == 1                                    # n_b > 1 needs rotations
    assert host(s=shape(n_buckets=1)) == 1                        # n_b == 1 forbids them
    assert host(dev=ctypes.c_void_p((1 << 20) + 16)) == 1         # not 256-aligned
    assert host(n=need - 1) == 3


def test_kmeans_takes_any_bucket_count_from_two(L):
    n = ctypes.c_size_t()
    for nb, ok in [(7, True), (2, True), (32768, True), (1, False), (32769, False)]:
        shp = _flags(shape(n_buckets=nb), lsh.FLAG_KMEANS)
        st = L.lsh_attn_forward_workspace_size(ctypes.byref(shp), ctypes.byref(n))
        assert (st == 0) == ok, nb
    # without the flag an odd count is refused
    assert L.lsh_attn_forward_workspace_size(ctypes.byref(shape(n_buckets=7)),
                                             ctypes.byref(n)) == 1
