"""lsh_attn_forward_noalloc: the forward pass for callers that cannot allocate.

Some callers of this library can neither call cudaMalloc nor hand over a
workspace: a plugin inside a host framework that owns all device memory
through its own pool and gives the plugin only its input and output buffers,
or a latency-critical path where cudaMalloc (which can synchronise the whole
device and take an unpredictable time) is not allowed.  For them the library
keeps the forward pass's intermediates in a scratch array of its own.

The GPU test calls the entry point through the C ABI twice in a row, with
different inputs and shapes so that anything left in the shared scratch by
the first call would show in the second, and checks each result against
lsh_attn_forward (the workspace entry point).  Both entry points launch the
same kernels in the same order on the same inputs, so the results must be
bit-identical.
This file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

import lsh_bucketed_sparse_b200 as lsh
from lsh_bucketed_sparse_b200 import workloads as W


def _noalloc(wl, qk, v, rot):
    """One call of lsh_attn_forward_noalloc through ctypes."""
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype)
    out = torch.empty_like(qk)
    lse = torch.empty(wl.batch, wl.heads, wl.seq_len, dtype=torch.float32, device=qk.device)
    st = lsh.lib().lsh_attn_forward_noalloc(
        ctypes.byref(shp), ctypes.c_void_p(qk.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        None if rot is None else ctypes.c_void_p(rot.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lsh.lib().lsh_attn_last_error()
    return out, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    calls = [
        W.small("noalloc-a", batch=1, heads=4, seq_len=2048, n_hashes=4, n_buckets=64, seed=21),
        W.small("noalloc-b", batch=2, heads=2, seq_len=1024, d_k=128, n_hashes=2, n_buckets=32,
                chunk_len=128, causal=False, seed=22),
    ]
    for wl in calls:
        shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                             wl.chunk_len, wl.causal, wl.dtype)
        assert lsh.lsh_attn_forward_workspace_size(shp) <= lsh.NOALLOC_SCRATCH_BYTES
        qk, v, rot = [t.cuda() if t is not None else None for t in W.make_inputs(wl)]
        out, lse = _noalloc(wl, qk, v, rot)
        ref_out, ref_lse = lsh.lsh_attn_forward(qk, v, rot, wl.n_hashes, wl.n_buckets,
                                                wl.chunk_len, wl.causal)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), f"{wl.name}: out differs from lsh_attn_forward"
        assert torch.equal(lse, ref_lse), f"{wl.name}: lse differs from lsh_attn_forward"
    lsh.lsh_attn_device_check()


def test_noalloc_refuses_problems_beyond_its_scratch():
    # Checked on the host before anything touches the GPU.
    shp = lsh.make_shape(1, 8, 65536, 64, 8, 1024, 64, True, torch.bfloat16)
    assert lsh.lsh_attn_forward_workspace_size(shp) > lsh.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    st = lsh.lib().lsh_attn_forward_noalloc(ctypes.byref(shp), fake, fake, fake, fake, fake,
                                            ctypes.c_void_p(0))
    assert st == 3  # LSH_ERR_WORKSPACE
    assert b"scratch" in lsh.lib().lsh_attn_last_error()
