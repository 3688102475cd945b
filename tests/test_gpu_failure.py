"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait inside the tensor-core kernels gives up after a time limit; the
kernel then records an error word, every role of the CTA leaves its loop,
work already in flight lands, and the kernel returns, so the context stays
usable.  lsh_attn_test_hash_first_wait(0) makes the first wait of the hash's
MMA thread give up at once (before any MMA is issued); lsh_attn_device_check
must then report LSH_ERR_DEVICE_TIMEOUT, and the next normal call on the same
stream must produce the oracle's buckets.
"""

import numpy as np
import pytest
import torch

import lsh_bucketed_sparse_b200 as lsh
from lsh_bucketed_sparse_b200 import workloads as W

import parity as P

LSH_ERR_DEVICE_TIMEOUT = 5


@pytest.mark.gpu
def test_hash_wait_that_runs_out_reports_timeout_and_next_call_is_clean():
    from oracle import lsh_oracle as O
    # bf16, d = 64, 64 projections per round: the tensor-core hash
    wl = W.small("timeout", batch=1, heads=2, seq_len=1024, n_hashes=2, n_buckets=128, seed=31)
    qk, _, rot = W.make_inputs(wl)
    qd, rd = qk.cuda(), rot.cuda()
    lib = lsh.lib()
    lsh.lsh_attn_device_check()  # nothing pending from earlier tests
    prev = lib.lsh_attn_test_hash_first_wait(0)
    try:
        lsh.lsh_attn_hash(qd, rd, wl.n_buckets, wl.n_hashes)
        with pytest.raises(lsh.LshError) as err:
            lsh.lsh_attn_device_check()
        assert err.value.status == LSH_ERR_DEVICE_TIMEOUT
        assert b"bounded wait" in lib.lsh_attn_last_error()
    finally:
        assert lib.lsh_attn_test_hash_first_wait(prev) == 0
    # the error word was cleared by the check; the context is usable
    buckets, inv_norm = lsh.lsh_attn_hash(qd, rd, wl.n_buckets, wl.n_hashes)
    lsh.lsh_attn_device_check()
    ob, margins = O.hash_all(qk, rot, wl.n_buckets)
    P.check_buckets(buckets, ob, margins)
    norms = np.linalg.norm(qk.to(torch.float64).numpy(), axis=-1)
    np.testing.assert_allclose(inv_norm.cpu().numpy(), 1.0 / norms, rtol=1e-5)


def test_first_wait_hook_round_trips():
    # host side only: the hook returns the previous limit (2 s by default)
    lib = lsh.lib()
    prev = lib.lsh_attn_test_hash_first_wait(12345)
    assert prev == 2_000_000_000
    assert lib.lsh_attn_test_hash_first_wait(prev) == 12345
