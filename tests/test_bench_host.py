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


def test_gpus_without_torchrun_relaunches_under_torch_distributed_run(monkeypatch):
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    assert bench.main(["--gpus", "4", "--steps", "2", "--warmup", "3"]) == 0
    (cmd,) = calls
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-6:] == [bench.os.path.abspath(bench.__file__), "--gpus", "4", "--steps", "2",
                        "--warmup", "3"][-6:]


def test_world_size_must_match_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--gpus", "4", "--warmup", "3"]) == 2


def test_rank_inputs_are_the_headline_shape_with_per_rank_seeds():
    wl = W.small("ranks", batch=1, heads=2, seq_len=128, n_hashes=2, n_buckets=8)
    a = bench.rank_inputs(wl, 0, 2)
    b = bench.rank_inputs(wl, 1, 2)
    assert a[0].shape == b[0].shape == (1, 2, 128, 64)
    assert not bool((a[0] == b[0]).all())
    same = W.make_inputs(wl)
    assert bool((a[0] == same[0]).all()) and bool((a[1] == same[1]).all())


def test_roofline_of_uses_the_dominant_stage_and_both_peak_sets():
    wl = W.HEADLINE
    stage_ms = {"hash": 0.2, "sort": 0.05, "chunked_attention": 0.5, "combine": 0.1}
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0,
          "source": "test"}
    r = bench.roofline_of(wl, stage_ms, 0.85, pk)
    m = bench.stage_model(wl)["chunked_attention"]
    assert r["kernel"] == "chunked_attention" and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(m["bytes"] / 0.5e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0)
    assert r["frac_nominal"] == pytest.approx(r["achieved"] / 8000.0)
    total = sum(x["bytes"] for x in bench.stage_model(wl).values())
    assert r["pass_roofline_ms"] == pytest.approx(total / 6000e9 * 1e3)
    assert r["pass_frac"] == pytest.approx(r["pass_roofline_ms"] / 0.85)
    assert r["pass_frac_nominal"] < r["pass_frac"]
