#!/usr/bin/env python
"""LSH attention forward throughput on B200: tokens/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores

A step is one whole forward pass (hash -> sort -> chunked attention ->
combine) over one batch of the workload, with inputs resident in HBM.  The
default workload is the long-text shape: batch 1 x 8 heads, L = 65536,
d_k = 64, bf16, 8 hashes, 1024 buckets, chunks of 64, causal.  Inputs are
seeded synthetic N(0, 1) data.  L2 is flushed (a 256 MiB write) before every
timed step; each step is timed with CUDA events on the launching stream.  At
one GPU the line also carries `per_workload`: every named workload timed the
same way (tokens/s, stage times, roofline fractions).

Multi-GPU: `--gpus N` (N > 1) started without torchrun re-launches itself
under torch.distributed.run with N local ranks, one per GPU.  The job is an
N-times larger batch of (batch, head) problems: rank r owns the r-th slice of
batch*heads pairs (the headline workload's shape, its own seeded inputs).
Hashing, sorting, the windows and the combine never cross heads, so there is
no collective on the data path ("scaling": "weak"); the NCCL process group
carries only the barriers and the max-over-ranks of the timings.

Prints ONE JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lsh_bucketed_sparse_b200 as lsh  # noqa: E402
from lsh_bucketed_sparse_b200 import workloads as W  # noqa: E402

METRIC = "LSH-attention fwd tokens/s at L=65536, 8 hashes; % of HBM/tensor roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (HGX: 8 TB/s HBM3e, 2.25 PFLOP/s dense bf16); every
# fraction is also reported against these.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# The files each stage's captured kernel is built from (its source and the
# headers it includes, paths from the repository root): a DRAM-traffic record
# in profiles/traffic.json holds only while their hash is unchanged.
CSRC = "lsh_bucketed_sparse_b200/csrc/"
_HEADERS = [CSRC + "common.cuh", CSRC + "internal.h", "include/lsh_attn.h"]
KERNEL_SOURCES = {
    "hash": [CSRC + "hash_tc.cu", CSRC + "sm100.cuh"] + _HEADERS,
    "sort": [CSRC + "sort.cu"] + _HEADERS,
    "chunked_attention": [CSRC + "attn_tc64.cu", CSRC + "sm100.cuh",
                          CSRC + "step_split.cuh"] + _HEADERS,
    "combine": [CSRC + "combine.cu"] + _HEADERS,
}


# ----------------------------------------------------------------- helpers --
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def window_pairs(wl):
    """(query, key) pairs of every window: per (batch, head) and round, chunk
    k's n_q queries meet the n_w keys of chunks k-1 and k (the first chunk
    only itself; the last chunk may be short)."""
    L, c = wl.seq_len, wl.chunk_len
    per_round = 0
    for k in range(-(-L // c)):
        nq = min(c, L - k * c)
        nw = min((k + 1) * c, L) - (k - 1) * c if k > 0 else nq
        per_round += nq * nw
    return wl.batch * wl.heads * wl.n_hashes * per_round


# fp32 lanes per SM of a B200 (4 partitions x 32) for the CUDA-core roofline
FP32_LANES_PER_SM = 128
N_SMS = 148


def stage_model(wl):
    """Algorithmic bytes (HBM) and FLOPs per launch of each stage."""
    BH, L, d, n_h, half, c = wl.batch * wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, \
        wl.n_buckets // 2, wl.chunk_len
    e = 2 if wl.dtype == torch.bfloat16 else 4
    slots = BH * n_h * L
    x = BH * L * d * e
    rot = n_h * d * half * e
    return {
        "hash": {"bytes": x + rot + 2 * slots + 4 * BH * L,
                 "flops": 2.0 * BH * L * d * half * n_h},
        "sort": {"bytes": 2 * slots + 4 * slots, "flops": 0.0},
        "chunked_attention": {"bytes": 4 * slots + n_h * 2 * x + n_h * 4 * BH * L
                              + n_h * (x + 4 * BH * L),
                              "flops": 4.0 * BH * n_h * L * (2 * c) * d},
        "combine": {"bytes": n_h * (x + 4 * BH * L) + x + 4 * BH * L, "flops": 0.0},
    }


def source_sha(stage):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[stage]:
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(stage, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        rec = t[stage]
        if rec.get("source_sha") != source_sha(stage) or rec.get("workload") != workload:
            return None
        return float(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms from before
    the timed region to its end; summary() keeps the samples whose own
    timestamps fall inside the region marked with start() / stop()."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append(ln.strip())

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except OSError:
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        t_end = time.time() + 3.0  # until nvidia-smi is producing samples
        while not self.lines and time.time() < t_end:
            time.sleep(0.01)
        return self

    def start(self):
        self.t0 = datetime.datetime.now()

    def stop(self):
        self.t1 = datetime.datetime.now()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)  # the sample that covers the end of the region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)

    def summary(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]), f[1:]))
            except ValueError:
                continue
        if not rows:
            return None
        if self.t0 is not None and self.t1 is not None:
            pad = datetime.timedelta(milliseconds=60)
            inside = [r for r in rows if self.t0 <= r[0] <= self.t1 + pad]
            rows = inside or rows
        max_mhz = max(r[2] for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4)
                          if r[3][5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max_mhz,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ distributed --
def launch_ranks(args, argv):
    """`--gpus N` without torchrun: run this script under torch.distributed.run
    with N local ranks (rendezvous on 127.0.0.1) and return its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def rank_inputs(wl, rank, world, kmeans=False):
    """Host inputs of this rank's (batch, head) slice: the headline shape,
    seeded per rank (rank 0 gets the workload's own seed)."""
    from lsh_bucketed_sparse_b200 import sharding
    a, b = sharding.head_range(wl.batch * world, wl.heads, rank, world)
    assert b - a == wl.batch * wl.heads
    seed = wl.seed + 7919 * rank
    qk, v, rot = W.make_inputs(wl, seed=seed)
    if kmeans:
        rot = W.make_centroids(wl, seed=wl.seed)
    return qk, v, rot


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------- CPU baseline --
def oracle_sample(wl, rounds, heads=1, inputs=None):
    """Time the oracle (as it stands) on the first ``heads`` (batch, head)
    pairs and ``rounds`` hashing rounds of each: hash, sort, chunked
    attention, combine.  Returns (seconds, tokens-equivalent of the full
    workload processed)."""
    import numpy as np
    from oracle import lsh_oracle as O
    qk, v, rot = W.make_inputs(wl) if inputs is None else inputs
    rounds = min(rounds, wl.n_hashes)
    heads = min(heads, wl.batch * wl.heads)
    R = O.as_f64(rot[:rounds]) if rot is not None else None
    dt = 0.0
    for h in range(heads):
        x = O.as_f64(qk.reshape(-1, wl.seq_len, wl.d_k)[h])
        vv = O.as_f64(v.reshape(-1, wl.seq_len, wl.d_k)[h])
        t0 = time.perf_counter()
        b, _ = O.hash_head(x, R, wl.n_buckets)
        perm, _ = O.sort_head(b)
        o = np.empty((rounds, wl.seq_len, wl.d_k))
        lse = np.empty((rounds, wl.seq_len))
        for r in range(rounds):
            o[r], lse[r] = O.attend_round(x, vv, perm[r], wl.chunk_len, wl.causal)
        O.combine_head(o, lse)
        dt += time.perf_counter() - t0
    frac = heads * rounds / (wl.n_hashes * wl.batch * wl.heads)  # share of the workload
    return dt, wl.tokens * frac


def cpu_threads():
    try:
        import numpy  # noqa: F401
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        n = 1
    return int(n)


def cpu_baseline(wl, rounds, heads):
    rounds = min(rounds, wl.n_hashes)
    heads = min(heads, wl.batch * wl.heads)
    dt, toks = oracle_sample(wl, rounds, heads)
    return {"value": toks / dt, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{heads} of {wl.batch * wl.heads} (batch, head) pairs of {wl.name}, "
                      f"{rounds} of {wl.n_hashes} hashing rounds each, full length: hash, sort, "
                      f"chunked attention, combine in float64 numpy; {dt:.2f} s, scaled to "
                      f"the whole workload",
            "seconds": dt, "host_cpus": len(os.sched_getaffinity(0))}


def run_reference(args, wl):
    rank, world, _ = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(wl, 1)
    times, toks = [], 0.0
    for _ in range(args.steps):
        dt, t = oracle_sample(wl, 1)
        times.append(dt)
        toks = t
    total = sum(times)
    value = toks * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(wl.describe(), sample="one (batch, head), one hashing round per step"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(),
                             "kind": "oracle",
                             "sample": "one (batch, head) and one hashing round of the workload "
                                       "per step, scaled to the whole workload"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, wl):
    """Time lsh_attn_backward (gradients of out w.r.t. qk and v with the hash
    and sort held fixed) on GPU 0; the forward stages run once beforehand."""
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    qk_h, v_h, rot_h = W.make_inputs(wl)
    qk, v = qk_h.to(dev), v_h.to(dev)
    rot = rot_h.to(dev) if rot_h is not None else None
    g = W.make_upstream(wl).to(dev)
    b, inv = lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes)
    perm, _, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False)
    o_r, l_r = lsh.lsh_attn_chunked_fwd(qk, v, inv, perm, wl.chunk_len, wl.causal,
                                        n_buckets=wl.n_buckets)
    out, lse = lsh.lsh_attn_combine(o_r, l_r)
    del o_r, l_r
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype)
    ws = torch.empty(lsh.lsh_attn_backward_workspace_size(shp), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        return lsh.lsh_attn_backward(qk, v, inv, perm, out, lse, g, wl.chunk_len, wl.causal,
                                     n_buckets=wl.n_buckets, workspace=ws)
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    ms = 0.0
    with ClockSampler(0) as clocks:
        clocks.start()
        for k in range(args.steps):
            flush.fill_(float(k))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
        clocks.stop()
    lsh.lsh_attn_device_check()
    ms_per_step = ms / args.steps
    clk = clocks.summary()
    # Algorithmic work: five d-long products per window pair (S, dP, dV, dK_hat,
    # dQ), 2 FLOPs per multiply-add, against the fp32 CUDA-core rate at the
    # clock the samples saw (nominal maximum when none were taken).
    flops = 10.0 * wl.d_k * window_pairs(wl)
    mhz = clk.get("sm_max_mhz") or 1965.0
    peak = N_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    achieved = flops / (ms_per_step / 1e3) / 1e12
    print(json.dumps({
        "metric": "LSH-attention bwd tokens/s (d qk, d v; hash and sort held fixed)",
        "value": wl.tokens / (ms_per_step / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (gradients)", "data": "synthetic",
        "config": dict(wl.describe(), l2="flushed before every timed step (256 MiB write)",
                       variant="backward: d qk, d v of out with the hash and sort held fixed "
                               "(CUDA cores: register tiles for c = 64, d = 64, else a warp "
                               "per query; float32 atomics)"),
        "roofline": {"kernel": "backward pairs", "bound": "alu", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{N_SMS} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 FLOPs x "
                                    f"{mhz:.0f} MHz (unit counts and clock, not measured)",
                     "algorithmic_flops": flops, "window_pairs": window_pairs(wl)},
        "clocks": clk, "gpu_launches": 3 * args.steps}), flush=True)
    return 0


def run_one_stage(args, wl):
    """Time one stage of the pass by itself on GPU 0 (inputs prepared by the
    earlier stages outside the timed loop).  Used to profile a single kernel."""
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    qk_h, v_h, rot_h = W.make_inputs(wl)
    qk, v = qk_h.to(dev), v_h.to(dev)
    rot = rot_h.to(dev) if rot_h is not None else None
    b, inv = lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes)
    perm = o_r = l_r = None
    if args.only_stage in ("sort", "chunked_attention", "combine"):
        perm, _, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False)
    if args.only_stage in ("chunked_attention", "combine"):
        o_r, l_r = lsh.lsh_attn_chunked_fwd(qk, v, inv, perm, wl.chunk_len, wl.causal,
                                            n_buckets=wl.n_buckets)
    if args.only_stage != "chunked_attention":
        del v
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    calls = {
        "hash": lambda: lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes),
        "sort": lambda: lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=False),
        "chunked_attention": lambda: lsh.lsh_attn_chunked_fwd(
            qk, v, inv, perm, wl.chunk_len, wl.causal, n_buckets=wl.n_buckets),
        "combine": lambda: lsh.lsh_attn_combine(o_r, l_r),
    }
    fn = calls[args.only_stage]
    for _ in range(args.warmup):
        flush.fill_(1.0)
        fn()
    ms = 0.0
    for k in range(args.steps):
        flush.fill_(float(k))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms += e0.elapsed_time(e1)
    lsh.lsh_attn_device_check()
    m = stage_model(wl)[args.only_stage]
    sec = ms / args.steps / 1e3
    print(json.dumps({"stage": args.only_stage, "workload": wl.name, "ms": sec * 1e3,
                      "GB/s": m["bytes"] / sec / 1e9, "TFLOP/s": m["flops"] / sec / 1e12}),
          flush=True)
    return 0


# -------------------------------------------------------------- measuring --
def step_fn(wl, qk, v, rot, dev, args):
    """One fused forward (lsh_attn_forward) over device inputs, outputs and
    workspace allocated here."""
    shp = lsh.make_shape(wl.batch, wl.heads, wl.seq_len, wl.d_k, wl.n_hashes, wl.n_buckets,
                         wl.chunk_len, wl.causal, wl.dtype, dedup=args.dedup,
                         bucket_mask=args.bucket_mask, kmeans=args.kmeans)
    ws = torch.empty(lsh.lsh_attn_forward_workspace_size(shp), dtype=torch.uint8, device=dev)
    out = torch.empty_like(qk)
    lse = torch.empty(wl.batch, wl.heads, wl.seq_len, dtype=torch.float32, device=dev)

    def step():
        lsh.lsh_attn_forward(qk, v, rot, wl.n_hashes, wl.n_buckets, wl.chunk_len, wl.causal,
                             workspace=ws, out=out, lse=lse, dedup=args.dedup,
                             bucket_mask=args.bucket_mask, kmeans=args.kmeans)
    return step, shp


def stage_times(wl, qk, v, rot, stream, flush, n, args):
    """Device time of each stage through the four stage calls (the same
    kernels as the fused call), averaged over n passes after two warm-ups."""
    stage_ms = {k: 0.0 for k in ("hash", "sort", "chunked_attention", "combine")}
    for it in range(n + 2):
        flush.fill_(2.0)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record(stream)
        b, inv = lsh.lsh_attn_hash(qk, rot, wl.n_buckets, wl.n_hashes, kmeans=args.kmeans)
        ev[1].record(stream)
        perm, undo, _ = lsh.lsh_attn_sort(b, wl.n_buckets, want_undo=args.dedup)
        ev[2].record(stream)
        if args.dedup or args.bucket_mask:
            o_r, l_r = lsh.lsh_attn_chunked_fwd_ex(
                qk, v, inv, perm, wl.chunk_len, wl.causal, undo=undo if args.dedup else None,
                buckets=b if args.bucket_mask else None, n_buckets=wl.n_buckets)
        else:
            o_r, l_r = lsh.lsh_attn_chunked_fwd(qk, v, inv, perm, wl.chunk_len, wl.causal,
                                                n_buckets=wl.n_buckets)
        ev[3].record(stream)
        lsh.lsh_attn_combine(o_r, l_r)
        ev[4].record(stream)
        torch.cuda.synchronize()
        if it >= 2:
            for j, k in enumerate(stage_ms):
                stage_ms[k] += ev[j].elapsed_time(ev[j + 1]) / n
        del b, inv, perm, undo, o_r, l_r
    return stage_ms


def roofline_of(wl, stage_ms, ms_per_step, pk):
    """Roofline of the dominant stage (its algorithmic bytes or FLOPs over its
    device time, against the measured or fallback peak and the nominal one)
    and of the whole pass (max of bytes / HBM peak and FLOPs / tensor peak)."""
    model = stage_model(wl)
    dom = max(stage_ms, key=stage_ms.get)
    sec = stage_ms[dom] / 1e3
    m = model[dom]
    if m["flops"] / (pk["bf16_tflops_sustained"] * 1e12) > m["bytes"] / (pk["hbm_gbs"] * 1e9):
        achieved, peak, nominal, unit, bound = m["flops"] / sec / 1e12, \
            pk["bf16_tflops_sustained"], NOMINAL_PEAKS["bf16_tflops"], "TFLOP/s", "tensor"
    else:
        achieved, peak, nominal, unit, bound = m["bytes"] / sec / 1e9, pk["hbm_gbs"], \
            NOMINAL_PEAKS["hbm_gbs"], "GB/s", "hbm"
    r = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": achieved / peak, "peak_source": pk["source"],
         "peak_nominal": nominal, "frac_nominal": achieved / nominal,
         "algorithmic_bytes": m["bytes"], "algorithmic_flops": m["flops"],
         "stage_ms": stage_ms}
    total_bytes = sum(x["bytes"] for x in model.values())
    total_flops = sum(x["flops"] for x in model.values())
    t_roof = max(total_bytes / (pk["hbm_gbs"] * 1e9), total_flops / (pk["bf16_tflops"] * 1e12))
    t_nom = max(total_bytes / (NOMINAL_PEAKS["hbm_gbs"] * 1e9),
                total_flops / (NOMINAL_PEAKS["bf16_tflops"] * 1e12))
    r["pass_roofline_ms"] = t_roof * 1e3
    r["pass_frac"] = t_roof * 1e3 / ms_per_step
    r["pass_roofline_ms_nominal"] = t_nom * 1e3
    r["pass_frac_nominal"] = t_nom * 1e3 / ms_per_step
    return r


def per_workload(dev, stream, flush, steps, args, pk):
    """Every named workload on this GPU: the fused pass timed as the headline
    (L2 flushed before each step, CUDA events), tokens/s, stage times and the
    roofline fractions."""
    rows = []
    for wl in W.WORKLOADS:
        qk_h, v_h, rot_h = W.make_inputs(wl)
        qk, v = qk_h.to(dev), v_h.to(dev)
        rot = rot_h.to(dev) if rot_h is not None else None
        step, _ = step_fn(wl, qk, v, rot, dev, args)
        for _ in range(3):
            flush.fill_(1.0)
            step()
        ms = 0.0
        for k in range(steps):
            flush.fill_(float(k))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
        ms /= steps
        st = stage_times(wl, qk, v, rot, stream, flush, min(steps, 5), args)
        lsh.lsh_attn_device_check()
        roof = roofline_of(wl, st, ms, pk)
        rows.append({"workload": wl.name, "value": wl.tokens / (ms / 1e3), "unit": UNIT,
                     "ms_per_step": ms, "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32",
                     "config": wl.describe(), "roofline": roof})
        del qk, v, rot, step
    return rows


# ----------------------------------------------------------------- main --
def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.HEADLINE.name, choices=list(W.BY_NAME))
    ap.add_argument("--cpu-rounds", type=int, default=8,
                    help="hashing rounds of each sampled head the CPU baseline times")
    ap.add_argument("--cpu-heads", type=int, default=2,
                    help="(batch, head) pairs the CPU baseline times (about 10 s on 16 "
                         "threads for the long-text workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-workload table of the one-GPU line")
    ap.add_argument("--dedup", action="store_true",
                    help="the pass with the duplicate-count correction; a separate "
                         "measurement, not the headline")
    ap.add_argument("--bucket-mask", action="store_true",
                    help="the pass with the bucket-equality mask; a separate measurement, not "
                         "the headline")
    ap.add_argument("--kmeans", action="store_true",
                    help="routing-style assignment to n_buckets centroids instead of the "
                         "random-rotation hash; a separate measurement")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (hash and sort fixed) on the workload; a "
                         "separate measurement, not the headline")
    ap.add_argument("--only-stage", choices=["hash", "sort", "chunked_attention", "combine"],
                    help="time one stage call alone (for profiling); prints its own JSON line")
    args = ap.parse_args(argv)
    wl = W.BY_NAME[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.only_stage:
        return run_one_stage(args, wl)
    if args.backward:
        return run_backward(args, wl)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return launch_ranks(args, argv)
    if world_env is not None and int(world_env) != args.gpus:
        print(f"bench.py: WORLD_SIZE={world_env} but --gpus {args.gpus}", file=sys.stderr)
        return 2

    rank, world, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    qk_h, v_h, rot_h = rank_inputs(wl, rank, world, kmeans=args.kmeans)
    qk, v = qk_h.to(dev), v_h.to(dev)
    rot = rot_h.to(dev) if rot_h is not None else None
    step, shp = step_fn(wl, qk, v, rot, dev, args)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    lsh.lsh_attn_device_check()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    launches0 = lsh.lsh_attn_kernel_launches()
    with ClockSampler(local) as clocks:
        clocks.start()
        for k in range(args.steps):
            flush.fill_(float(k))
            starts[k].record(stream)
            step()
            ends[k].record(stream)
        torch.cuda.synchronize()
        clocks.stop()
    launches = lsh.lsh_attn_kernel_launches() - launches0
    barrier(world)
    lsh.lsh_attn_device_check()
    ms_local = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms_total = max_over_ranks(ms_local, world)
    ms_per_step = ms_total / args.steps
    value = world * wl.tokens * args.steps / (ms_total / 1e3)

    stage_ms = stage_times(wl, qk, v, rot, stream, flush, min(args.steps, 10), args)

    # End to end through the host-buffer entry point: every step copies its
    # inputs in from pinned host memory and its outputs back, inside the
    # timed region.  Steps alternate between two caller streams, each with
    # its own device buffer and host output buffers (as a caller streaming
    # batches would), so one step's copies in may start while the previous
    # step's last heads are still computed and copied out.
    pin = [t.pin_memory() if t is not None else None for t in (qk_h, v_h, rot_h)]
    n_dev = lsh.lsh_attn_forward_host_device_bytes(shp)
    lanes = []
    for _ in range(2):
        lanes.append({
            "stream": torch.cuda.Stream(device=dev),
            "out": torch.empty_like(qk_h).pin_memory(),
            "lse": torch.empty(wl.batch, wl.heads, wl.seq_len, dtype=torch.float32).pin_memory(),
            "dbuf": torch.empty(n_dev, dtype=torch.uint8, device=dev),
        })

    def e2e_step(k):
        ln = lanes[k % 2]
        lsh.lsh_attn_forward_host(shp, pin[0], pin[1], pin[2], ln["out"], ln["lse"], ln["dbuf"],
                                  stream=ln["stream"])

    for k in range(4):
        e2e_step(k)
    e2e_steps = min(args.steps, 10)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for ln in lanes:
        ln["stream"].wait_stream(stream)
    for k in range(e2e_steps):
        e2e_step(k)
    for ln in lanes:
        stream.wait_stream(ln["stream"])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in pin if t is not None)
    d2h = lanes[0]["out"].numel() * lanes[0]["out"].element_size() + lanes[0]["lse"].numel() * 4
    del pin, lanes

    pk = peaks()
    roofline = roofline_of(wl, stage_ms, ms_per_step, pk)
    roofline["traffic"] = traffic_for(roofline["kernel"], wl.name)

    variant = args.dedup or args.bucket_mask or args.kmeans
    table = None
    if rank == 0 and world == 1 and not variant and not args.no_per_workload:
        del qk, v, rot, step
        table = per_workload(dev, stream, flush, min(args.steps, 20), args, pk)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not variant:
        cpu = cpu_baseline(wl, args.cpu_rounds, args.cpu_heads)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": dict(wl.describe(), l2="flushed before every timed step (256 MiB write)",
                           parallelism=(f"{world} GPU(s): rank r owns the r-th slice of "
                                        f"{wl.batch * world}x{wl.heads} (batch, head) problems; "
                                        "no collective on the data path"),
                           **({"variant": " + ".join(
                               (["duplicate-count correction (LSH_FLAG_DEDUP)"] if args.dedup
                                else []) +
                               (["bucket-equality mask (LSH_FLAG_BUCKET_MASK)"]
                                if args.bucket_mask else []) +
                               (["routing-style assignment to n_buckets centroids "
                                 "(LSH_FLAG_KMEANS)"] if args.kmeans else []))}
                              if variant else {})),
            "clocks": clocks.summary(),
            "e2e": {"value": world * wl.tokens / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            # kernels this library launched during the timed steps (host count)
            "gpu_launches": launches,
            "roofline": roofline,
            "cpu_baseline": cpu,
        }
        if table is not None:
            line["per_workload"] = table
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
