#!/usr/bin/env python
"""Benchmark: linear-attention forward tokens/s and achieved HBM GB/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--shard heads|seq] [--no-extras]

Default workload (one step = one pass of the whole forward path, phi feature map, chunk
aggregates, inter-chunk prefix and intra-chunk output, over one batch): the long-context
causal forward, B=1, H=32, n=131072, d=D=128, bf16 I/O, fp32 state, inputs N(0,1)/sqrt(d)
seed 3.  Inputs (3.2 GB) and output (1.1 GB) are larger than the 126 MB L2, so no flush
is needed between timed steps.

Multi-GPU (torchrun, one process per GPU): heads are independent, so each rank runs its
own batch element of the workload (batch index = rank) with no data-path collective;
value = all ranks' tokens / the max over ranks of the device time ("scaling": "weak").
``--shard seq`` instead splits one sequence per head over the ranks: each rank computes its
block's state, the ranks all-gather the block states once, and each continues its block
from the states before it ("scaling": "strong"; linear_attention_linattn_b200.seqshard).

"e2e" is the same step through the C entry point on pinned host buffers
(linattn_forward_host): every step copies q, k, v in and the output back, in head groups whose
copies overlap one another's work; the host link bounds it.

At N=1 the line also carries the decode step (256 x 32 states, d = 128, 512 steps), the
batched 8x16x8192x64 forward (both modes) and the small latency cases under "extras", and
the oracle's throughput on a bounded sample under "cpu_baseline".

``--impl reference`` times the float64 CPU oracle (the reference implementation for
this library) on the same workload and metric, each step a bounded sample, on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_linattn_b200 import inputs, seqshard  # noqa: E402

METRIC = "linear-attention fwd tokens/sec and achieved HBM GB/s (fraction of B200 peak)"
MAIN = "longctx_1x32x131072x128_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ accounting
def forward_bytes(B, H, n, d, elem):
    """Algorithmic bytes of one forward: read q, k, v and write out once (4 n d per head)."""
    return 4 * B * H * n * d * elem


def decode_bytes(heads, d, elem=2):
    """Algorithmic bytes of one decode step: fp32 state (D*d + D) read and written once, plus
    q, k, v read and out written (4 token vectors)."""
    return heads * (2 * (d * d + d) * 4 + 4 * d * elem)


def code_hash(path: str) -> str:
    """sha256 of a C/CUDA source with its comments, trailing blanks and empty lines removed, so
    that only a change of the code itself changes it."""
    import hashlib
    import re
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/ncu_traffic.json (an ncu
    capture, scaled to the full launch), or None when there is none or the code of the
    kernel's source file has changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        table = json.load(f)
    rec = table.get(f"{kernel} | {workload}")
    if not rec:
        return None
    if code_hash(os.path.join(ROOT, rec["source"])) != rec["source_code_sha256"]:
        return None
    return float(rec["dram_bytes_per_launch"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained",
                                                     j["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxs.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sms:
            return None
        return {"sm_mhz": float(np.median(sms)), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_heads(B: int, H: int, rank: int):
    """(batch, head) pairs rank `rank` owns: batch elements [rank*B, (rank+1)*B) of the
    global batch (weak scaling: every rank runs one copy of the workload's shape)."""
    return [(rank * B + b, h) for b in range(B) for h in range(H)]


# ------------------------------------------------------------------ timing helpers
def time_steps(fn, steps, warmup, world, clocks=None):
    """W untimed steps, then K steps between barrier+synchronize; returns (ms per step
    (max over ranks), per-step device ms list).  Events are on the launching stream."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    if clocks:
        clocks.start()
        time.sleep(0.3)
    ev[0].record(stream)
    for i in range(steps):
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    if clocks:
        time.sleep(0.2)
    barrier(world)
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = ev[0].elapsed_time(ev[steps])
    return max_over_ranks(total / steps, world), per


def forward_launches(dtype: str, causal: bool, unit: int):
    """Names of the launches of one forward call, in order, and the algorithmic bytes of each
    (unit: the bytes of one [B,H,n,d] tensor)."""
    if dtype == "bf16":
        return (["tc_kernel<state> (segment aggregates, K1)",
                 "scan_states_kernel (prefix, K2)" if causal else "scan_states_kernel (totals, K2)",
                 "tc_kernel<causal out> (K3)" if causal else "tc_kernel<non-causal out> (K3)"],
                [2 * unit, 0, 4 * unit if causal else 2 * unit])
    return (["simt_chunk_state_kernel (K1)", "scan_states_kernel (K2)",
             "simt_chunk_out_kernel (K3)"], [2 * unit, 0, 4 * unit if causal else 2 * unit])


def backward_launches(causal: bool, unit: int):
    """Names of the launches of one bf16 backward call, in order, and the algorithmic bytes of
    each (unit: the bytes of one [B,H,n,d] tensor): K1 reads k, v (and stores psi(k) to the
    workspace); B1 reads q, psi(k), v, dout and writes dq (and a, b and psi(q) for the suffix
    walk); B3 reads psi(q), psi(k), v (and a, b) and writes dk, dv."""
    return (["bwd_aggregate_kernel (forward records, K1)",
             "scan_states_kernel (prefix, K2)" if causal else "scan_states_kernel (totals, K2)",
             "bwd_prefix_kernel (dq, B1)",
             "scan_states_kernel (suffix, K2)" if causal else "scan_states_kernel (totals, K2)",
             "bwd_suffix_kernel (dk, dv, B3)"],
            [2 * unit, 0, 5 * unit, 0, 5 * unit if causal else 4 * unit])


def time_launches(fn, steps, warmup, names):
    """Per-launch device times of a multi-kernel call: before each timed call the library is
    given events (linattn_profile_events) that it records after each of its launches on the
    call's stream; returns the mean ms of each launch."""
    import ctypes

    import torch

    import linear_attention_linattn_b200 as la
    lib = la.load_library()
    k = len(names)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(k)] for _ in range(steps)]
    arrs = []
    for i in range(steps):
        for e in evs[i]:
            e.record(stream)  # materialise the handles
    torch.cuda.synchronize()
    for i in range(steps):
        arr = (ctypes.c_void_p * k)(*[e.cuda_event for e in evs[i]])
        arrs.append(arr)
        starts[i].record(stream)
        lib.linattn_profile_events(arr, k)
        fn()
        lib.linattn_profile_events(None, 0)
    torch.cuda.synchronize()
    per = np.zeros(k)
    for i in range(steps):
        prev = starts[i]
        for j in range(k):
            per[j] += prev.elapsed_time(evs[i][j])
            prev = evs[i][j]
    return {nm: float(per[j] / steps) for j, nm in enumerate(names)}


# ------------------------------------------------------------------ oracle baseline
def oracle_sample(workload: str, target_s: float = 12.0, one_thread_s: float = 0.0):
    """Times the float64 oracle on a bounded sample of the workload (host cores, OpenMP over
    heads); with one_thread_s > 0 also on one thread, on a sample of about that many seconds."""
    import oracle
    w = inputs.WORKLOADS[workload]
    cores = os.cpu_count() or 1
    causal = True if True in w.causal else False
    oracle.set_threads(cores)
    # calibrate on one head of 4096 tokens
    q, k, v = inputs.forward_qkv(w.seed, 1, 1, min(w.n, 4096), w.d, w.scaled)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, causal)
    per_head_token = (time.perf_counter() - t0) / min(w.n, 4096)
    heads = min(w.B * w.H, cores)
    n_s = int(max(256, min(w.n, target_s / max(per_head_token, 1e-9))))
    q, k, v = inputs.forward_qkv(w.seed, 1, heads, n_s, w.d, w.scaled)
    if "bf16" in w.dtypes:
        q, k, v = (inputs.round_bf16(x) for x in (q, k, v))
    t0 = time.perf_counter()
    oracle.forward(q, k, v, causal)
    dt = time.perf_counter() - t0
    # tokens in the workload's unit: a token carries all H heads of its batch element
    tokens = heads * n_s / w.H
    rec = {"value": tokens / dt, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
           "threads": int(oracle.get_threads()),
           "sample": f"{heads} heads x {n_s} tokens of the {workload} workload "
                     f"({'causal' if causal else 'non-causal'}), float64, {dt:.1f} s"}
    if one_thread_s > 0:
        n1 = int(max(256, min(w.n, one_thread_s / max(per_head_token, 1e-9))))
        oracle.set_threads(1)
        t0 = time.perf_counter()
        oracle.forward(q[:, :1, :n1], k[:, :1, :n1], v[:, :1, :n1], causal)
        dt1 = time.perf_counter() - t0
        oracle.set_threads(cores)
        rec["one_thread"] = {"value": n1 / w.H / dt1, "unit": "tokens/s", "threads": 1,
                             "sample": f"1 head x {n1} tokens, float64, {dt1:.1f} s"}
    return rec


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = inputs.WORKLOADS[args.workload]
    vals = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(args.workload, target_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
        if i >= args.warmup:
            vals.append(r["value"])
    v = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": w.tokens / v * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": w.B, "H": w.H, "n": w.n, "d": w.d,
                       "causal": True in w.causal, "global_batch": w.B, "seq_len": w.n,
                       "parallelism": "host cores (OpenMP over heads)"},
            "cpu_baseline": dict(r, value=v),
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def main_forward(args, world, rank, local):
    import torch

    import linear_attention_linattn_b200 as la
    w = inputs.WORKLOADS[args.workload]
    if args.max_heads and args.max_heads < w.H:
        import dataclasses
        w = dataclasses.replace(w, H=args.max_heads)
    causal = True in w.causal
    if args.mode is not None:
        causal = args.mode == "causal"
    dtype = "bf16" if "bf16" in w.dtypes else "f32"
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    elem = 2 if dtype == "bf16" else 4
    seq = args.shard == "seq"
    if seq:
        # one sequence per head split over the ranks: rank r holds tokens
        # [r*n/N, (r+1)*n/N) of every head (strong scaling, one all-gather of block states)
        if w.n % (world * 64) != 0:
            raise SystemExit(f"--shard seq needs n divisible by 64 * ranks (n = {w.n})")
        blk = w.n // world
        q, k, v = inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled)
        q, k, v = (np.ascontiguousarray(x[:, :, rank * blk:(rank + 1) * blk]) for x in (q, k, v))
        shape = (w.B, w.H, blk, w.d)
    else:
        # this rank's batch element of the workload: b = rank (weak scaling over ranks)
        q, k, v = inputs.forward_qkv(w.seed, w.B * world, w.H, w.n, w.d, w.scaled,
                                     heads=rank_heads(w.B, w.H, rank))
        shape = (w.B, w.H, w.n, w.d)
    qh = torch.from_numpy(q.reshape(shape)).to(tdt).pin_memory()
    kh = torch.from_numpy(k.reshape(shape)).to(tdt).pin_memory()
    vh = torch.from_numpy(v.reshape(shape)).to(tdt).pin_memory()
    del q, k, v
    qd, kd, vd = qh.cuda(), kh.cuda(), vh.cuda()
    out = torch.empty_like(qd)
    backward = args.pass_ == "backward"
    if backward:
        if seq or dtype != "bf16":
            raise SystemExit("--pass backward times the bf16 backward on whole heads")
        gd = torch.from_numpy(inputs.forward_qkv(w.seed + 1, w.B, w.H, shape[2], w.d,
                                                 w.scaled)[0]).to(tdt).cuda()

    def step():
        if backward:
            la.backward(qd, kd, vd, gd, causal)
        elif seq:
            seqshard.forward_sequence_sharded(qd, kd, vd, causal)
        else:
            la.forward(qd, kd, vd, causal, out=out)

    clocks = ClockSampler(local)
    l0 = la.linattn_launch_count()
    ms, per = time_steps(step, args.steps, args.warmup, world, clocks=clocks)
    launches = (la.linattn_launch_count() - l0) // (args.steps + args.warmup) * args.steps
    clk = clocks.stop()
    assert la.device_error() == la.LINATTN_OK

    tokens_rank = w.B * shape[2]
    value = tokens_rank * world / (ms * 1e-3)
    pk = peaks()
    alg = forward_bytes(w.B, w.H, shape[2], w.d, elem)  # this rank's share
    unit = w.B * w.H * shape[2] * w.d * elem  # one [B,H,n,d] tensor (this rank's share)
    names, kbytes = (backward_launches(causal, unit) if backward
                     else forward_launches(dtype, causal, unit))
    if backward:
        alg = 7 * unit  # reads q, k, v, dout; writes dq, dk, dv
    if seq:
        # block state (aggregates, total), the start state, then the forward from it
        names = ["block state: aggregates (K1)", "block state: total (K2)",
                 "sum_states_kernel"] + names
        kbytes = [2 * unit, 0, 0] + kbytes
    launch_ms = time_launches(step, max(3, min(args.steps, 10)), 2, names)
    top = max(launch_ms, key=launch_ms.get)
    kernel_ms = launch_ms[top]
    kernel_alg = kbytes[names.index(top)]
    achieved = kernel_alg / (kernel_ms * 1e-3) / 1e9

    # end to end through the public API: pinned host -> device, forward, device -> host
    outh = torch.empty_like(qh).pin_memory()

    def e2e_step():
        if seq:
            a, b_, c = (x.to("cuda", non_blocking=True) for x in (qh, kh, vh))
            o = seqshard.forward_sequence_sharded(a, b_, c, causal)
            outh.copy_(o, non_blocking=True)
        else:
            # the C entry point on host buffers: head groups copied in, run and copied out
            # on the library's streams, the copies of one group overlapping the others' work
            la.forward_host(qh, kh, vh, causal, out=outh)

    e2e = None
    if not args.no_e2e and not backward:
        e2e_steps = max(1, min(args.steps, 3))
        e2e_ms, _ = time_steps(e2e_step, e2e_steps, 1, world)
        e2e = {"value": tokens_rank * world / (e2e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": 3 * qh.numel() * elem,
               "d2h_bytes_per_step": outh.numel() * elem,
               "path": ("to device, sequence-sharded forward, to host" if seq else
                        "linattn_forward_host: head groups copied in, run and copied out on "
                        "three streams")}
        # the host link's own rate on one input tensor, for context
        t0, t1, t2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        t0.record()
        tmp = qh.to("cuda", non_blocking=True)
        t1.record()
        outh.copy_(tmp, non_blocking=True)
        t2.record()
        torch.cuda.synchronize()
        e2e["h2d_gbs"] = qh.numel() * elem / (t0.elapsed_time(t1) * 1e-3) / 1e9
        e2e["d2h_gbs"] = qh.numel() * elem / (t1.elapsed_time(t2) * 1e-3) / 1e9
        del tmp

    line = {
        "metric": METRIC + (" (backward pass)" if backward else ""), "value": value,
        "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong" if seq else "weak", "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic (per head default_rng([seed, b, h]) draws q, k, v N(0,1), times 1/sqrt(d); bf16-rounded)",
        "config": {"workload": args.workload + (f" (first {w.H} heads)" if args.max_heads else "")
                   + (f" [{args.mode}]" if args.mode else "")
                   + (" [backward]" if backward else ""),
                   "B": w.B, "H": w.H, "n": w.n, "d": w.d,
                   "causal": causal, "global_batch": w.B if seq else w.B * world,
                   "seq_len": w.n,
                   "parallelism": (f"sequence split over {world} ranks (one all-gather of "
                                   "block states)") if seq else
                                  f"dp{world} (independent heads, no collective)",
                   "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                     "traffic": kernel_traffic(top, args.workload),
                     "peak_source": pk["source"] + " (burst copy bandwidth)",
                     "kernel": top, "kernel_ms": kernel_ms,
                     "algorithmic_bytes_per_launch": kernel_alg,
                     "launch_ms": launch_ms,
                     "whole_step": {"algorithmic_bytes": alg, "ms": ms,
                                    "gbs": alg / (ms * 1e-3) / 1e9,
                                    "frac": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    return line


def main_decode(args, world, rank, local):
    """Decode workload as the timed step: one linattn_decode_step over all states."""
    import torch

    import linear_attention_linattn_b200 as la
    from linear_attention_linattn_b200 import workloads
    w = inputs.WORKLOADS[args.workload]
    S, z, qs, ks, vs = workloads.decode_inputs(args.workload)
    T = qs.shape[0]
    out = torch.empty_like(qs[0])
    it = [0]

    def step():
        t = it[0] % T
        la.decode_step(S, z, qs[t], ks[t], vs[t], out=out)
        it[0] += 1

    clocks = ClockSampler(local)
    l0 = la.linattn_launch_count()
    ms, per = time_steps(step, args.steps, args.warmup, world, clocks=clocks)
    launches = (la.linattn_launch_count() - l0) // (args.steps + args.warmup) * args.steps
    clk = clocks.stop()
    assert la.device_error() == la.LINATTN_OK
    pk = peaks()
    alg = decode_bytes(w.B * w.H, w.d)
    kernel_ms = float(np.mean(per))
    achieved = alg / (kernel_ms * 1e-3) / 1e9
    return {
        "metric": "linear-attention decode-step tokens/sec and achieved HBM GB/s",
        "value": w.B * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(d), prefill state from linattn_forward_state)",
        "config": {"workload": args.workload, "Bseq": w.B, "H": w.H, "d": w.d,
                   "parallelism": f"dp{world} (independent states, no collective)",
                   "l2": "state (541 MB) larger than L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": None,
                     "peak_source": pk["source"], "algorithmic_bytes": alg,
                     "kernel": "decode_step_kernel<128>", "kernel_ms": kernel_ms},
        "gpu_launches": int(launches), "clocks": clk,
    }


def extras(args):
    """Other workloads at N=1: decode, batched forward, small latency cases."""
    import torch

    import linear_attention_linattn_b200 as la
    from linear_attention_linattn_b200 import workloads
    pk = peaks()
    res = {}
    # decode: 512 steps of 256 x 32 states, d = 128
    S, z, qs, ks, vs = workloads.decode_inputs("decode_256x32x128")
    T = qs.shape[0]
    out = torch.empty_like(qs[0])
    for t in range(3):
        la.decode_step(S, z, qs[t], ks[t], vs[t], out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(T):
        la.decode_step(S, z, qs[t], ks[t], vs[t], out=out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / T
    b = decode_bytes(256 * 32, 128)
    res["decode_256x32x128"] = {"ms_per_step": ms, "tokens_per_s": 256 / (ms * 1e-3),
                                "head_states_per_s": 256 * 32 / (ms * 1e-3),
                                "gbs": b / (ms * 1e-3) / 1e9,
                                "frac_hbm": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                "algorithmic_bytes_per_step": b, "steps": T}
    del S, z, qs, ks, vs
    torch.cuda.empty_cache()
    # batched forward, both modes
    name = "batched_8x16x8192x64_bf16"
    w = inputs.WORKLOADS[name]
    q, k, v = workloads.forward_inputs(name, "bf16")
    o = torch.empty_like(q)
    for causal in (False, True):
        ms, _ = time_steps(lambda: la.forward(q, k, v, causal, out=o), 20, 3, 1)
        alg = forward_bytes(w.B, w.H, w.n, w.d, 2)
        res[f"{name}_{'causal' if causal else 'noncausal'}"] = {
            "ms": ms, "tokens_per_s": w.B * w.n / (ms * 1e-3), "gbs": alg / (ms * 1e-3) / 1e9,
            "frac_hbm": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    # backward pass on the same shape: reads q, k, v, dout and writes dq, dk, dv
    dout = torch.randn_like(o)
    for causal in (True, False):
        fn = lambda: la.backward(q, k, v, dout, causal)  # noqa: E731
        ms, _ = time_steps(fn, 10, 3, 1)
        alg = 7 * w.B * w.H * w.n * w.d * 2
        names = backward_launches(causal, 0)[0]
        res[f"backward_{name}_{'causal' if causal else 'noncausal'}"] = {
            "ms": ms, "tokens_per_s": w.B * w.n / (ms * 1e-3), "gbs": alg / (ms * 1e-3) / 1e9,
            "frac_hbm": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], "algorithmic_bytes": alg,
            "launch_ms": time_launches(fn, 5, 2, names),
            "path": "tensor cores (tcgen05, TMEM, TMA), 5 launches"}
    # FAVOR+ (Performer's positive random features) on the same shape, causal: the features of
    # q and k (m of them), then the pass on them; m = d and m = 2 d
    for m in (w.d, 2 * w.d):
        W = torch.randn(m, w.d, device="cuda")
        ms, _ = time_steps(lambda: la.forward_favor(q, k, v, W, True), 10, 3, 1)
        # q, k, v read and out written, plus the features written and read back
        alg = 4 * w.B * w.H * w.n * w.d * 2 + 2 * 2 * w.B * w.H * w.n * m * 2
        res[f"favor_m{m}_{name}_causal"] = {
            "ms": ms, "tokens_per_s": w.B * w.n / (ms * 1e-3), "gbs": alg / (ms * 1e-3) / 1e9,
            "frac_hbm": alg / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], "algorithmic_bytes": alg,
            "m": m, "path": "features and pass on the tensor cores (identity feature map)"}
    del q, k, v, o, dout
    # latency cases
    for name, dtypes in (("noncausal_1x1x512x64_f32", ("f32",)),
                         ("causal_1x1x4096x64", ("f32", "bf16"))):
        w = inputs.WORKLOADS[name]
        for dt in dtypes:
            q, k, v = workloads.forward_inputs(name, dt)
            o = torch.empty_like(q)
            causal = True in w.causal
            fn = lambda: la.forward(q, k, v, causal, out=o)  # noqa: E731
            ms, _ = time_steps(fn, 50, 5, 1)
            # back-to-back calls of a small problem measure the host's call rate; the device
            # time of one call is the sum of its launches
            dev = time_launches(fn, 20, 5, forward_launches(dt, causal, 0)[0])
            dev_us = sum(dev.values()) * 1e3
            res[f"{name}_{dt}"] = {"us": ms * 1e3, "device_us": dev_us,
                                   "tokens_per_s": w.B * w.n / (ms * 1e-3)}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=MAIN, choices=list(inputs.WORKLOADS))
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shard", choices=["heads", "seq"], default="heads",
                    help="heads: every rank runs its own batch element (weak scaling); seq: "
                         "one sequence per head split over the ranks (strong scaling)")
    ap.add_argument("--mode", choices=["causal", "noncausal"], default=None,
                    help="for a workload that has both modes (default: causal)")
    ap.add_argument("--max-heads", type=int, default=0,
                    help="profiling aid: run only the first N heads of the workload")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward"], default="forward",
                    help="backward: time the bf16 backward pass (dq, dk, dv) on the workload")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import torch
    torch.cuda.set_device(local)
    if inputs.WORKLOADS[args.workload].kind == "decode":
        line = main_decode(args, world, rank, local)
        args.no_extras = args.no_cpu_baseline = True
    else:
        line = main_forward(args, world, rank, local)
    if world == 1 and rank == 0:
        if not args.no_extras:
            line["extras"] = extras(args)
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(args.workload, one_thread_s=6.0)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
