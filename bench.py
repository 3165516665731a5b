#!/usr/bin/env python
"""Benchmark of the gated-delta-rule prefill (and decode step) on B200.

``python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]``

One step = one ``gdn_chunk_prefill`` call over the 4096-token workload (B=1, T=4096, H=32,
dk=dv=128, bf16 q/k/v, fp32 g/beta, C=32, zero initial state, final state written).  Under torchrun
every rank runs its own independent prefill (weak scaling, no data-path collective).  The line also
carries the recurrent decode step (B=64, H=32, d=128, 1000 chained steps) as ``decode``.
``--shard heads`` instead splits one layer's 32 heads over the ranks (strong scaling; ``--gather``
adds an all-gather of the outputs to every step).

Timing: CUDA events on the launching stream, W warm-up steps, barrier + synchronize around the K
timed steps, max over ranks.  L2: every step reads one of three rotating input sets (about 300 MB
of q/k/v in total, above the 126 MB L2), so no step finds its inputs in L2.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule prefill tokens/s per layer (H=32,d=128); % of roofline"
UNIT = "tokens/s"
C = 32
H, D, T_PREFILL = 32, 128, 4096
WORKLOAD = "prefill_4k"
WORKLOAD_DESC = ("B=1, T=4096, H=32, dk=dv=128, bf16 q/k/v (q,k L2-normalised), fp32 g=-softplus(N(0,1))*0.1 "
                 "and beta=sigmoid(N(0,1)), zero initial state, C=32, fp32 final state")

# Algorithmic work per (token, head), chunk size C, head size d (dk = dv = d):
#   whole method      6 d^2 + 10 C d       (K K^T, Q K^T, W/U', intra-chunk P U, S-products, carry)
#   chunk-parallel    8 C d                (K K^T 2Cd, Q K^T 2Cd, W and U' 4Cd)
#   state-dependent   6 d^2 + 2 C d        (W S^T and Q S^T 4 d^2, P U 2 C d, carry 2 d^2)
def flops_whole(d=D):
    return 6 * d * d + 10 * C * d


def flops_scan(d=D):
    return 6 * d * d + 2 * C * d


def flops_prep(d=D):
    return 8 * C * d


# Per-kernel roofline model.  "alu": fp32 CUDA-core FMAs, 1x the algorithmic flops, against the fp32
# FMA peak derived from unit counts (148 SMs x 128 lanes x 2 flop x max SM clock).  "tensor": TF32
# tensor cores with the 3xTF32 split, 3x the algorithmic flops, against the TF32 peak (measured
# bf16 GEMM peak x nominal TF32/bf16 ratio 1.1/2.25).  "hbm": algorithmic bytes against the measured
# copy bandwidth.
KERNELS = {
    "gdn_scan_tc_kernel": dict(bound="tensor", flops_per_token_head=flops_scan(), split=3),
    "gdn_scan_pair_kernel": dict(bound="tensor", flops_per_token_head=flops_scan(), split=3),
    "gdn_prep_kernel": dict(bound="tensor", flops_per_token_head=flops_prep(), split=3),
    "gdn_prep_pair_kernel": dict(bound="tensor", flops_per_token_head=flops_prep(), split=3),
    "gdn_plan_kernel": dict(bound="latency"),
    "gdn_decode_step_kernel": dict(bound="hbm"),
    "gdn_decode_verify_kernel": dict(bound="hbm"),
    "gdn_l2norm_kernel": dict(bound="hbm"),
}
# dram__bytes_read.sum + dram__bytes_write.sum per launch from the last ncu capture of that kernel
# on the bench workload (None until captured, and reset whenever the kernel changes).  The decode
# and verify figures undercount writes: ncu starts each replay from a clean L2, and 56-58 MB of the
# written states are still resident (dirty) in L2 when the launch ends.
TRAFFIC = {
    "gdn_scan_pair_kernel": 202.50e6 + 24.83e6,
    "gdn_prep_pair_kernel": 68.21e6 + 45.12e6,
    "gdn_l2norm_kernel": 67.12e6 + 21.02e6,
    "gdn_decode_step_kernel": 135.83e6 + 77.84e6,
    "gdn_decode_verify_kernel": 140.59e6 + 479.75e6,
    "gdn_decode_verify_kernel (tree, verify_tree_b64_k8)": 147.02e6 + 1019.77e6,
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        j = json.load(open(p))
        return dict(hbm_gbs=float(j["hbm_gbs"]), bf16_tflops=float(j["bf16_tflops"]),
                    bf16_tflops_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    sm_max_mhz=float(j.get("sm_max_mhz", 1965.0)), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
                    source="fallback")


# Nominal dense peaks of one B200, stated for the "% of roofline" the metric asks for beside the
# measured-peak figures: TF32 tensor 1.125 PFLOP/s (half the 2:4-sparse datasheet figure), HBM3e 8 TB/s.
NOMINAL_TF32_TFLOPS = 1125.0
NOMINAL_HBM_GBS = 8000.0


def prefill_api_bytes(T, Hh, d, N, state_in, es=2):
    """Algorithmic bytes of one prefill call: the API's inputs and outputs only (q, k, v, out in the
    storage type of es bytes, g and beta fp32, state_in if given and state_out fp32)."""
    return 4 * T * Hh * d * es + 2 * T * Hh * 4 + (2 if state_in else 1) * N * Hh * d * d * 4


def method_roofline_of(T, Hh, d, N, state_in, call_ms, peaks, es=2):
    """Whole-call roofline of the method, max(3 F T H / TF32 peak, API bytes / HBM peak), against the
    measured call time; at the measured-derived peaks (the headline) and at the nominal ones."""
    flops3 = 3 * flops_whole(d) * T * Hh
    nbytes = prefill_api_bytes(T, Hh, d, N, state_in, es)

    def at(tf32, hbm):
        t_flop, t_byte = flops3 / (tf32 * 1e12), nbytes / (hbm * 1e9)
        r = max(t_flop, t_byte)
        return dict(bound="tensor(TF32 x3)" if t_flop >= t_byte else "hbm", roofline_us=r * 1e6,
                    frac=r / (call_ms / 1e3), tf32_peak_tflops=tf32, hbm_peak_gbs=hbm)
    tf32, _, _ = peak_for("tensor", peaks)
    return dict(achieved_us=call_ms * 1e3, flops_x3=flops3, api_bytes=nbytes,
                measured_peaks=at(tf32, peaks["hbm_gbs"]), nominal_peaks=at(NOMINAL_TF32_TFLOPS, NOMINAL_HBM_GBS),
                headline="measured_peaks")


def peak_for(bound, peaks):
    if bound == "tensor":
        return peaks["bf16_tflops"] * (1.1 / 2.25), "TFLOP/s", "%s bf16 GEMM x 1.1/2.25 (TF32)" % peaks["source"]
    if bound == "alu":
        return 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12, "TFLOP/s", "fp32 FMA: 148 SM x 128 x 2 x max clock"
    if bound == "hbm":
        return peaks["hbm_gbs"], "GB/s", "%s copy bandwidth" % peaks["source"]
    return None, None, None


# ---------------------------------------------------------------------------------------------------
# multi-rank timing: every rank times its own independent work; the job is as slow as its slowest rank
# ---------------------------------------------------------------------------------------------------
def max_over_ranks(x, world, device=None):
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_passes(fn, n, world, dev, stream):
    """Times n calls of fn(i) on `stream` with CUDA events (max over ranks), then runs them again with
    an event pair around every library launch; returns (ms of the first pass, per-kernel profile of
    the second).  The first pass has no events between launches, which would serialise them."""
    import torch
    import torch.distributed as dist
    from linear_attention_10_b200 import gdn
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    gdn.gdn_profile_start()
    for i in range(n):
        fn(i)
    torch.cuda.synchronize()
    return ms, gdn.gdn_profile_stop()


def job_throughput(units_per_rank_step, steps, world, max_ms):
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank_step * world * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="gdn_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            if self.bus_id and not self.bus_id.endswith(f[0].lower()[-len(self.bus_id):]) and \
                    f[0].lower()[-12:] != self.bus_id[-12:]:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), util=float(f[4]),
                                 reasons=[n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown",
                                                             "sw_thermal_slowdown", "sw_power_cap"), f[5:9])
                                          if v.lower() == "active"]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        busy = [r for r in rows if r["util"] > 0] or rows
        reasons = sorted({x for r in busy for x in r["reasons"]})
        return dict(sm_mhz=statistics.median(r["sm"] for r in busy), sm_max_mhz=max(r["smax"] for r in rows),
                    reasons=reasons, samples=len(busy))


# ---------------------------------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------------
def oracle_layer_rate(inp, budget_s=15.0, max_heads=None, tokens=None):
    """Time the fp64 single-thread oracle over whole heads of the workload until ``budget_s`` is
    spent; returns (tokens/s for the full layer of H heads, seconds, heads, tokens)."""
    import numpy as np
    import oracle
    q, k, v, g, b = (inp[n].float().cpu().numpy().astype(np.float64) for n in ("q", "k", "v", "g", "beta"))
    Tt = q.shape[0] if tokens is None else min(tokens, q.shape[0])
    Hh = q.shape[1]
    heads, spent = 0, 0.0
    for h in range(Hh if max_heads is None else min(max_heads, Hh)):
        sl = slice(h, h + 1)
        t0 = time.perf_counter()
        oracle.recurrence(q[:Tt, sl], k[:Tt, sl], v[:Tt, sl], g[:Tt, sl], b[:Tt, sl])
        spent += time.perf_counter() - t0
        heads += 1
        if spent >= budget_s:
            break
    per_layer_s = spent / heads * Hh
    return Tt / per_layer_s, spent, heads, Tt


# The same fp64 oracle on every host core: one process per head of the layer (a spawn pool, so no
# CUDA context is inherited).  Each worker builds the seeded workload once, outside the timed map.
_ORACLE_INPUTS = None


def _oracle_worker_init(workload):
    global _ORACLE_INPUTS
    import numpy as np
    from linear_attention_10_b200.workloads import workload_inputs
    inp = workload_inputs(workload, device="cpu")
    _ORACLE_INPUTS = tuple(inp[n].float().numpy().astype(np.float64) for n in ("q", "k", "v", "g", "beta"))


def _oracle_worker_head(h):
    import oracle
    q, k, v, g, b = _ORACLE_INPUTS
    sl = slice(h, h + 1)
    oracle.recurrence(q[:, sl], k[:, sl], v[:, sl], g[:, sl], b[:, sl])
    return h


def oracle_layer_rate_all_cores(H, tokens, repeats=3):
    """Tokens/s of the whole layer with the single-thread oracle run on all H heads at once, one head
    per process on min(host cores, H) processes; median of `repeats` passes.  Returns (tokens/s,
    processes, median seconds)."""
    import multiprocessing as mp
    procs = max(1, min(os.cpu_count() or 1, H))
    ctx = mp.get_context("spawn")
    walls = []
    with ctx.Pool(procs, initializer=_oracle_worker_init, initargs=(WORKLOAD,)) as pool:
        pool.map(_oracle_worker_head, range(procs), chunksize=1)      # every worker built its inputs
        for _ in range(repeats):
            t0 = time.perf_counter()
            pool.map(_oracle_worker_head, range(H), chunksize=1)
            walls.append(time.perf_counter() - t0)
    wall = statistics.median(walls)
    return tokens / wall, procs, wall


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle, timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    import torch
    from linear_attention_10_b200.workloads import workload_inputs
    inp = workload_inputs(WORKLOAD, device="cpu")
    q, k, v, g, b = (inp[n].float().numpy().astype(np.float64) for n in ("q", "k", "v", "g", "beta"))
    # calibrate the cost of one token of one head, then size each step to keep the run short
    t0 = time.perf_counter()
    oracle.recurrence(q[:256, :1], k[:256, :1], v[:256, :1], g[:256, :1], b[:256, :1])
    per_tok = (time.perf_counter() - t0) / 256
    budget = 150.0
    L = int(max(64, min(T_PREFILL, budget / max(args.steps + args.warmup, 1) / per_tok)))
    times = []
    for i in range(args.warmup + args.steps):
        h = i % H
        sl = slice(h, h + 1)
        t0 = time.perf_counter()
        oracle.recurrence(q[:L, sl], k[:L, sl], v[:L, sl], g[:L, sl], b[:L, sl])
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    per_step = sum(times) / len(times)           # seconds for L tokens of one head
    value = L / (per_step * H)                   # tokens/s of a whole layer (H heads)
    sample = "fp64 oracle recurrence, 1 head x %d tokens of the %s workload per step (layer rate = tokens / (step time x %d heads))" % (L, WORKLOAD, H)
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=per_step * 1e3, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f64", data="synthetic", impl="reference",
                config=dict(workload="%s: %s" % (WORKLOAD, WORKLOAD_DESC), global_batch=1, seq_len=T_PREFILL,
                            parallelism="host CPU, 1 thread"),
                cpu_baseline=dict(value=value, unit=UNIT, cores=1, kind="oracle", sample=sample),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)



# ---------------------------------------------------------------------------------------------------
# the other prefill workloads of the method (varlen resume, 128K context, tiny fp32)
# ---------------------------------------------------------------------------------------------------
WORKLOAD_DESCS = {
    "varlen_resume": "4 packed sequences of 8192/3000/517/13000 tokens (24,709), H=32, dk=dv=128, bf16 q/k/v, "
                     "initial states ~N(0,0.05^2) per sequence, C=32, final states written",
    "long_128k": "B=1, T=131072, H=32, dk=dv=128, bf16 q/k/v, zero initial state, C=32 (4096 chunks, scanned in "
                 "2048 sequential steps of two)",
    "tiny_fp32": "B=1, T=128 (4 chunks), H=2, dk=dv=64, fp32 q/k/v, g~U[-0.5,0), zero initial state",
}
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant kernel for these workloads
# (None until captured, reset whenever the kernel changes).  long_128k: captured on its first 32,768
# tokens (512 pairs of chunks; the full launch holds too much memory for a multi-pass capture) and
# scaled by the pair count 2,048 / 512, the traffic per pair-row being the same at every length.
TRAFFIC_BY_WORKLOAD = {
    ("long_128k", "gdn_scan_pair_kernel"): (1619.12e6 + 258.24e6) * 2048 / 512,
}


def l2_flush_buffer(dev):
    import torch
    return torch.empty(256 << 20, dtype=torch.uint8, device=dev)


def bench_prefill_workload(name, reps, world, dev, stream, peaks, rank, flush=None):
    """Times `reps` prefill calls of one named workload and returns its bench entry.  Workloads whose
    q/k/v exceed L2 run back to back between one event pair (no call finds its inputs in L2); smaller
    ones get an event pair per call with a 256 MB write between calls (outside the pairs) flushing L2,
    and report the median call.  A second pass with an event pair around every launch gives the
    per-kernel durations and the roofline of the dominant kernel."""
    import torch
    from linear_attention_10_b200 import gdn
    from linear_attention_10_b200.workloads import WORKLOADS, workload_inputs
    w = WORKLOADS[name]
    inp = workload_inputs(name, device=dev, seed=w.seed + 1000 * rank)
    T, N, Hh, d = w.total_tokens, len(w.lengths), w.H, w.dk
    es = 2 if w.dtype == "bf16" else 4
    out = torch.empty((T, Hh, w.dv), dtype=inp["q"].dtype, device=dev)
    st = torch.empty((N, Hh, w.dv, d), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.workspace_bytes(T, N, Hh, d, w.dv), dtype=torch.uint8, device=dev)

    def call(_i=0):
        gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                              state_in=inp["state_in"], out=out, state_out=st, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    big = 3 * T * Hh * d * es > 2 * 126e6
    if big:
        ms_all, prof = timed_passes(call, reps, world, dev, stream)
        call_ms = ms_all / reps
        timing = "%d calls back to back between one event pair (q/k/v %.0f MB > L2)" % (reps, 3 * T * Hh * d * es / 1e6)
    else:
        if flush is None:
            flush = l2_flush_buffer(dev)
        pairs = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            pairs.append((a, b))
        torch.cuda.synchronize()
        call_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in pairs), world, dev)
        gdn.gdn_profile_start()
        for _ in range(reps):
            flush.fill_(1)
            call()
        torch.cuda.synchronize()
        prof = gdn.gdn_profile_stop()
        timing = "median of %d calls, each between its own event pair, L2 flushed (256 MB write) between calls" % reps
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error in workload %s" % name)
    dom = max((n for n in prof if "flops_per_token_head" in KERNELS.get(n, {})), key=lambda n: prof[n][0])
    kms, kl = prof[dom]
    spec = KERNELS[dom]
    per_unit = flops_scan(d) if "scan" in dom else flops_prep(d)
    flops = per_unit * spec["split"] * T * Hh
    ach = flops / (kms / kl / 1e3) / 1e12
    pk, pu, pdesc = peak_for(spec["bound"], peaks)
    total = sum(v[0] for v in prof.values())
    roof = dict(kernel=dom, bound=spec["bound"], achieved=ach, peak=pk, unit=pu, frac=ach / pk, peak_source=pdesc,
                flops_per_launch=flops, avg_launch_us=kms / kl * 1e3, traffic=TRAFFIC_BY_WORKLOAD.get((name, dom)),
                kernels={n: dict(avg_us=v[0] / v[1] * 1e3, launches=v[1], share=v[0] / total) for n, v in prof.items()})
    entry = dict(workload="%s: %s" % (name, WORKLOAD_DESCS[name]), value=job_throughput(T, 1, world, call_ms),
                 unit=UNIT, us_per_call=call_ms * 1e3, reps=reps, timing=timing, roofline=roof,
                 method_roofline=method_roofline_of(T, Hh, d, N, w.state_std is not None, call_ms, peaks, es))
    del inp, out, st, ws
    return entry


def run_case(args, rank, world, local_rank):
    """--case NAME: only the prefill of one named workload (optionally its first --case-tokens tokens),
    --warmup + --steps calls, for profiler captures of one kernel on a bounded case."""
    import torch
    from linear_attention_10_b200 import gdn
    from linear_attention_10_b200.workloads import WORKLOADS, make_prefill_inputs
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.case]
    lengths = list(w.lengths)
    if args.case_tokens:
        keep, left = [], args.case_tokens
        for L in lengths:
            if left <= 0:
                break
            keep.append(min(L, left))
            left -= keep[-1]
        lengths = keep
    inp = make_prefill_inputs(lengths, w.H, w.dk, w.dv, w.dtype, w.gate, w.seed, w.state_std, dev)
    T, N = sum(lengths), len(lengths)
    ws = torch.empty(gdn.workspace_bytes(T, N, w.H, w.dk, w.dv), dtype=torch.uint8, device=dev)
    call = lambda: gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                         cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"], workspace=ws)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    if rank == 0:
        print(json.dumps(dict(case=args.case, lengths=lengths, H=w.H, d=w.dk, ms_per_call=ms,
                              tokens_per_s=T / (ms / 1e3))), flush=True)


# ---------------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from linear_attention_10_b200 import gdn
    from linear_attention_10_b200.workloads import (WORKLOADS, best_first_parents, make_decode_inputs,
                                                    make_verify_inputs, workload_inputs)

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    gdn.lib()
    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    # three rotating input sets (q/k/v of all three ~ 300 MB > L2)
    sets = [workload_inputs(WORKLOAD, device=dev, seed=1000 * rank + i) for i in range(3)]
    N = 1
    ws = torch.empty(gdn.workspace_bytes(T_PREFILL, N, H, D, D), dtype=torch.uint8, device=dev)
    out = torch.empty((T_PREFILL, H, D), dtype=torch.bfloat16, device=dev)
    st_out = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)

    def step(i):
        s = sets[i % 3]
        gdn.gdn_chunk_prefill(s["q"], s["k"], s["v"], s["g"], s["beta"], cu_seqlens=s["cu_seqlens"],
                              out=out, state_out=st_out, workspace=ws)

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error during warm-up")

    bus = None
    try:
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
    except Exception:
        try:
            p = torch.cuda.get_device_properties(dev)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        except Exception:
            bus = None
    clocks = ClockSampler(bus if isinstance(bus, str) else None)
    clocks.start()
    time.sleep(0.3)

    # ---- timed region: K prefill steps, as a caller runs them.  No event is recorded between the
    # three launches of a step here: an event there serialises them (the prep and scan kernels are
    # launched as programmatic dependents of their predecessors) and costs ~20 us per step ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error in the timed region")
    # ---- per-kernel durations: the same K steps again, with an event pair around every launch on the
    # launching stream (the roofline of the dominant kernel and the launch count come from here) ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    gdn.gdn_profile_start()
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    prof = gdn.gdn_profile_stop()
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error in the profiled pass")
    # ---- the per-call distribution: the same K steps with an event pair around each whole call (an
    # event between calls separates nothing: each call's first kernel is an ordinary launch) ----
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(stream)
        step(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    per_call_ms = sorted(max_over_ranks(a.elapsed_time(b_), world, dev) for a, b_ in evs)
    ms_per_step = ms / args.steps
    value = job_throughput(T_PREFILL, args.steps, world, ms)

    # ---- e2e: host (pinned) inputs -> device -> prefill -> host outputs, every step ----
    # Pipelined as a caller would run it: step i+1's inputs are copied in (copy-in stream) while step
    # i computes (compute stream) and step i-1's results are copied out (copy-out stream); device and
    # pinned host buffers are double-buffered and every hand-over is an event.
    host = {n: sets[0][n].cpu().pin_memory() for n in ("q", "k", "v", "g", "beta", "cu_seqlens")}
    dbuf = [{n: torch.empty_like(sets[0][n]) for n in host} for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    d_st = [torch.empty_like(st_out) for _ in range(2)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h_st = [torch.empty(st_out.shape, dtype=st_out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_out[0].numel() * h_out[0].element_size() + h_st[0].numel() * h_st[0].element_size()
    e2e_steps = max(3, min(args.steps, 50))      # enough steps to amortise filling and draining the pipeline
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(nsteps, start_ev):
        ev_in, ev_comp, ev_out = {}, {}, {}
        for i in range(nsteps):
            b = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(start_ev)
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])       # the compute that read dbuf[b] is done
                for n in host:
                    dbuf[b][n].copy_(host[n], non_blocking=True)
                ev_in[i] = torch.cuda.Event()
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[i])
                if i >= 2:
                    s_comp.wait_event(ev_out[i - 2])      # the copy-out that read d_out[b] is done
                x = dbuf[b]
                gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                                      out=d_out[b], state_out=d_st[b], workspace=ws, stream=s_comp)
                ev_comp[i] = torch.cuda.Event()
                ev_comp[i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                h_out[b].copy_(d_out[b], non_blocking=True)
                h_st[b].copy_(d_st[b], non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(s_out)
        return ev_out[nsteps - 1], ev_comp[nsteps - 1], ev_in[nsteps - 1]

    warm = torch.cuda.Event()
    warm.record(stream)
    e2e_run(2, warm)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    last = e2e_run(e2e_steps, e0)
    for ev in last:
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(T_PREFILL, e2e_steps, world, e2e_ms)
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error in the e2e region")
    # the host->device link alone: the same pinned input set copied 10 times on the copy-in stream
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s_in):
        c0.record(s_in)
        for _ in range(10):
            for n in host:
                dbuf[0][n].copy_(host[n], non_blocking=True)
        c1.record(s_in)
    torch.cuda.synchronize()
    h2d_ms = c0.elapsed_time(c1) / 10
    del dbuf, d_out, d_st

    # ---- decode step: B=64, 1000 chained steps ----
    decode = None
    if not args.no_decode:
        w = WORKLOADS["decode_b64"]
        dd = make_decode_inputs(w.decode_batch, w.H, w.dk, w.dv, w.decode_steps, dtype=w.dtype, gate=w.gate,
                                seed=w.seed + rank, state_std=w.state_std, device=dev)
        S = dd["state"].clone()
        dout = torch.empty((w.decode_batch, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        for s in range(3):
            gdn.gdn_decode_step(dd["q"][s], dd["k"][s], dd["v"][s], dd["g"][s], dd["beta"][s], S, out=dout)
        S.copy_(dd["state"])
        dms, dprof = timed_passes(lambda s: gdn.gdn_decode_step(dd["q"][s], dd["k"][s], dd["v"][s], dd["g"][s],
                                                                dd["beta"][s], S, out=dout),
                                  w.decode_steps, world, dev, stream)
        name = "gdn_decode_step_kernel"
        kms, kl = dprof.get(name, (dms, w.decode_steps))
        B_, H_, d_ = w.decode_batch, w.H, w.dk
        bytes_per_launch = 2 * B_ * H_ * d_ * d_ * 4 + B_ * H_ * (3 * d_) * 2 + B_ * H_ * 2 * 4 + B_ * H_ * d_ * 2
        ach = bytes_per_launch / (kms / kl / 1e3) / 1e9
        pk, pu, pdesc = peak_for("hbm", peaks)
        decode = dict(workload="decode_b64: B=64, H=32, dk=dv=128, bf16 q/k/v, fp32 state [64,32,128,128] in place, "
                               "%d chained steps, fresh inputs per step" % w.decode_steps,
                      value=job_throughput(B_, w.decode_steps, world, dms), unit="tokens/s",
                      us_per_step=dms / w.decode_steps * 1e3,
                      roofline=dict(kernel=name, bound="hbm", achieved=ach, peak=pk, unit=pu, frac=ach / pk,
                                    peak_source=pdesc, bytes_per_launch=bytes_per_launch,
                                    traffic=TRAFFIC.get(name)))
        del dd, S

    # ---- prefill_4k with state snapshots at 7 cut points (turn boundaries, not chunk-aligned) ----
    cuts_line = None
    if not args.no_cuts:
        cut_pos = torch.tensor([517, 1000, 1531, 2048, 2600, 3071, 3500], dtype=torch.int32, device=dev)
        ci = sets[0]
        snaps = torch.empty((cut_pos.numel(), H, D, D), dtype=torch.float32, device=dev)
        ws_c = torch.empty(gdn.workspace_bytes(T_PREFILL, N + cut_pos.numel(), H, D, D), dtype=torch.uint8,
                           device=dev)
        run_c = lambda: gdn.gdn_chunk_prefill_cuts(ci["q"], ci["k"], ci["v"], ci["g"], ci["beta"], cut_pos,
                                                   cu_seqlens=ci["cu_seqlens"], state_in=ci["state_in"],
                                                   snapshots=snaps, workspace=ws_c)
        for _ in range(3):
            run_c()
        torch.cuda.synchronize()
        reps = 20
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(reps):
            run_c()
        c1.record(stream)
        torch.cuda.synchronize()
        cms = max_over_ranks(c0.elapsed_time(c1), world, dev)
        cuts_line = dict(workload="prefill_4k with 7 cut points (517, 1000, 1531, 2048, 2600, 3071, 3500): "
                                  "chunks restart at each cut, 7 state snapshots written",
                         value=job_throughput(T_PREFILL, reps, world, cms), unit="tokens/s",
                         us_per_call=cms / reps * 1e3, inputs="first of the rotating input sets (L2-warm)")
        del snaps, ws_c

    # ---- prefill_4k with raw q/k: the library L2-normalises them (pre-pass into the workspace) ----
    norm_line = None
    if not args.no_norm:
        ni = sets[0]
        gen = torch.Generator(device=dev)
        gen.manual_seed(77)
        sc = torch.exp(torch.empty((T_PREFILL, H, 1), device=dev).uniform_(-3.0, 3.0, generator=gen))
        qr, kr = (ni["q"].float() * sc).to(ni["q"].dtype), (ni["k"].float() * sc.flip(0)).to(ni["k"].dtype)
        ws_n = torch.empty(gdn.workspace_bytes(T_PREFILL, N, H, D, D, gdn.GDN_BF16 | gdn.GDN_QK_L2NORM),
                           dtype=torch.uint8, device=dev)
        run_n = lambda: gdn.gdn_chunk_prefill(qr, kr, ni["v"], ni["g"], ni["beta"], cu_seqlens=ni["cu_seqlens"],
                                              workspace=ws_n, normalize_qk=True)
        for _ in range(3):
            run_n()
        torch.cuda.synchronize()
        reps = 20
        nms, nprof = timed_passes(lambda i: run_n(), reps, world, dev, stream)
        name = "gdn_l2norm_kernel"
        kms, kl = nprof.get(name, (nms, reps))
        bytes_per_launch = 4 * T_PREFILL * H * D * 2          # q, k read and their normalised copies written
        ach = bytes_per_launch / (kms / kl / 1e3) / 1e9
        pk, pu, pdesc = peak_for("hbm", peaks)
        norm_line = dict(workload="prefill_4k with raw q/k (vectors scaled by e^U[-3,3]); the library L2-normalises "
                                  "them in a pre-pass",
                         value=job_throughput(T_PREFILL, reps, world, nms), unit="tokens/s",
                         us_per_call=nms / reps * 1e3, inputs="first of the rotating input sets (L2-warm)",
                         roofline=dict(kernel=name, bound="hbm", achieved=ach, peak=pk, unit=pu, frac=ach / pk,
                                       peak_source=pdesc, bytes_per_launch=bytes_per_launch,
                                       avg_launch_us=kms / kl * 1e3, traffic=TRAFFIC.get(name)))
        del qr, kr, ws_n

    # ---- multi-token verify: B=64 sequences x 4 drafted tokens, every per-token state written ----
    verify = None
    if not args.no_verify:
        w = WORKLOADS["verify_b64_k4"]
        B_, Tk, H_, d_ = w.decode_batch, w.decode_steps, w.H, w.dk
        vd = make_verify_inputs(B_, H_, d_, d_, Tk, dtype=w.dtype, gate=w.gate, seed=w.seed + rank,
                                state_std=w.state_std, device=dev)
        vst = torch.empty((B_, Tk, H_, d_, d_), dtype=torch.float32, device=dev)
        vout = torch.empty((B_, Tk, H_, d_), dtype=torch.bfloat16, device=dev)
        run_v = lambda: gdn.gdn_decode_verify(vd["q"], vd["k"], vd["v"], vd["g"], vd["beta"], vd["state"],
                                              states_out=vst, out=vout)
        for _ in range(3):
            run_v()
        reps = 100
        vms, vprof = timed_passes(lambda i: run_v(), reps, world, dev, stream)
        name = "gdn_decode_verify_kernel"
        kms, kl = vprof.get(name, (vms, reps))
        per_bh = (1 + Tk) * d_ * d_ * 4 + Tk * ((3 * d_) * 2 + 2 * 4 + d_ * 2)
        bytes_per_launch = B_ * H_ * per_bh
        ach = bytes_per_launch / (kms / kl / 1e3) / 1e9
        pk, pu, pdesc = peak_for("hbm", peaks)
        verify = dict(workload="verify_b64_k4: B=64 sequences x 4 drafted tokens, H=32, dk=dv=128, bf16 q/k/v, "
                               "fp32 state read once, 4 per-token states written",
                      value=job_throughput(B_ * Tk, reps, world, vms), unit="tokens/s",
                      us_per_call=vms / reps * 1e3,
                      roofline=dict(kernel=name, bound="hbm", achieved=ach, peak=pk, unit=pu, frac=ach / pk,
                                    peak_source=pdesc, bytes_per_launch=bytes_per_launch,
                                    traffic=TRAFFIC.get(name)))
        del vd, vst, vout

    # ---- tree verify: B=64 sequences x 8 drafted tokens in a best-first tree ----
    verify_tree = None
    if not args.no_verify:
        w = WORKLOADS["verify_tree_b64_k8"]
        B_, Tk, H_, d_ = w.decode_batch, w.decode_steps, w.H, w.dk
        vd = make_verify_inputs(B_, H_, d_, d_, Tk, dtype=w.dtype, gate=w.gate, seed=w.seed + rank,
                                state_std=w.state_std, device=dev)
        tree = best_first_parents(Tk)
        par = torch.tensor([tree] * B_, dtype=torch.int32, device=dev)
        vst = torch.empty((B_, Tk, H_, d_, d_), dtype=torch.float32, device=dev)
        vout = torch.empty((B_, Tk, H_, d_), dtype=torch.bfloat16, device=dev)
        run_t = lambda: gdn.gdn_decode_verify_tree(vd["q"], vd["k"], vd["v"], vd["g"], vd["beta"], par, vd["state"],
                                                   states_out=vst, out=vout)
        for _ in range(3):
            run_t()
        reps = 50
        tms, tprof = timed_passes(lambda i: run_t(), reps, world, dev, stream)
        name = "gdn_decode_verify_kernel"
        kms, kl = tprof.get(name, (tms, reps))
        per_bh = (1 + Tk) * d_ * d_ * 4 + Tk * ((3 * d_) * 2 + 2 * 4 + d_ * 2)   # API bytes, as for the chain
        rereads = sum(1 for t in range(Tk) if tree[t] != t - 1 and tree[t] >= 0)
        bytes_per_launch = B_ * H_ * per_bh
        ach = bytes_per_launch / (kms / kl / 1e3) / 1e9
        pk, pu, pdesc = peak_for("hbm", peaks)
        verify_tree = dict(workload="verify_tree_b64_k8: B=64 sequences x 8 drafted tokens in the best-first tree "
                                    "%s (parent of each token, -1 = committed state), decode_b64 distributions"
                                    % tree,
                           value=job_throughput(B_ * Tk, reps, world, tms), unit="tokens/s",
                           us_per_call=tms / reps * 1e3,
                           roofline=dict(kernel=name, bound="hbm", achieved=ach, peak=pk, unit=pu, frac=ach / pk,
                                         peak_source=pdesc, bytes_per_launch=bytes_per_launch,
                                         note="API bytes only; %d tokens re-read their parent's state "
                                              "(%d x 64 KB per sequence-head more)" % (rereads, rereads),
                                         traffic=TRAFFIC.get("gdn_decode_verify_kernel (tree, verify_tree_b64_k8)")))
        del vd, vst, vout, par

    # ---- the other prefill workloads of the method ----
    workloads = None
    if not args.no_workloads:
        workloads = {}
        for wname, reps in (("varlen_resume", 20), ("long_128k", 5), ("tiny_fp32", 100)):
            workloads[wname] = bench_prefill_workload(wname, reps, world, dev, stream, peaks, rank)
            torch.cuda.empty_cache()

    clk = clocks.stop()

    # ---- roofline of the dominant prefill kernel ----
    dom = max((n for n in prof if "flops_per_token_head" in KERNELS.get(n, {})), key=lambda n: prof[n][0])
    kms, kl = prof[dom]
    spec = KERNELS[dom]
    units = T_PREFILL * H                             # (token, head) pairs per launch
    flops = spec["flops_per_token_head"] * spec["split"] * units
    ach = flops / (kms / kl / 1e3) / 1e12
    pk, pu, pdesc = peak_for(spec["bound"], peaks)
    total_prof_ms = sum(v[0] for v in prof.values())
    roofline = dict(kernel=dom, bound=spec["bound"], achieved=ach, peak=pk, unit=pu, frac=ach / pk,
                    peak_source=pdesc, flops_per_launch=flops, avg_launch_us=kms / kl * 1e3,
                    traffic=TRAFFIC.get(dom),
                    timing="CUDA events around each launch, in a second pass over the same K steps",
                    kernels={n: dict(avg_us=v[0] / v[1] * 1e3, launches=v[1], share=v[0] / total_prof_ms)
                             for n, v in prof.items()})
    # whole-call roofline of the method (TF32 3x split vs HBM), as the metric defines "% of roofline"
    method_roofline = method_roofline_of(T_PREFILL, H, D, N, False, ms_per_step, peaks)

    cpu = None
    cpu_all = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, spent, heads, toks = oracle_layer_rate(sets[0], budget_s=args.cpu_seconds)
        cpu = dict(value=rate, unit=UNIT, cores=1, kind="oracle",
                   sample="fp64 single-thread oracle recurrence over %d of %d heads x %d tokens of the %s workload "
                          "(%.1f s), scaled to a full layer" % (heads, H, toks, WORKLOAD, spent))
        if not args.no_cpu_all:
            arate, procs, awall = oracle_layer_rate_all_cores(H, T_PREFILL)
            cpu_all = dict(value=arate, unit=UNIT, cores=procs, kind="oracle",
                           host_cores=os.cpu_count(),
                           sample="the same single-thread fp64 oracle on all %d heads x %d tokens of the %s workload, "
                                  "one head per process on %d processes (spawn pool); median of 3 passes, %.2f s "
                                  "each" % (H, T_PREFILL, WORKLOAD, procs, awall))

    launches = sum(v[1] for v in prof.values())
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms_per_step, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16x3",
                per_call_ms=dict(median=statistics.median(per_call_ms), min=per_call_ms[0], max=per_call_ms[-1],
                                 calls=len(per_call_ms), timing="an event pair around each whole call"),
                data="synthetic",
                config=dict(workload="%s: %s" % (WORKLOAD, WORKLOAD_DESC), global_batch=world, seq_len=T_PREFILL,
                            parallelism="one independent prefill per GPU" if world > 1 else "1 GPU",
                            l2="3 rotating input sets, ~300 MB of q/k/v > 126 MB L2"),
                roofline=roofline, method_roofline=method_roofline, cpu_baseline=cpu,
                cpu_baseline_all_cores=cpu_all,
                e2e=dict(value=e2e_value, unit=UNIT, h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                         ms_per_step=e2e_ms / e2e_steps,
                         pipelining="copy-in, compute and copy-out on three streams, double-buffered",
                         steps=e2e_steps,
                         h2d_alone_ms_per_step=h2d_ms, h2d_gbs=h2d / (h2d_ms / 1e3) / 1e9,
                         bound="the host->device copy of each step's inputs (h2d_alone_ms_per_step)"),
                gpu_launches=launches, clocks=clk, decode=decode, verify=verify, verify_tree=verify_tree,
                cuts=cuts_line, norm=norm_line, workloads=workloads)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sharded(args, rank, world, local_rank):
    """--shard heads: one layer's prefill split by heads over the ranks (strong scaling).  Every rank
    builds the same layer (same seeds) and runs the library on its own contiguous block of heads;
    there is no data-path exchange.  value = the layer's tokens per second over the slowest rank.
    With --gather every step also all-gathers the output blocks (one NCCL all-gather), so that each
    rank holds the whole layer's output."""
    import torch
    import torch.distributed as dist
    from linear_attention_10_b200 import gdn
    from linear_attention_10_b200.shard import gather_heads, head_range, shard_heads
    from linear_attention_10_b200.workloads import workload_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    gdn.lib()
    stream = torch.cuda.current_stream()
    if args.gather and H % world:
        raise SystemExit("--gather needs the %d heads to divide evenly over %d ranks" % (H, world))
    h0, h1 = head_range(rank, world, H)
    Hl = h1 - h0
    sets = [shard_heads(workload_inputs(WORKLOAD, device=dev, seed=1000 + i), rank, world) for i in range(3)]
    ws = torch.empty(gdn.workspace_bytes(T_PREFILL, 1, Hl, D, D), dtype=torch.uint8, device=dev)
    out = torch.empty((T_PREFILL, Hl, D), dtype=torch.bfloat16, device=dev)
    st_out = torch.empty((1, Hl, D, D), dtype=torch.float32, device=dev)

    def step(i):
        s = sets[i % 3]
        gdn.gdn_chunk_prefill(s["q"], s["k"], s["v"], s["g"], s["beta"], cu_seqlens=s["cu_seqlens"],
                              out=out, state_out=st_out, workspace=ws)
        if args.gather:
            gather_heads(out, world)

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error during warm-up")
    clocks = ClockSampler(None)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    clk = clocks.stop()
    if gdn.gdn_get_device_status() != 0:
        raise RuntimeError("device status error in the timed region")
    if rank != 0:
        return
    value = T_PREFILL * args.steps / (ms / 1e3)
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms / args.steps, higher_is_better=True, scaling="strong", vs_baseline=None,
                dtype="bf16x3", data="synthetic",
                config=dict(workload="%s: %s" % (WORKLOAD, WORKLOAD_DESC), global_batch=1, seq_len=T_PREFILL,
                            parallelism="heads sharded over %d GPUs (%d heads on rank 0)%s"
                                        % (world, Hl, ", outputs all-gathered every step" if args.gather else ""),
                            l2="3 rotating input sets"),
                roofline=None, e2e=None, gpu_launches=3 * args.steps, clocks=clk,
                note="head-sharded layout of one layer; the default mode carries the roofline and e2e figures")
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-verify", action="store_true")
    ap.add_argument("--no-cuts", action="store_true")
    ap.add_argument("--no-norm", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the varlen / 128K / tiny prefill lines")
    ap.add_argument("--case", default=None, help="profiling aid: run only this workload's prefill")
    ap.add_argument("--case-tokens", type=int, default=0, help="with --case: keep only the first N tokens")
    ap.add_argument("--no-cpu-all", action="store_true", help="skip the all-cores oracle timing")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--shard", choices=["none", "heads"], default="none",
                    help="heads: split one layer's heads over the ranks instead of one prefill per rank")
    ap.add_argument("--gather", action="store_true", help="with --shard heads: all-gather the outputs every step")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.case:
        run_case(args, rank, world, local_rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.shard == "heads":
            run_sharded(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
