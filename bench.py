"""Benchmark of the context-parallel ring-attention hot path on B200.

One step = one pass of the hot path over the 128K full-prefill workload:
the load-balanced shard plan for 8 virtual ranks (host), the 8 pass-KV ring
steps (one cp_attn_partial launch each, tcgen05 kernel) and the 8-way LSE
merge into the bf16 output. Workload: Llama3-405B per-TP8-rank head slice,
N_H=16, N_KV=1, D_H=128, T=131072, bf16 inputs iid N(0,1)*0.5 (seeded,
synthetic). Inputs are resident in HBM and larger than L2 (no flush).
Beside the headline the same line reports: the roofline of the partial
kernel (per-launch CUDA events) with the DRAM traffic of the committed ncu
capture, the step with the merge fused into the partial kernel and with bf16
partial buffers, the step end to end from pinned host memory ("e2e"), the
split-KV decode workload (32 requests, 256 splits), the persistent-KV and
varlen workloads, cuDNN's fused attention on the same inputs (context only),
SM clocks sampled during the timed region, and the fp64 reference timed on
the host's cores on a sample of rows ("cpu_baseline").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 (launched by torchrun): every rank runs its own copy of the workload
(independent replicas, weak scaling, no data-path collective); the time is
the max over ranks and `value` counts the work of all ranks; the other
workloads, the context figure and the CPU baseline are measured at N = 1 only.
--impl reference times the fp64 reference (the host's cores) on the same
metric and configuration.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "causal prefill attn TFLOP/s; decode KV GB/s; % of B200 roofline, 1 GPU"
WORKLOAD = "prefill_128k"
DECODE = "decode_split"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "partial_bf16_prefill_128k.txt")
KERNEL_SOURCES = ["context_ring_attn_b200/csrc/partial_tc.cuh", "context_ring_attn_b200/csrc/common.cuh",
                  "context_ring_attn_b200/csrc/work.cuh"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def profiled_traffic():
    """Per-launch DRAM bytes of the partial kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    vals = {}
    with open(PROFILE_TRAFFIC) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------ reference arm
ORACLE_RUN = 256   # query rows per timed oracle call (the oracle's own row-group size)


def oracle_sample(budget_s: float, seed: int = 0, min_runs: int = 1, max_runs: int | None = None):
    """Time the fp64 oracle on runs of ORACLE_RUN consecutive query rows of the
    128K prefill starting at seeded random positions (all 16 heads, each row
    against its causal prefix), until budget_s of oracle time is spent and at
    least min_runs runs are done. Returns (flops, seconds, n_rows)."""
    from context_ring_attn_b200 import synth
    from oracle import attention as OA

    w = synth.WORKLOADS[WORKLOAD]
    t, n_h, n_kv, d = w["t"], w["n_h"], w["n_kv"], w["d"]
    k = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_K, t, (n_kv, d), w["std"]), "bf16")[0]
    v = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_V, t, (n_kv, d), w["std"]), "bf16")[0]
    k64, v64 = k.astype(np.float64), v.astype(np.float64)
    rng = np.random.default_rng(12345 + seed)
    flops, spent, n_rows, runs = 0.0, 0.0, 0, 0
    k_pos = np.arange(t)
    while (spent < budget_s or runs < min_runs) and (max_runs is None or runs < max_runs):
        r0 = int(rng.integers(0, t - ORACLE_RUN + 1))
        rows = np.arange(r0, r0 + ORACLE_RUN)
        q = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], rows), "bf16")[0]
        end = r0 + ORACLE_RUN
        t0 = time.perf_counter()
        OA.attention(q, k64[:end], v64[:end], rows, k_pos[:end])
        spent += time.perf_counter() - t0
        flops += 4.0 * d * n_h * float(np.sum(rows + 1))
        n_rows += ORACLE_RUN
        runs += 1
    return flops, spent, n_rows


SPEC = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}   # nominal dense bf16 and HBM3e of a B200


def headline_config(t: int, n_h: int, n_kv: int, d: int, n_ranks: int, world: int) -> dict:
    """The workload description both arms report (same keys, same values)."""
    pairs = t * (t + 1) // 2
    return {"workload": WORKLOAD if t == 131072 else f"{WORKLOAD} (T={t} profiling variant)",
            "T": t, "N_H": n_h, "N_KV": n_kv, "D_H": d, "cp_ranks": n_ranks,
            "plan": "load-balanced 16 chunks", "ring": "pass-KV", "merge": "final 8-way",
            "flops_per_step": 4.0 * d * n_h * pairs, "causal_pairs_per_head": pairs,
            "l2": "no flush: inputs larger than L2 (Q 537 MB, partials 8.6 GB per step)",
            "parallelism": f"{world} independent replica(s)"}


def peak_clock_mhz(peaks: dict):
    """Median SM clock under which the measured peaks were taken, if the peaks
    file records one (any numeric field whose name mentions a median SM clock)."""
    def walk(obj, path=""):
        if isinstance(obj, dict):
            for k, v in obj.items():
                yield from walk(v, f"{path}.{k}".lower())
        elif isinstance(obj, (int, float)) and not isinstance(obj, bool):
            yield path, float(obj)
    cands = [(p, v) for p, v in walk(peaks) if ("mhz" in p or "clock" in p) and "median" in p and "max" not in p]
    return cands[0][1] if cands else None


def fractions(achieved: float, peak: float, spec: float, peaks: dict, clk) -> dict:
    """achieved as a fraction of the measured peak, of the nominal spec peak,
    and of the measured peak scaled to the clock the kernel ran at."""
    out = {"frac_spec": achieved / spec, "spec_peak": spec}
    pc = peak_clock_mhz(peaks)
    run_mhz = (clk or {}).get("sm_mhz")
    if pc and run_mhz:
        out["frac_at_run_clock"] = achieved / (peak * run_mhz / pc)
        out["peak_clock_mhz"] = pc
        out["run_clock_mhz"] = run_mhz
    else:
        out["frac_at_run_clock"] = None
        out["note"] = "the peaks file records no median SM clock: no clock-normalised fraction"
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    cores = blas_threads()
    per_step = max(2.0, min(8.0, 120.0 / max(1, args.steps)))
    oracle_sample(0.0, seed=1000, max_runs=1)  # warm caches and BLAS threads (not timed)
    for i in range(args.warmup):
        oracle_sample(0.0, seed=2000 + i, max_runs=1)
    flops = secs = 0.0
    rows = 0
    for i in range(args.steps):
        f, s, n = oracle_sample(per_step, seed=i)
        flops, secs, rows = flops + f, secs + s, rows + n
    value = flops / secs / 1e12
    sample = (f"{rows} query rows of the 128K causal prefill in runs of {ORACLE_RUN} consecutive rows at seeded "
              f"random positions, all 16 heads, fp64 numpy, each row against its whole causal prefix; "
              f"{args.steps} steps of >= {per_step:.0f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(131072, 16, 1, 128, 8, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------ our arm
def run_ours(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    from context_ring_attn_b200 import binding as B
    from context_ring_attn_b200 import ring, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    w = synth.WORKLOADS[WORKLOAD]
    t, n_h, n_kv, d, n_ranks = w["t"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    if args.tokens:
        t = args.tokens
    scale = 1.0 / math.sqrt(d)
    q = synth.device_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], "bf16", dev)
    k = synth.device_rows(w["seed"], synth.TENSOR_K, t, (n_kv, d), w["std"], "bf16", dev)
    v = synth.device_rows(w["seed"], synth.TENSOR_V, t, (n_kv, d), w["std"], "bf16", dev)
    segs = [ring.Segment(t, 0, 0, 0)]
    o_parts, lse_parts = ring.partial_buffers(t, n_h, d, n_ranks, dev)
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((t, n_h), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    sched0 = ring.RingSchedule(segs, segs, n_ranks, B.CP_PASS_KV)
    pairs = sched0.pairs(True)
    step_flops = 4.0 * d * n_h * pairs
    step_pairs = [sum(B.cp_block_pairs(sched0.ranges, sched0.blocks[s * n_ranks + i], True)
                      for i in range(n_ranks)) for s in range(n_ranks)]

    ev_part = []  # (start, end, flops) of each partial launch in the timed region
    ev_merge = []

    nvtx = torch.cuda.nvtx

    def step(record: bool):
        nvtx.range_push("plan")
        sched = ring.RingSchedule(segs, segs, n_ranks, B.CP_PASS_KV)   # host plan, every step
        nvtx.range_pop()
        for s in range(n_ranks):
            blocks = sched.step_blocks(s, t)
            nvtx.range_push(f"ring step {s}")
            if record:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            B.cp_attn_partial(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges, blocks, n_ranks,
                              o_parts, lse_parts, ws)
            if record:
                e1.record(stream)
                ev_part.append((e0, e1, 4.0 * d * n_h * step_pairs[s]))
            nvtx.range_pop()
        nvtx.range_push("merge")
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        B.cp_attn_merge(o_parts, lse_parts, n_ranks, t, t, n_h, d, out, lse)
        if record:
            e1.record(stream)
            ev_merge.append((e0, e1))
        nvtx.range_pop()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    B.cp_check_status(ws)

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    B.cp_check_status(ws)
    elapsed_ms = t_start.elapsed_time(t_end)
    part_ms = sum(a.elapsed_time(b) for a, b, _ in ev_part)
    part_flops = sum(f for _, _, f in ev_part)
    merge_ms = sum(a.elapsed_time(b) for a, b in ev_merge)
    if world > 1:
        tt = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        elapsed_ms = float(tt.item())

    # the same step with the LSE merge fused into the partial kernel's epilogue:
    # one running (O, LSE) buffer, the last ring step writes the bf16 output
    o_acc = o_parts[:t]

    def fused_step():
        sched = ring.RingSchedule(segs, segs, n_ranks, B.CP_PASS_KV)
        for s in range(n_ranks):
            blocks = sched.step_blocks(s, t, part_of=lambda _p: 0)
            B.cp_attn_partial_fused(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges, blocks, n_ranks,
                                    o_acc, lse, s > 0, out if s == n_ranks - 1 else None, ws)

    fused_ms = None
    for _ in range(0 if args.no_fused else max(2, args.warmup)):
        fused_step()
    barrier()
    torch.cuda.synchronize()
    if not args.no_fused:
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            fused_step()
        f1.record(stream)
        torch.cuda.synchronize()
        B.cp_check_status(ws)
        fused_ms = f0.elapsed_time(f1) / args.steps
    if world > 1 and fused_ms is not None:
        tt = torch.tensor([fused_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        fused_ms = float(tt.item())

    # the same step with bf16 partial O buffers (cp_attn_partial_bf16_parts, then
    # cp_attn_merge_bf16_parts): half the partial bytes written and read
    o_parts16 = o_parts.view(-1).view(torch.bfloat16)[:n_ranks * t * n_h * d].view(n_ranks * t, n_h, d)  # same memory

    def bf16_step():
        sched = ring.RingSchedule(segs, segs, n_ranks, B.CP_PASS_KV)
        for s in range(n_ranks):
            B.cp_attn_partial_bf16_parts(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges,
                                         sched.step_blocks(s, t), n_ranks, o_parts16, lse_parts, ws)
        B.cp_attn_merge(o_parts16, lse_parts, n_ranks, t, t, n_h, d, out, lse)

    bf16_ms = None
    if not args.no_fused:
        for _ in range(max(2, args.warmup)):
            bf16_step()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            bf16_step()
        f1.record(stream)
        torch.cuda.synchronize()
        B.cp_check_status(ws)
        bf16_ms = f0.elapsed_time(f1) / args.steps
    if world > 1 and bf16_ms is not None:
        tt = torch.tensor([bf16_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        bf16_ms = float(tt.item())

    e2e = run_e2e(args, q, k, v, out, lse, o_parts, lse_parts, ws, segs, n_ranks, n_h, n_kv, world, dev,
                  step_flops, barrier) if not args.no_e2e else None
    # The other workloads, the library context and the CPU baseline are
    # measured at N = 1 only: with N > 1 every rank would repeat the same
    # single-GPU figures while all N GPUs are held.
    single = world == 1
    decode = run_decode(args, dev) if single and not args.no_decode else None
    context = run_library_context(args, dev) if single and not args.no_context else None
    secondary = {}
    if single and not args.no_secondary:
        for name in ("persistent_kv", "varlen_prefill"):
            secondary[name] = run_secondary(args, dev, name)
        secondary["varlen_prefill_fused_merge"] = run_secondary(args, dev, "varlen_prefill", "fused")
        secondary["varlen_prefill_running_merge"] = run_secondary(args, dev, "varlen_prefill", "running")

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    peak_t = float(peaks["bf16_tflops_sustained"])
    achieved = part_flops / (part_ms * 1e-3) / 1e12
    traffic = profiled_traffic() if t == w["t"] else None
    value = world * step_flops * args.steps / (elapsed_ms * 1e-3) / 1e12
    merge_bytes = n_ranks * t * n_h * (d + 1) * 4 + t * n_h * (d * 2 + 4)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": headline_config(t, n_h, n_kv, d, n_ranks, world),
        "roofline": {"kernel": "partial_bf16_kernel", "bound": "tensor", "achieved": achieved, "peak": peak_t,
                     "unit": "TFLOP/s", "frac": achieved / peak_t, "traffic": traffic,
                     "peak_kind": f"bf16_tflops_sustained ({peak_kind})",
                     "kernel_ms_per_step": part_ms / args.steps,
                     **fractions(achieved, peak_t, SPEC["bf16_tflops"], peaks, clk)},
        "merge": {"ms_per_step": merge_ms / args.steps,
                  "gbs": merge_bytes / (merge_ms / args.steps * 1e-3) / 1e9,
                  "frac_hbm": merge_bytes / (merge_ms / args.steps * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                  "frac_hbm_spec": merge_bytes / (merge_ms / args.steps * 1e-3) / 1e9 / SPEC["hbm_gbs"]},
        "fused_merge": None if fused_ms is None else {
            "value": world * step_flops / (fused_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": fused_ms,
            "note": "same step, LSE merge in the partial kernel's epilogue (cp_attn_partial_fused): "
                    "8 launches, one running buffer, no merge pass"},
        "bf16_partials": None if bf16_ms is None else {
            "value": world * step_flops / (bf16_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": bf16_ms,
            "note": "same step with bf16 partial O buffers (cp_attn_partial_bf16_parts + cp_attn_merge_bf16_parts): "
                    "8 launches + one 8-way merge reading half the partial bytes"},
        "e2e": e2e,
        "gpu_launches": args.steps * (n_ranks + 1),
        "clocks": clk,
    }
    if decode:
        line["decode"] = decode
    if context:
        line["library_context"] = context
    if secondary:
        line["workloads"] = secondary
    if not single:
        line["secondary_legs"] = "decode, other workloads, library context and cpu_baseline are measured at N=1 only"
    if single and not args.no_cpu_baseline:
        f, s, n = oracle_sample(0.0, seed=0, min_runs=args.cpu_rows // ORACLE_RUN)
        rate = f / s
        line["cpu_baseline"] = {
            "value": rate / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} query rows of the 128K causal prefill in runs of {ORACLE_RUN} consecutive rows at "
                      f"seeded random positions, all 16 heads, fp64 numpy against each row's causal prefix "
                      f"({s:.1f} s)",
            "rows": n, "rows_per_s": n / s, "seconds": s,
            "extrapolated_full_step_s": step_flops / rate,
            "extrapolated_note": "extrapolated: one full 128K step's flops at the sampled rate"}
    print(json.dumps(line), flush=True)


def run_e2e(args, q, k, v, out, lse, o_parts, lse_parts, ws, segs, n_ranks, n_h, n_kv, world, dev, step_flops,
            barrier):
    import torch
    import torch.distributed as dist

    from context_ring_attn_b200 import binding as B
    from context_ring_attn_b200 import ring

    stream = torch.cuda.current_stream()
    # ---- end to end through the public API with host buffers (pinned). Every
    # step copies its Q, K, V from pinned host memory and its O and LSE back;
    # over a run of steps the copies of the next and previous steps proceed on
    # their own streams (the copy engines) while the current step computes:
    # device inputs and outputs are double-buffered and ordered by events.
    bufs = [(q, k, v, out, lse), tuple(torch.empty_like(x) for x in (q, k, v, out, lse))]
    hosts = []
    for b in range(2):
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        hq.copy_(q)
        hk.copy_(k)
        hv.copy_(v)
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        hosts.append((hq, hk, hv, ho, hl))
    torch.cuda.synchronize()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    computed = [None, None]   # compute of the last step that used buffer b is done
    drained = [None, None]    # D2H of the last step that used buffer b is done

    def e2e_step(i):
        b = i % 2
        dq, dk, dv, do, dl = bufs[b]
        hq, hk, hv, ho, hl = hosts[b]
        with torch.cuda.stream(s_in):
            if computed[b] is not None:
                s_in.wait_event(computed[b])
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            ready = ev()
            ready.record(s_in)
        stream.wait_event(ready)
        if drained[b] is not None:
            stream.wait_event(drained[b])
        ring.run_ring(ring.RingSchedule(segs, segs, n_ranks, B.CP_PASS_KV), dq, dk, dv, n_h, n_kv, do, dl,
                      o_parts=o_parts, lse_parts=lse_parts, workspace=ws)
        computed[b] = ev()
        computed[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            ho.copy_(do, non_blocking=True)
            hl.copy_(dl, non_blocking=True)
            drained[b] = ev()
            drained[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(4, args.steps)   # as many steps as the device-resident measurement
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(drained[b])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        tt = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = out.numel() * 2 + lse.numel() * 4
    del bufs, hosts
    return {"value": world * step_flops * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
            "note": "per step: H2D of Q/K/V from pinned host memory, the ring, D2H of O/LSE; copies of "
                    "neighbouring steps overlap the compute on two copy streams (double-buffered)"}


def run_secondary(args, dev, name: str, merge_override: str | None = None):
    """The other prefill workloads, each a full ring schedule per step:
    persistent-KV partial prefill (T=4096 new over P=126976 cached, 128/8
    heads, pass-Q, 8-way merge) and the varlen batch (8 sequences, 262144
    tokens, 128/8 heads, pass-KV; bf16 partial buffers, 8.6 GB per part, and
    one 8-way merge; merge_override="fused" times the merge in the partial
    kernel's epilogue with one fp32 running buffer, "running" separate 2-way
    merges)."""
    import torch

    from context_ring_attn_b200 import binding as B
    from context_ring_attn_b200 import ring, synth

    w = synth.WORKLOADS[name]
    n_h, n_kv, d, n = w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    scale = 1.0 / math.sqrt(d)
    shrink = max(1, args.shrink)   # profiling captures: every length divided by this (the mix kept)
    if name == "persistent_kv":
        t, p = w["t"] // shrink, w["p"] // shrink
        q_segs = [ring.Segment(t, 0, p, 0)]
        kv_segs = [ring.Segment(p, 0, 0, 0), ring.Segment(t, p, p, 0)]
        kv_rows, variant, merge = p + t, B.CP_PASS_Q, "final"
        desc = {"T": t, "P": p, "ring": "pass-Q", "merge": "final 8-way"}
    else:
        lens = [ln // shrink for ln in synth.varlen_lengths(w["seed"], w["n_seq"], w["total"])]
        t = sum(lens)
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        q_segs = kv_segs = [ring.Segment(int(ln), int(s0), 0, i) for i, (ln, s0) in enumerate(zip(lens, starts))]
        kv_rows, variant, merge = t, B.CP_PASS_KV, "final_bf16"
        desc = {"seq_lens": [int(x) for x in lens], "ring": "pass-KV",
                "merge": ("final 8-way over bf16 partial buffers (cp_attn_partial_bf16_parts, then "
                          "cp_attn_merge_bf16_parts)")}
    if merge_override == "running":
        merge = "running"
        desc["merge"] = "running 2-way (cp_attn_merge after every step)"
    elif merge_override == "fused":
        merge = "fused"
        desc["merge"] = "fused into the partial kernel's epilogue (cp_attn_partial_fused), one running buffer"
    q = synth.device_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], "bf16", dev)
    k = synth.device_rows(w["seed"], synth.TENSOR_K, kv_rows, (n_kv, d), w["std"], "bf16", dev)
    v = synth.device_rows(w["seed"], synth.TENSOR_V, kv_rows, (n_kv, d), w["std"], "bf16", dev)
    n_bufs = n if merge in ("final", "final_bf16") else (1 if merge == "fused" else 2)
    o_parts, lse_parts = ring.partial_buffers(t, n_h, d, n_bufs, dev,
                                              torch.bfloat16 if merge == "final_bf16" else torch.float32)
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((t, n_h), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sched0 = ring.RingSchedule(q_segs, kv_segs, n, variant)
    pairs = sched0.pairs(True)
    step_flops = 4.0 * d * n_h * pairs
    ev_part, ev_merge = [], []

    def step(record):
        sched = ring.RingSchedule(q_segs, kv_segs, n, variant)
        for s_ in range(n):
            if merge in ("final", "final_bf16"):
                target = lambda pt: pt
            elif merge == "fused":
                target = lambda _pt: 0
            else:
                target = lambda _pt, _t=(0 if s_ == 0 else 1): _t
            blocks = sched.step_blocks(s_, t, part_of=target)
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) if record else None
            if e:
                e[0].record(stream)
            if merge == "fused":
                B.cp_attn_partial_fused(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges, blocks, n,
                                        o_parts, lse, s_ > 0, out if s_ == n - 1 else None, ws)
            elif merge == "final_bf16":
                B.cp_attn_partial_bf16_parts(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges, blocks,
                                             n, o_parts, lse_parts, ws)
            else:
                B.cp_attn_partial(q, k, v, n_h, n_kv, scale, True, sched.ranges, sched.n_ranges, blocks, n,
                                  o_parts, lse_parts, ws)
            if e:
                e[1].record(stream)
                ev_part.append(e)
            if merge == "running" and s_ > 0:
                last = s_ == n - 1
                e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) if record else None
                if e:
                    e[0].record(stream)
                B.cp_attn_merge(o_parts, lse_parts, 2, t, t, n_h, d, out if last else o_parts,
                                lse if last else lse_parts)
                if e:
                    e[1].record(stream)
                    ev_merge.append((e, 2 * t * n_h * (d + 1) * 4 + t * n_h * ((2 * d + 4) if last else (d + 1) * 4)))
        if merge in ("final", "final_bf16"):
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) if record else None
            if e:
                e[0].record(stream)
            B.cp_attn_merge(o_parts, lse_parts, n, t, t, n_h, d, out, lse)
            if e:
                e[1].record(stream)
                part_bytes = n * t * n_h * (d * (2 if merge == "final_bf16" else 4) + 4)
                ev_merge.append((e, part_bytes + t * n_h * (2 * d + 4)))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    steps = max(2, args.steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step(True)
    e1.record(stream)
    torch.cuda.synchronize()
    B.cp_check_status(ws)
    ms = e0.elapsed_time(e1) / steps
    part_ms = sum(a.elapsed_time(b) for a, b in ev_part) / steps
    merge_ms = sum(a.elapsed_time(b) for (a, b), _ in ev_merge) / steps
    merge_bytes = sum(nb for _, nb in ev_merge) / steps
    no_merge = merge_ms == 0
    peaks, kind = load_peaks()
    peak_t = float(peaks["bf16_tflops_sustained"])
    res = {"value": step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "steps": steps,
           "flops_per_step": step_flops, "N_H": n_h, "N_KV": n_kv, "cp_ranks": n, **desc,
           "partial_tflops": step_flops / (part_ms * 1e-3) / 1e12,
           "partial_frac": step_flops / (part_ms * 1e-3) / 1e12 / peak_t,
           "partial_frac_spec": step_flops / (part_ms * 1e-3) / 1e12 / SPEC["bf16_tflops"],
           "merge_gbs": None if no_merge else merge_bytes / (merge_ms * 1e-3) / 1e9,
           "merge_frac_hbm": None if no_merge else merge_bytes / (merge_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
           "peak_kind": f"bf16_tflops_sustained / hbm_gbs ({kind})"}
    del q, k, v, o_parts, lse_parts, out, lse
    torch.cuda.empty_cache()
    return res


def run_library_context(args, dev):
    """Context figure, not the product path: cuDNN's fused attention (torch's
    scaled_dot_product_attention restricted to the cuDNN backend) on the same
    causal 128K problem as one unsharded call, K/V expanded to the 16 query
    heads, same bf16 inputs. Timed with CUDA events after warm-up."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel

    from context_ring_attn_b200 import synth

    w = synth.WORKLOADS[WORKLOAD]
    t, n_h, d = w["t"], w["n_h"], w["d"]
    if args.tokens:
        t = args.tokens
    try:
        q = synth.device_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], "bf16", dev)
        k = synth.device_rows(w["seed"], synth.TENSOR_K, t, (1, d), w["std"], "bf16", dev)
        v = synth.device_rows(w["seed"], synth.TENSOR_V, t, (1, d), w["std"], "bf16", dev)
        qh = q.permute(1, 0, 2).unsqueeze(0).contiguous()
        kh = k.permute(1, 0, 2).expand(n_h, t, d).unsqueeze(0).contiguous()
        vh = v.permute(1, 0, 2).expand(n_h, t, d).unsqueeze(0).contiguous()
        del q, k, v
        stream = torch.cuda.current_stream()
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            for _ in range(2):
                F.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
            torch.cuda.synchronize()
            reps = 5
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                F.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
            e1.record(stream)
            torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        flops = 4.0 * d * n_h * t * (t + 1) / 2
        del qh, kh, vh
        torch.cuda.empty_cache()
        return {"cudnn_sdpa": {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms,
                               "note": "context only: one unsharded causal call through cuDNN's fused attention "
                                       "(torch SDPA, cuDNN backend), K/V expanded to 16 heads; not this library"}}
    except Exception as exc:   # a missing backend is reported, not fatal
        torch.cuda.empty_cache()
        return {"cudnn_sdpa": {"unavailable": f"{type(exc).__name__}: {str(exc)[:200]}"}}


def run_decode(args, dev):
    """Split-KV decode: 32 requests, 16 heads on 1 KV head, 256 splits; GB/s
    of K/V read (each byte once)."""
    import torch

    from context_ring_attn_b200 import binding as B
    from context_ring_attn_b200 import synth

    w = synth.WORKLOADS[DECODE]
    lens = synth.decode_lengths(w["seed"], w["batch"], w["lo"], w["hi"])
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(offsets[-1])
    b, n_h, n_kv, d, ns = w["batch"], w["n_h"], w["n_kv"], w["d"], w["n_splits"]
    q = synth.device_rows(w["seed"], synth.TENSOR_Q, b, (n_h, d), w["std"], "bf16", dev)
    k = synth.device_rows(w["seed"], synth.TENSOR_K, total, (n_kv, d), w["std"], "bf16", dev)
    v = synth.device_rows(w["seed"], synth.TENSOR_V, total, (n_kv, d), w["std"], "bf16", dev)
    off = torch.from_numpy(offsets).to(dev)
    out = torch.empty((b, n_h, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, n_h), dtype=torch.float32, device=dev)
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, b, n_h, d, ns), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        B.cp_decode(q, k, v, off, n_h, n_kv, ns, 1 / math.sqrt(d), out, lse, ws)
    torch.cuda.synchronize()
    iters = max(10, args.steps)
    kv_bytes = total * n_kv * d * 2 * 2
    peaks, kind = load_peaks()

    def timed(fn, between=None):
        """Median device time of fn over iterations; `between` runs before each
        one, outside the timed region."""
        ts = []
        for _ in range(iters):
            if between is not None:
                between()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(c) for a, c in ts)

    run = lambda: B.cp_decode(q, k, v, off, n_h, n_kv, ns, 1 / math.sqrt(d), out, lse, ws)  # noqa: E731
    # K/V (1.26 GB) is ten times L2: no flush is needed between iterations. A
    # 256 MB write between iterations leaves L2 full of dirty lines that the
    # decode must write back, a 256 MB read leaves it full of clean ones: both
    # are reported beside the headline.
    ms = timed(run)
    ms_wflush = timed(run, lambda: flush.fill_(1))
    ms_rflush = timed(run, lambda: flush.view(torch.int32).sum())
    B.cp_check_status(ws)
    gbs = kv_bytes / (ms * 1e-3) / 1e9

    # the same decode captured once in a CUDA graph and replayed
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        B.cp_decode(q, k, v, off, n_h, n_kv, ns, 1 / math.sqrt(d), out, lse, ws)
    g.replay()
    graph_ms = timed(g.replay)
    B.cp_check_status(ws)
    del g

    # context-parallel decode over 8 virtual ranks: per-rank partials + merge
    from context_ring_attn_b200 import ring
    n_cp = 8
    cp = ring.DecodeCP(k, v, offsets, n_cp)
    o_parts, lse_parts, ws_cp = cp.buffers(q, ns)
    q_ranks = q.repeat(n_cp, 1, 1)
    run_cp = lambda: cp.run(q_ranks, n_kv, ns, 1 / math.sqrt(d), out, lse, o_parts, lse_parts, ws_cp)
    for _ in range(3):
        run_cp()
    cp_ms = timed(run_cp)
    B.cp_check_status(ws_cp)
    return {"value": gbs, "unit": "GB/s", "ms": ms, "kv_bytes": kv_bytes, "batch": b, "n_splits": ns,
            "frac_hbm": gbs / float(peaks["hbm_gbs"]), "peak": float(peaks["hbm_gbs"]),
            "frac_hbm_spec": gbs / SPEC["hbm_gbs"],
            "peak_kind": f"hbm_gbs ({kind})",
            "l2": "no flush: K/V (1.26 GB) is larger than L2",
            "after_l2_write_flush": {"ms": ms_wflush, "value": kv_bytes / (ms_wflush * 1e-3) / 1e9, "unit": "GB/s",
                                     "note": "a 256 MB buffer written before each iteration (its dirty lines are "
                                             "written back during the decode)"},
            "after_l2_read_flush": {"ms": ms_rflush, "value": kv_bytes / (ms_rflush * 1e-3) / 1e9, "unit": "GB/s",
                                    "note": "a 256 MB buffer read before each iteration"},
            "note": "balanced split kernel (8 ranges per SM) + per-head merge, median of iterations",
            "graph": {"ms": graph_ms, "value": kv_bytes / (graph_ms * 1e-3) / 1e9, "unit": "GB/s",
                      "note": "cp_decode captured once in a CUDA graph, replayed"},
            "cp8": {"ms": cp_ms, "value": kv_bytes / (cp_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "note": "KV sharded over 8 virtual ranks (load-balanced chunks of every request); "
                            "every rank decodes every query against its shard (one batched launch), "
                            "then the 8-way LSE merge"}}


SWEEP_MISS = (0.01, 0.025, 0.0325, 0.05, 0.10, 0.20, 0.50, 1.00)
SWEEP_LINKS = {"rdma_400gbps": 50e9, "nvlink_peer_measured": 770e9}


def run_sweep(args, dev):
    """Algorithm 1 sweep: persistent-KV prefill with T + P = 128000 (128/8
    heads, D_H 128, bf16, 8 virtual ranks) at the method page's miss rates.
    Per point and variant, the GPU time of the whole ring schedule (all N^2
    blocks, running 2-way merges) is measured on one GPU; a rank of an N-GPU
    ring does 1/N of it and 1/N^2 per ring step. The ring's exposed transfer
    is modelled per link: pass-KV (N-1) hops of a KV shard, each hidden under
    a step up to its length; pass-Q (N-1) hops of a Q shard likewise, plus the
    all-to-all of the fp32 partials (not overlapped). The selector is
    cp_select_ring_variant fed the measured step time."""
    import torch

    from context_ring_attn_b200 import binding as B
    from context_ring_attn_b200 import ring, synth

    n_h, n_kv, d, n, total = 128, 8, 128, 8, 128000
    scale = 1.0 / math.sqrt(d)
    seed = synth.WORKLOADS["persistent_kv"]["seed"]
    q_all = synth.device_rows(seed, synth.TENSOR_Q, total, (n_h, d), 0.5, "bf16", dev)
    k = synth.device_rows(seed, synth.TENSOR_K, total, (n_kv, d), 0.5, "bf16", dev)
    v = synth.device_rows(seed, synth.TENSOR_V, total, (n_kv, d), 0.5, "bf16", dev)
    o_all = torch.empty((2 * total, n_h, d), dtype=torch.float32, device=dev)
    l_all = torch.empty((2 * total, n_h), dtype=torch.float32, device=dev)
    out_all = torch.empty((total, n_h, d), dtype=torch.bfloat16, device=dev)
    lse_all = torch.empty((total, n_h), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    points = []
    for miss in SWEEP_MISS:
        t = int(round(miss * total))
        p = total - t
        q = q_all[:t]
        q_segs = [ring.Segment(t, 0, p, 0)]
        kv_segs = [ring.Segment(p, 0, 0, 0), ring.Segment(t, p, p, 0)] if p > 0 else [ring.Segment(t, 0, 0, 0)]
        res = {"miss_rate": miss, "T": t, "P": p}
        for name, variant in (("pass_kv", B.CP_PASS_KV), ("pass_q", B.CP_PASS_Q)):
            sched = ring.RingSchedule(q_segs, kv_segs, n, variant)

            def once():
                ring.run_ring(sched, q, k, v, n_h, n_kv, out_all[:t], lse_all[:t], True, scale,
                              o_all[:2 * t], l_all[:2 * t], ws, merge="running")
            once()
            reps = 3
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                once()
            e1.record(stream)
            torch.cuda.synchronize()
            res[name + "_gpu_ms"] = e0.elapsed_time(e1) / reps
        B.cp_check_status(ws)
        flops = 4.0 * d * n_h * (t * p + t * (t + 1) / 2)
        res["tflop"] = flops / 1e12
        res["links"] = {}
        for lname, bw in SWEEP_LINKS.items():
            r = {}
            for name in ("pass_kv", "pass_q"):
                rank_ms = res[name + "_gpu_ms"] / n
                step_ms = rank_ms / n
                if name == "pass_kv":
                    hop_ms = (t + p) / n * n_kv * d * 2 * 2 / bw * 1e3
                    a2a_ms = 0.0
                else:
                    hop_ms = t / n * n_h * d * 2 / bw * 1e3
                    a2a_ms = (n - 1) * (t / n) * n_h * (d + 1) * 4 / bw * 1e3
                r[name + "_ms"] = rank_ms + (n - 1) * max(0.0, hop_ms - step_ms) + a2a_ms
            step_kv_s = res["pass_kv_gpu_ms"] / n / n * 1e-3
            var, why = B.cp_select_ring_variant(t, p, n_h, n_kv, d, n, 2, bw, step_kv_s)
            r["faster"] = "pass_kv" if r["pass_kv_ms"] <= r["pass_q_ms"] else "pass_q"
            r["selected"] = "pass_kv" if var == B.CP_PASS_KV else "pass_q"
            r["selector_condition"] = why
            res["links"][lname] = r
        points.append(res)
    del q_all, k, v, o_all, l_all, out_all, lse_all
    torch.cuda.empty_cache()
    return {"workload": "persistent-KV prefill, T+P=128000, N_H=128, N_KV=8, D_H=128, bf16, 8 virtual ranks",
            "links_bytes_per_s": SWEEP_LINKS, "points": points,
            "note": "gpu_ms: whole ring schedule on one GPU (measured); per-link totals are one rank of an "
                    "8-GPU ring (measured compute / 8 + modelled exposed transfer)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=2048, help="query rows the CPU baseline times (runs of 256)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-context", action="store_true", help="skip the cuDNN context figure")
    ap.add_argument("--no-fused", action="store_true", help="skip timing the fused-merge variant of the step")
    ap.add_argument("--no-secondary", action="store_true", help="skip the persistent-KV and varlen workloads")
    ap.add_argument("--only-decode", action="store_true", help="time the split-KV decode workload alone")
    ap.add_argument("--only-workload", choices=["persistent_kv", "varlen_prefill"], default=None,
                    help="time one of the other prefill workloads alone (prints its own line)")
    ap.add_argument("--merge", choices=["fused", "running"], default=None,
                    help="with --only-workload varlen_prefill: the merge mode")
    ap.add_argument("--shrink", type=int, default=1,
                    help="with --only-workload: divide every length by this (smaller profiling captures)")
    ap.add_argument("--sweep-miss-rate", action="store_true",
                    help="Algorithm 1 sweep of pass-KV vs pass-Q over KV-cache miss rates (prints its own line)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="shorter sequence for profiling captures (default: the full 131072)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    import torch.distributed as dist
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    try:
        if args.only_decode:
            print(json.dumps({"decode": run_decode(args, torch.device("cuda", local))}), flush=True)
            return
        if args.only_workload:
            res = run_secondary(args, torch.device("cuda", local), args.only_workload, args.merge)
            print(json.dumps({args.only_workload: res, "shrink": args.shrink}), flush=True)
            return
        if args.sweep_miss_rate:
            if rank == 0:
                print(json.dumps({"sweep": run_sweep(args, torch.device("cuda", local))}), flush=True)
            return
        run_ours(args, rank, world)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
