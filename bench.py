#!/usr/bin/env python
"""Prefill benchmark of the DSA / IndexCache hot path on B200.

One step = one pass of the whole hot path over one 200000-token prefill: the
4-layer F,S,S,S stack through ``ic_layer_stack`` (F layer: lightning indexer ->
exact top-k (k=2048) -> T_cache; every layer: sparse MLA attention over
T_cache).  Inputs are seeded synthetic tensors resident in HBM (they are larger
than L2, so no flush is needed between steps).

Rank 0 prints one JSON line.  Besides the contract keys it carries:
  roofline      the dominant kernel (the tensor-core indexer) against the
                measured bf16 peak, from CUDA events recorded after every launch
                inside the timed region (ic_trace_begin / ic_trace_end);
  stages        per-kernel device time per step and its own roofline;
  all_f         the same stack with every layer F, and the F,S,S,S speed-up;
  e2e           the metric through the C ABI with host buffers (H2D of the
                step's inputs and D2H of its result inside the timed region);
  cpu_baseline  the fp64 CPU oracle on a bounded sample of rows, extrapolated;
  decode        64 sequences x 1 new token over a 200000-token context (e4m3
                indexer key cache, bf16 latent KV cache), F,S,S,S and all-F,
                against the measured HBM bandwidth;
  stack_32k     the 8-layer F,S,S,S,F,S,S,S stack at L=32768 against all-F,
                with the overlap of adjacent layers' index sets under all-F.

``--impl reference`` times the CPU oracle (the reference of this repository)
on the same workload, metric and unit instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_attention_indexer_sum_b200 import synth  # noqa: E402

METRIC = "prefill tokens/s (indexer+top-k+sparse attn) at L=200K; % of roofline"
# DRAM bytes (read + write) per causal (query, key) pair of the bf16 tensor-core
# indexer, from one ncu capture of the current kernel on 512 query rows at
# position 100000 (`profile_cases indexer_longrows`: 203.9 MB for 51,331,328
# pairs).  The score writes dominate and grow with the pairs; keys and queries
# come from L2.  A launch's traffic is this figure times its pairs.
INDEXER_BF16_DRAM_BYTES_PER_PAIR = 203.9e6 / 51331328
# The same for the e4m3 indexer (`profile_cases indexer_longrows_e4m3`, same rows and
# positions, the kernel with four one-token epilogue warps per lane quadrant:
# 20.7 MB read + 152.0 MB written for the same 51,331,328 pairs).
INDEXER_E4M3_DRAM_BYTES_PER_PAIR = 172.78e6 / 51331328
UNIT = "tokens/s"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms; only samples taken inside mark()..stop() count."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.dev = device_id
        self.proc = None
        self.t_mark = None
        self.path = os.path.join("/tmp", "ic_clocks_%d.csv" % os.getpid())

    def mark(self):
        self.t_mark = time.time()

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception as e:  # pragma: no cover - no nvidia-smi
            log("clock sampling unavailable:", e)
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        t_end = time.time()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        import datetime
        with open(self.path) as f:
            for ln in f:
                p = [x.strip() for x in ln.split(",")]
                if len(p) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    if self.t_mark is not None and not (self.t_mark <= ts <= t_end + 0.2):
                        continue
                    sm.append(float(p[1]))
                    mx = max(mx, float(p[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ fp8 peak
def measure_fp8_peak(dev, sustain_s: float = 3.0):
    """Dense e4m3 GEMM throughput on this GPU, the denominator of the e4m3 indexer's
    roofline: torch._scaled_mm (cuBLASLt) on 8192^3 e4m3 x e4m3 -> bf16 with unit
    fp32 scales, 2 n^3 flop per call, CUDA events on the current stream.  Burst: the
    best of 10 timed groups of 5 calls.  Sustained: calls back to back for
    `sustain_s` seconds under the power cap, with the SM clocks sampled meanwhile.
    Both accumulation modes are timed and the faster one is the peak."""
    n = 8192
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)
    flop = 2.0 * n ** 3
    stream = torch.cuda.current_stream(dev)
    res = {"how": "torch._scaled_mm e4m3 %d^3 -> bf16, unit scales; burst = best of 10 groups "
                  "of 5 calls, sustained = back to back for %.0f s" % (n, sustain_s)}
    best = None
    for fast in (False, True):
        def mm(fast=fast):
            return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one,
                                    out_dtype=torch.bfloat16, use_fast_accum=fast)
        try:
            for _ in range(5):
                mm()
            torch.cuda.synchronize(dev)
        except Exception as e:  # no fp8 GEMM on this torch / GPU
            res["error_fast_accum_%s" % fast] = str(e).splitlines()[0][:200]
            continue
        burst = min(_timed(mm, 5, stream) for _ in range(10))
        if best is None or burst < best[1]:
            best = (fast, burst, mm)
        res["burst_tflops_fast_accum_%s" % str(fast).lower()] = flop / (burst * 1e-3) / 1e12
    if best is None:
        return res
    fast, burst, mm = best
    calls = max(10, int(sustain_s * 1e3 / burst))
    clocks = ClockSampler("GPU-%s" % torch.cuda.get_device_properties(dev).uuid)
    clocks.start()
    time.sleep(0.3)
    clocks.mark()
    ms = _timed(mm, calls, stream)
    res.update(fp8_tflops=flop / (burst * 1e-3) / 1e12,
               fp8_tflops_sustained=flop / (ms * 1e-3) / 1e12, use_fast_accum=fast,
               sustained_calls=calls, clocks=clocks.stop())
    del a, b
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------ ranks
def reduce_max(x: float, world: int, device) -> float:
    """The largest of every rank's x (one all-reduce; the identity on one rank).
    Every rank must call it the same number of times, in the same order."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own sequence (weak scaling) and
    the job takes as long as its slowest rank."""
    return world * tokens_per_rank / (ms_max * 1e-3)


# ------------------------------------------------------------------------------ workload
def make_inputs(wl, device, pattern_all, fp8: bool, seed: int):
    """Device tensors for every layer; indexer inputs for every layer that is F in any
    of the patterns run."""
    from sparse_attention_indexer_sum_b200 import binding as ic
    kinds_any = [any(p[i] == "F" for p in pattern_all) for i in range(wl.layers)]
    layers = []
    for l in range(wl.layers):
        d = {}
        if kinds_any[l]:
            d.update(synth.indexer_inputs(wl, l, device=device, seed=seed))
            if fp8:
                d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
                d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
        d.update(synth.attn_inputs(wl, l, device=device, seed=seed))
        d["out"] = torch.empty(wl.L, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=device)
        d["lse"] = torch.empty(wl.L, wl.Hq, dtype=torch.float32, device=device)
        layers.append(d)
        torch.cuda.synchronize()
    return layers


def kinds_of(pattern):
    return [c for c in pattern if c in "FS"]


def time_stack(step, args, stream, dev, barrier, max_over_ranks):
    """W warm-up steps; K steps timed untraced between two CUDA events on the launching
    stream (clocks sampled meanwhile; the max over ranks); then K more steps with an
    event after every launch, for the per-kernel split.  Returns
    (ms_per_step, clocks, launches in the traced K steps, trace)."""
    from sparse_attention_indexer_sum_b200 import binding as ic
    for _ in range(args.warmup):
        step()
    ic.ic_device_status(stream)
    barrier()
    clocks = ClockSampler("GPU-%s" % torch.cuda.get_device_properties(dev).uuid)
    clocks.start()
    time.sleep(0.5)
    clocks.mark()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    ic.ic_device_status(stream)
    cap = max(4096, 256 * args.steps)
    ic.ic_trace_begin(cap, stream=stream)
    for _ in range(args.steps):
        step()
    n_launch, trace = ic.ic_trace_end(cap)
    ic.ic_device_status(stream)
    barrier()
    return ms, clk, n_launch, trace


def stack_roofline(trace, steps, wl, fp8, peaks, fp8_sustained=None):
    """Per-kernel device time and algorithmic work of a traced pass, and the roofline
    object of the dominant kernel (the tensor-core indexer)."""
    agg = {}
    for name, kms, work in trace:
        a = agg.setdefault(name, [0, 0.0, 0.0])
        a[0] += 1
        a[1] += kms
        a[2] += work
    tot_ms = sum(a[1] for a in agg.values())
    dom = "indexer_tc_e4m3" if fp8 else "indexer_tc_bf16"
    d_n, d_ms, d_work = agg.get(dom, [0, 0.0, 0.0])
    bf16_peak = peaks["bf16_sustained"]
    if fp8 and fp8_sustained:
        peak = fp8_sustained
        peak_src = "e4m3 GEMM measured in this run (torch._scaled_mm 8192^3, sustained) %.1f " \
                   "TFLOP/s" % peak
    elif fp8:
        peak = 2.0 * bf16_peak
        peak_src = "%s bf16 sustained %.1f TFLOP/s x2 (e4m3 nominal ratio; no fp8 GEMM " \
                   "measurement)" % (peaks["source"], bf16_peak)
    else:
        peak = bf16_peak
        peak_src = "%s bf16 sustained %.1f TFLOP/s" % (peaks["source"], bf16_peak)
    achieved = d_work / (d_ms * 1e-3) / 1e12 if d_ms > 0 else 0.0
    stages = {}
    for name, (n, kms, work) in sorted(agg.items()):
        st = {"launches_per_step": n / steps, "ms_per_step": kms / steps,
              "share": kms / tot_ms if tot_ms else 0.0}
        if name.startswith("indexer_tc"):
            st.update(bound="tensor", achieved_tflops=work / (kms * 1e-3) / 1e12,
                      unit="TFLOP/s")
        else:
            st.update(bound="hbm", achieved_gbs=work / (kms * 1e-3) / 1e9,
                      frac_hbm=work / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"], unit="GB/s")
        stages[name] = st
    pairs_per_launch = d_work / d_n / (2.0 * wl.H * wl.D) if d_n else 0.0
    per_pair = INDEXER_E4M3_DRAM_BYTES_PER_PAIR if fp8 else INDEXER_BF16_DRAM_BYTES_PER_PAIR
    traffic = per_pair * pairs_per_launch if per_pair else None
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak if peak else None, "traffic": traffic,
                "traffic_source": None if not per_pair else
                "ncu dram__bytes_read.sum + dram__bytes_write.sum of the same kernel on 512 "
                "rows at position 100000 (%.2f B per causal pair), times the pairs of a "
                "launch" % per_pair,
                "peak_source": peak_src,
                "work_per_launch": d_work / d_n if d_n else None,
                "launches": d_n, "ms_per_launch": d_ms / d_n if d_n else None}
    return stages, roofline


def run_ours(args, rank, world, local_rank):
    from sparse_attention_indexer_sum_b200 import binding as ic
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    wl = synth.WORKLOADS[args.workload]
    assert not wl.decode and wl.attn == "mla", "bench workloads are MLA prefill stacks"
    pattern = wl.pattern
    allf = ",".join("F" * wl.layers)
    fp8 = args.indexer == "e4m3"
    shard = args.shard == "rows"
    t0 = time.time()
    # weak scaling: every rank its own sequence (seed = rank); rows sharding: every rank
    # the same sequence, running only its zig-zag share of the query rows
    layers = make_inputs(wl, dev, [kinds_of(pattern)] + ([kinds_of(allf)] if args.compare else []),
                         fp8, seed=0 if shard else rank)
    log("rank %d: inputs ready in %.1f s (%.1f GB allocated)" %
        (rank, time.time() - t0, torch.cuda.memory_allocated(dev) / 1e9))
    desc = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D,
                        idx_dtype=ic.IC_E4M3 if fp8 else ic.IC_BF16, heads=wl.Hq, dk=wl.Dk,
                        dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, dtype=torch.float32, device=dev)
    t_cache = torch.empty(wl.L, wl.k, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    if shard:
        from sparse_attention_indexer_sum_b200.sharding import zigzag_row_ranges
        row_names = ("q_idx", "q_scale", "w", "q", "out", "lse")
        pieces = []
        for r0, n in zigzag_row_ranges(wl.L, world, rank):
            lay = [{f: (v[r0:r0 + n] if f in row_names else v) for f, v in d.items()}
                   for d in layers]
            pieces.append((r0, n, lay, t_cache[r0:r0 + n]))

        def step(pat=pattern):
            for r0, n, lay, tc in pieces:
                ic.ic_layer_stack_rows(pat, desc, lay, r0, n, tc, ws, stream=stream)
    else:
        def step(pat=pattern):
            ic.ic_layer_stack(pat, desc, layers, t_cache, ws, stream=stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    fp8_peak = measure_fp8_peak(dev) if rank == 0 and world == 1 else None
    ms, clk, n_launch, trace = time_stack(step, args, stream, dev, barrier, max_over_ranks)
    fp8_sus = (fp8_peak or {}).get("fp8_tflops_sustained")
    stages, roofline = stack_roofline(trace, args.steps, wl, fp8, peaks, fp8_sus)
    achieved = roofline["achieved"]
    value = wl.L / (ms * 1e-3) if shard else job_throughput(wl.L, world, ms)
    log("rank %d: %.2f ms/step, %.0f tokens/s, indexer %.1f TFLOP/s" % (rank, ms, value, achieved))

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if shard else "weak",
        "vs_baseline": None, "dtype": "e4m3+bf16" if fp8 else "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "L": wl.L, "layers": wl.layers, "pattern": pattern,
                   "k": wl.k, "indexer": "H_I=64 d_I=128 %s (fp32 accumulate)" %
                   ("e4m3 per-row scales" if fp8 else "bf16"),
                   "attention": "absorbed MLA 16 heads x 576 -> 512, bf16",
                   "batch_per_gpu": 1,
                   "parallelism": ("one sequence, query rows in zig-zag shares per GPU" if shard
                                   else "independent sequence per GPU" if world > 1
                                   else "single GPU"),
                   "l2": "inputs larger than L2 (no flush needed)"},
        "gpu_launches": n_launch, "roofline": roofline, "stages": stages, "clocks": clk,
        "timing": "%d steps untraced between CUDA events (value); the per-kernel split and "
                  "the roofline come from a second pass of %d steps with an event after "
                  "every launch" % (args.steps, args.steps),
    }
    if fp8_peak is not None:
        res["fp8_peak_measured"] = fp8_peak

    if args.e4m3_line and not fp8 and not shard:
        # the same stack with the e4m3 indexer on the same inputs (quantised per row)
        lay8 = [dict(d) for d in layers]
        for l, c in enumerate(kinds_of(pattern)):
            if c == "F":
                lay8[l]["q_idx"], lay8[l]["q_scale"] = ic.ic_quant_e4m3_rows(layers[l]["q_idx"])
                lay8[l]["k_idx"], lay8[l]["k_scale"] = ic.ic_quant_e4m3_rows(layers[l]["k_idx"])
        desc8 = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq,
                             dk=wl.Dk, dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale)

        def step8():
            ic.ic_layer_stack(pattern, desc8, lay8, t_cache, ws, stream=stream)
        ms8, clk8, n8, trace8 = time_stack(step8, args, stream, dev, barrier, max_over_ranks)
        stages8, roof8 = stack_roofline(trace8, args.steps, wl, True, peaks, fp8_sus)
        res["prefill_e4m3"] = {
            "pattern": pattern, "indexer": "e4m3 per-row scales (q per token and head, k per "
            "token), fp32 accumulate; attention bf16", "ms_per_step": ms8,
            "value": job_throughput(wl.L, world, ms8), "unit": UNIT, "gpu_launches": n8,
            "roofline": roof8, "stages": stages8, "clocks": clk8,
            "speedup_over_bf16_indexer": ms / ms8}
        log("e4m3 indexer: %.2f ms/step, indexer %.1f TFLOP/s = %.2f of %s" % (
            ms8, roof8["achieved"], roof8["frac"] or 0.0, roof8["peak_source"]))
        del lay8
        torch.cuda.empty_cache()

    if args.compare:
        for _ in range(1):
            step(allf)
        barrier()
        ka = max(2, args.steps // 2)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(ka):
            step(allf)
        e1.record(stream)
        barrier()
        ms_f = max_over_ranks(e0.elapsed_time(e1) / ka)
        res["all_f"] = {"pattern": allf, "ms_per_step": ms_f,
                        "value": (1 if shard else world) * wl.L / (ms_f * 1e-3),
                        "speedup_fsss_over_all_f": ms_f / ms}

    if args.e2e and shard:
        res["e2e"] = {"value": None, "unit": UNIT,
                      "note": "not measured in the rows-sharded mode (run the default mode)"}
    elif args.e2e:
        res["e2e"] = run_e2e(wl, layers, pattern, desc, t_cache, ws, stream, dev, args, barrier,
                             max_over_ranks, world)
    if args.cpu_baseline and rank == 0 and world == 1:
        res["cpu_baseline"] = cpu_baseline(wl, layers, budget_s=args.cpu_budget)
    if world == 1 and (args.decode or args.stack32k):
        del layers, ws, t_cache
        torch.cuda.empty_cache()
        if args.decode:
            res["decode"] = run_decode(args, dev, peaks, barrier)
            torch.cuda.empty_cache()
        if args.stack32k:
            res["stack_32k"] = run_stack32k(args, dev, barrier)
            torch.cuda.empty_cache()
    return res


def _timed(fn, steps, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / steps


def run_decode(args, dev, peaks, barrier):
    """Config 5: one decode step of 64 sequences (one new token each at position
    199999) through ic_decode_step, F,S,S,S and all-F.  HBM-bound: the roofline is
    the algorithmic bytes of the step (fp8 key cache + scales read by the indexer,
    the scores written and read back by the top-k, the gathered latent rows, q and
    out of every layer) over the measured copy bandwidth."""
    from sparse_attention_indexer_sum_b200 import binding as ic
    wl = synth.WORKLOADS["decode_200k"]
    B, L, k = wl.batch, wl.L, wl.k
    layers = []
    for l in range(wl.layers):
        d = synth.indexer_inputs(wl, l, device=dev)
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        kb = d.pop("k_idx")
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(kb)
        del kb
        d.update(synth.attn_inputs(wl, l, device=dev))
        d["out"] = torch.empty(B, 1, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=dev)
        d["lse"] = torch.empty(B, 1, wl.Hq, dtype=torch.float32, device=dev)
        layers.append(d)
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    desc = ic.make_desc(L=L, k=k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq, dk=wl.Dk,
                        dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale, batch=B, decode=True)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, dtype=torch.float32, device=dev)
    t_cache = torch.empty(B, k, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    allf = ",".join("F" * wl.layers)
    steps = 50

    def step(pat):
        ic.ic_decode_step(pat, desc, layers, t_cache, ws, stream=stream)

    kk = min(k, L)
    idx_b = B * L * (wl.D + 4)                      # e4m3 key cache + per-token scales
    score_b = B * L * 4 * 2 + B * kk * 4            # scores out and back in, T out
    t_b = B * kk * 4                                # T out (fused: the scores stay on chip)
    attn_b = B * kk * wl.Dk * 2 + B * wl.Hq * (wl.Dk + wl.Dv) * 2 + B * kk * 4

    def bytes_of(pat, fused=False):
        f = sum(1 for c in pat if c == "F")
        return f * (idx_b + (t_b if fused else score_b)) + wl.layers * attn_b

    out = {"workload": wl.name, "batch": B, "context": L, "k": k, "pattern": wl.pattern,
           "indexer": "e4m3 key cache + per-token f32 scales",
           "kv_cache": "bf16 576-d latent", "l2": "inputs larger than L2 (no flush needed)",
           "algorithmic_bytes": "per F layer the e4m3 key cache and scales read, the scores "
                                "written and read back, T written; per layer the gathered "
                                "latent rows, q, out and T read"}
    for pat, key in ((wl.pattern, None), (allf, "all_f")):
        for _ in range(max(3, args.warmup)):
            step(pat)
        ic.ic_device_status(stream)
        barrier()
        # the step time without tracing: an event between launches costs a few
        # microseconds each and stops consecutive kernels from overlapping
        ms_eager = _timed(lambda: step(pat), steps, stream)
        ic.ic_device_status(stream)
        # the same step captured once in a CUDA graph and replayed, as a serving
        # loop runs it (one host launch per step)
        try:
            graph = ic.decode_step_graph(pat, desc, layers, t_cache, ws)
            run, how = graph.replay, "CUDA graph replay of the step"
        except Exception as e:  # capture refused on this machine: time eager calls instead
            graph = None
            run = lambda: step(pat)  # noqa: E731
            how = "eager calls (graph capture failed: %s)" % str(e).splitlines()[0][:160]
            log("decode:", how)
        for _ in range(3):
            run()
        ic.ic_device_status(stream)
        # long enough (~0.5 s) for the 200 ms clock samples to see it
        n_graph = max(steps, int(500.0 / max(ms_eager, 1e-3)))
        clocks = ClockSampler("GPU-%s" % torch.cuda.get_device_properties(dev).uuid)
        clocks.start()
        time.sleep(0.5)
        clocks.mark()
        ms = _timed(run, n_graph, stream)
        clk = clocks.stop()
        ic.ic_device_status(stream)
        del graph, run
        # then a traced pass of the same steps for the per-stage split (its
        # stage times add up to the traced step, slightly longer than `ms`)
        cap = 64 * steps
        ic.ic_trace_begin(cap, stream=stream)
        ms_traced = _timed(lambda: step(pat), steps, stream)
        n_launch, trace = ic.ic_trace_end(cap)
        ic.ic_device_status(stream)
        hb = bytes_of(pat)
        gbs = hb / (ms * 1e-3) / 1e9
        r = {"pattern": pat, "ms_per_step": ms, "value": B / (ms * 1e-3), "unit": "tokens/s",
             "hbm_bytes_per_step": hb, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
             "frac_hbm": gbs / peaks["hbm_gbs"], "gpu_launches_per_step": n_launch / steps,
             "timing": "%s, %d steps" % (how, n_graph),
             "clocks": clk, "ms_per_step_eager": ms_eager,
             "ms_per_step_traced": ms_traced}
        if key is None:
            agg = {}
            for name, kms, work in trace:
                a = agg.setdefault(name, [0, 0.0, 0.0])
                a[0] += 1
                a[1] += kms
                a[2] += work
            st = {}
            for name, (n, kms, work) in sorted(agg.items()):
                if name.startswith("indexer_topk"):
                    byt = idx_b * n                      # cache read; candidates stay on chip
                elif name.startswith("indexer"):
                    byt = (idx_b + B * L * 4) * n        # cache read + scores written
                elif name == "topk":
                    byt = (B * L * 4 + B * kk * 4) * n
                else:
                    byt = work
                g = byt / (kms * 1e-3) / 1e9
                st[name] = {"launches_per_step": n / steps, "ms_per_step": kms / steps,
                            "achieved_gbs": g, "frac_hbm": g / peaks["hbm_gbs"]}
            r["stages"] = st
            out.update(r)
        else:
            out[key] = r
    out["speedup_fsss_over_all_f"] = out["all_f"]["ms_per_step"] / out["ms_per_step"]
    # the same F,S,S,S step with the indexer and the top-k fused
    desc_u = ic.make_desc(L=L, k=k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq, dk=wl.Dk,
                          dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale, batch=B, decode=True,
                          flags=ic.IC_STACK_FUSED_TOPK)
    ws_u = torch.empty(ic.ic_stack_workspace_size(desc_u) // 4 + 1, dtype=torch.float32,
                       device=dev)
    step_u = lambda: ic.ic_decode_step(wl.pattern, desc_u, layers, t_cache, ws_u,  # noqa: E731
                                       stream=stream)
    for _ in range(3):
        step_u()
    ic.ic_device_status(stream)
    ms_u = _timed(step_u, steps, stream)
    ic.ic_device_status(stream)
    hb_f = bytes_of(wl.pattern, fused=True)
    out["fused_topk"] = {"ms_per_step_eager": ms_u, "value": B / (ms_u * 1e-3),
                         "hbm_bytes_per_step": hb_f,
                         "frac_hbm": hb_f / (ms_u * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "note": "IC_STACK_FUSED_TOPK: indexer and top-k fused, the scores never "
                                 "written; eager calls (compare with ms_per_step_eager)"}
    del ws_u
    # the same F,S,S,S step over fp8 latent caches (ic_pack_kv_e4m3 rows of 656 bytes)
    for d in layers:
        d["kv"] = ic.ic_pack_kv_e4m3(d["kv"])
        torch.cuda.empty_cache()
    desc8 = ic.make_desc(L=L, k=k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq, dk=wl.Dk,
                         dv=wl.Dv, attn_dtype=ic.IC_E4M3, scale=wl.scale, batch=B, decode=True,
                         ld_kv=ic.KV8_ROW_BYTES)
    ws8 = torch.empty(ic.ic_stack_workspace_size(desc8) // 4 + 1, dtype=torch.float32, device=dev)
    step8 = lambda: ic.ic_decode_step(wl.pattern, desc8, layers, t_cache, ws8,  # noqa: E731
                                      stream=stream)
    for _ in range(3):
        step8()
    ic.ic_device_status(stream)
    ms8 = _timed(step8, steps, stream)
    ic.ic_device_status(stream)
    ic.ic_trace_begin(64 * steps, stream=stream)
    _timed(step8, steps, stream)
    _, tr8 = ic.ic_trace_end(64 * steps)
    ic.ic_device_status(stream)
    attn8 = [ms for name, ms, _ in tr8 if name == "attn_mla_kv8"]
    attn8_b = B * kk * ic.KV8_ROW_BYTES + B * wl.Hq * (wl.Dk + wl.Dv) * 2 + B * kk * 4
    hb8 = sum(1 for c in wl.pattern if c == "F") * (idx_b + score_b) + wl.layers * attn8_b
    out["fp8_kv"] = {
        "pattern": wl.pattern, "kv_cache": "fp8 latent rows: 512 e4m3 (four 128-dim groups with "
        "fp32 scales) + 64 bf16 rope = 656 B", "ms_per_step_eager": ms8,
        "value": B / (ms8 * 1e-3), "unit": "tokens/s", "hbm_bytes_per_step": hb8,
        "frac_hbm": hb8 / (ms8 * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "attn_ms_per_launch": sum(attn8) / max(1, len(attn8)),
        "attn_frac_hbm": (attn8_b / (sum(attn8) / max(1, len(attn8)) * 1e-3) / 1e9 /
                          peaks["hbm_gbs"]) if attn8 else None,
        "speedup_over_bf16_kv_eager": out["ms_per_step_eager"] / ms8}
    del ws8
    log("decode fp8 kv: %.3f ms/step eager (bf16 cache %.3f ms eager)" % (
        ms8, out["ms_per_step_eager"]))
    log("decode: %.3f ms/step (%.0f tokens/s), %.0f GB/s = %.2f of HBM; all-F %.3f ms" % (
        out["ms_per_step"], out["value"], out["achieved_gbs"], out["frac_hbm"],
        out["all_f"]["ms_per_step"]))
    return out


def _overlap(Ta, Tb):
    """Mean over rows of |Ta & Tb| / |Ta| for ascending, -1 padded index rows."""
    big = torch.iinfo(torch.int32).max
    A = torch.where(Ta < 0, torch.full_like(Ta, big), Ta).contiguous()
    Bq = torch.where(Tb < 0, torch.full_like(Tb, big), Tb).contiguous()
    pos = torch.searchsorted(A, Bq).clamp_(max=A.shape[1] - 1)
    hit = (A.gather(1, pos) == Tb) & (Tb >= 0)
    n = (Ta >= 0).sum(1).clamp_(min=1)
    return hit.sum(1).double() / n.double()


def run_stack32k(args, dev, barrier):
    """Config 3: the 8-layer F,S,S,S,F,S,S,S stack at L=32768 against all-F, and the
    overlap of adjacent layers' index sets when every layer runs its own indexer."""
    from sparse_attention_indexer_sum_b200 import binding as ic
    wl = synth.WORKLOADS["stack_32k"]
    allf = ",".join("F" * wl.layers)
    layers = make_inputs(wl, dev, [kinds_of(allf)], False, seed=0)
    desc = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=ic.IC_BF16, heads=wl.Hq,
                        dk=wl.Dk, dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, dtype=torch.float32, device=dev)
    t_cache = torch.empty(wl.L, wl.k, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = 5
    res = {"workload": wl.name, "L": wl.L, "layers": wl.layers, "k": wl.k,
           "pattern": wl.pattern}
    for pat, key in ((wl.pattern, "ms_per_step"), (allf, "all_f_ms_per_step")):
        for _ in range(max(3, args.warmup)):
            ic.ic_layer_stack(pat, desc, layers, t_cache, ws, stream=stream)
        barrier()
        res[key] = _timed(lambda: ic.ic_layer_stack(pat, desc, layers, t_cache, ws,
                                                    stream=stream), steps, stream)
    res["value"] = wl.L / (res["ms_per_step"] * 1e-3)
    res["all_f_value"] = wl.L / (res["all_f_ms_per_step"] * 1e-3)
    res["speedup_fs_over_all_f"] = res["all_f_ms_per_step"] / res["ms_per_step"]
    # every layer F, one at a time, keeping each layer's T
    prev, ov = None, []
    rows_ge_k = torch.arange(wl.L, device=dev) >= wl.k - 1
    for l in range(wl.layers):
        ic.ic_layer_stack("F", desc, [layers[l]], t_cache, ws, stream=stream)
        cur = t_cache.clone()
        if prev is not None:
            o = _overlap(prev, cur)
            ov.append((float(o.mean()), float(o[rows_ge_k].mean())))
        prev = cur
    ic.ic_device_status(stream)
    res["overlap_adjacent_all_f"] = {
        "mean_all_rows": sum(a for a, _ in ov) / len(ov),
        "mean_rows_with_more_than_k_candidates": sum(b for _, b in ov) / len(ov),
        "per_pair": [round(b, 4) for _, b in ov],
        "definition": "|T_l & T_(l+1)| / |T_l| averaged over query rows, every layer F"}
    log("stack_32k: %.2f ms (F/S) vs %.2f ms (all-F), speed-up %.2fx, adjacent overlap %.3f" % (
        res["ms_per_step"], res["all_f_ms_per_step"], res["speedup_fs_over_all_f"],
        res["overlap_adjacent_all_f"]["mean_rows_with_more_than_k_candidates"]))
    return res


def run_e2e(wl, layers, pattern, desc, t_cache, ws, stream, dev, args, barrier, max_over_ranks,
            world):
    """The metric through the C ABI with HOST buffers: every step copies its inputs from
    pinned host memory and reads its result (last layer's output and the index set) back.

    Steps are pipelined over three streams, as a serving loop would run them: while
    step s computes, step s+1's inputs stream in (host -> device) and step s-1's
    result streams out (device -> host). Inputs and results are double-buffered on
    the device. The timed region opens before the first input copy and closes after
    the last result has reached the host, so every byte of every step is inside it."""
    from sparse_attention_indexer_sum_b200 import binding as ic
    kinds = kinds_of(pattern)
    names_f = ["q_idx", "q_scale", "k_idx", "k_scale", "w", "q", "kv"]
    try:
        host_in = []
        for l, d in enumerate(layers):
            hs = {}
            for n in names_f:
                if n in d and (kinds[l] == "F" or n in ("q", "kv")):
                    h = torch.empty(d[n].shape, dtype=d[n].dtype, pin_memory=True)
                    h.copy_(d[n])
                    hs[n] = h
            host_in.append(hs)
        out_h = torch.empty(layers[-1]["out"].shape, dtype=torch.bfloat16, pin_memory=True)
        t_h = torch.empty(t_cache.shape, dtype=torch.int32, pin_memory=True)
    except RuntimeError as e:
        return {"value": None, "unit": UNIT, "error": "pinned host buffers: %s" % e}
    h2d = sum(t.numel() * t.element_size() for hs in host_in for t in hs.values())
    d2h = out_h.numel() * out_h.element_size() + t_h.numel() * t_h.element_size()

    # device buffer set 1: fresh tensors for everything copied in or read back
    sets = [layers, []]
    for l, d in enumerate(layers):
        e = dict(d)
        for n in host_in[l]:
            e[n] = torch.empty_like(d[n])
        if l == len(layers) - 1:
            e["out"] = torch.empty_like(d["out"])
        sets[1].append(e)
    t_caches = [t_cache, torch.empty_like(t_cache)]
    copy_s, back_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free, done, back_done = ([ev(), ev()] for _ in range(4))
    for b in range(2):  # every buffer starts free
        in_free[b].record(stream)
        back_done[b].record(back_s)

    def copy_in(b):
        copy_s.wait_event(in_free[b])
        with torch.cuda.stream(copy_s):
            for d, hs in zip(sets[b], host_in):
                for n, h in hs.items():
                    d[n].copy_(h, non_blocking=True)
        in_ready[b].record(copy_s)

    def compute(b):
        stream.wait_event(in_ready[b])
        stream.wait_event(back_done[b])  # the last read-back of this set's result is done
        ic.ic_layer_stack(pattern, desc, sets[b], t_caches[b], ws, stream=stream)
        in_free[b].record(stream)
        done[b].record(stream)

    def copy_back(b):
        back_s.wait_event(done[b])
        with torch.cuda.stream(back_s):
            out_h.copy_(sets[b][-1]["out"], non_blocking=True)
            t_h.copy_(t_caches[b], non_blocking=True)
        back_done[b].record(back_s)

    def run(nsteps, t0=None):
        if t0 is not None:
            copy_s.wait_event(t0)
        copy_in(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                copy_in((i + 1) % 2)  # next step's inputs, alongside this step's compute
            compute(i % 2)
            copy_back(i % 2)
        stream.wait_stream(back_s)
        stream.wait_stream(copy_s)

    run(2)  # warm-up
    barrier()
    ke = max(2, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(ke, t0=e0)
    e1.record(stream)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / ke)
    return {"value": world * wl.L / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ke,
            "pipelined": "inputs of step s+1 copied in and result of step s copied out "
                         "while step s+1 / s computes; first copy-in and last copy-out "
                         "inside the timed region"}


# ------------------------------------------------------------------------------ CPU oracle
class OracleSample:
    """Host (fp64) copies of what the oracle needs for sampled query rows of the stack."""

    def __init__(self, wl, layers_dev):
        self.wl = wl
        self.kinds = kinds_of(wl.pattern)
        self.layers = layers_dev
        self.k_idx = {}
        self.kv = []
        for l, d in enumerate(layers_dev):
            if self.kinds[l] == "F":
                self.k_idx[l] = d["k_idx"].double().cpu().numpy()
            self.kv.append(d["kv"].double().cpu().numpy())

    def run(self, rows, nthreads):
        """Runs the oracle stack on the query rows `rows`; returns per-stage seconds."""
        import oracle
        wl = self.wl
        rows_t = torch.from_numpy(rows.astype(np.int64)).to(self.layers[0]["q"].device)
        t_idx = t_topk = t_attn = 0.0
        T = None
        for l, d in enumerate(self.layers):
            if self.kinds[l] == "F":
                q = d["q_idx"][rows_t].double().cpu().numpy()
                w = d["w"][rows_t].double().cpu().numpy()
                t0 = time.perf_counter()
                I = oracle.indexer_scores_at(q, self.k_idx[l], w, rows, nthreads=nthreads)
                t_idx += time.perf_counter() - t0
                I32 = I.astype(np.float32)
                t0 = time.perf_counter()
                T = oracle.topk(I32, wl.k, valid=(rows + 1).astype(np.int32), nthreads=nthreads)
                t_topk += time.perf_counter() - t0
            qa = d["q"][rows_t].double().cpu().numpy()
            t0 = time.perf_counter()
            oracle.sparse_attn(qa, self.kv[l], T, wl.scale, dv=wl.Dv, nthreads=nthreads)
            t_attn += time.perf_counter() - t0
        return t_idx, t_topk, t_attn


def extrapolate(wl, rows, t_idx, t_topk, t_attn):
    """Full-workload seconds from the sample: indexer and top-k scale with the causal pair
    count (sum of t+1 over rows), attention with the row count."""
    pairs_sample = float((rows.astype(np.float64) + 1).sum())
    pairs_total = wl.L * (wl.L + 1) / 2.0
    return (t_idx + t_topk) * pairs_total / pairs_sample + t_attn * wl.L / len(rows)


def cpu_baseline(wl, layers_dev, budget_s=15.0):
    import oracle
    oracle.build()
    nthreads = oracle.default_threads()
    samp = OracleSample(wl, layers_dev)
    g = np.random.default_rng(1234)
    # calibrate on one row per thread, then size the sample to the time budget
    rows = np.sort(g.choice(wl.L, size=nthreads, replace=False)).astype(np.int64)
    t = samp.run(rows, nthreads)
    per_round = max(sum(t), 1e-3)
    rounds = int(max(1, min(64, (budget_s - per_round) / per_round)))
    more = np.sort(g.choice(wl.L, size=rounds * nthreads, replace=False)).astype(np.int64)
    t2 = samp.run(more, nthreads)
    rows_all = np.concatenate([rows, more])
    t_all = [a + b for a, b in zip(t, t2)]
    total = extrapolate(wl, rows_all, *t_all)
    return {"value": wl.L / total, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": "%d random query rows of the %d-token %s stack (fp64 indexer, top-k and "
                      "attention on all %d layers), %.1f s measured on %d host threads, "
                      "extrapolated to the full step by causal pair count (indexer, top-k) "
                      "and row count (attention)" % (len(rows_all), wl.L, wl.pattern, wl.layers,
                                                     sum(t_all), nthreads),
            "extrapolated_s_per_step": total}


def run_reference(args):
    """The CPU oracle as the reference arm: each step is a bounded sample of the workload."""
    import oracle
    oracle.build()
    wl = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    # inputs come from the same generators (drawn on the GPU when there is one)
    layers = []
    kinds = kinds_of(wl.pattern)
    for l in range(wl.layers):
        d = {}
        if kinds[l] == "F":
            d.update(synth.indexer_inputs(wl, l, device=dev))
        d.update(synth.attn_inputs(wl, l, device=dev))
        layers.append(d)
    nthreads = oracle.default_threads()
    samp = OracleSample(wl, layers)
    g = np.random.default_rng(99)
    n = nthreads
    totals = []
    for s in range(args.warmup + args.steps):
        rows = np.sort(g.choice(wl.L, size=n, replace=False)).astype(np.int64)
        t_idx, t_topk, t_attn = samp.run(rows, nthreads)
        if s >= args.warmup:
            totals.append(extrapolate(wl, rows, t_idx, t_topk, t_attn))
    sec = statistics.mean(totals)
    value = wl.L / sec
    sample = ("%d random query rows per step of the %d-token F,S,S,S stack, fp64 oracle on %d "
              "host threads, extrapolated by causal pair count" % (n, wl.L, nthreads))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "L": wl.L, "layers": wl.layers,
                       "pattern": wl.pattern, "k": wl.k},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(nthreads, n),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_200k",
                    choices=["prefill_200k", "stack_32k", "prefill_8k"])
    ap.add_argument("--indexer", default="bf16", choices=["bf16", "e4m3"])
    ap.add_argument("--no-compare", dest="compare", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--shard", default="sequences", choices=["sequences", "rows"],
                    help="sequences: one independent 200K prefill per GPU (weak scaling, the "
                         "default); rows: one prefill, its query rows shared out over the GPUs "
                         "in zig-zag chunks (strong scaling)")
    ap.add_argument("--no-decode", dest="decode", action="store_false",
                    help="skip the decode (64 x 1 token at 200K context) measurement")
    ap.add_argument("--no-e4m3-line", dest="e4m3_line", action="store_false",
                    help="skip the same stack with the e4m3 indexer (key prefill_e4m3)")
    ap.add_argument("--no-stack32k", dest="stack32k", action="store_false",
                    help="skip the 8-layer L=32768 stack and its layer-overlap report")
    args = ap.parse_args()
    if args.warmup < 3:
        log("note: fewer than 3 warm-up steps requested")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
