#!/usr/bin/env python3
"""MoE-layer throughput of one DWDP rank's MoE block (tokens/s) and the
roofline fraction of its grouped expert GEMM.

A step is one pass of the whole block over one batch: router + top-k,
permutation, grouped SwiGLU FFN over the split (local + remote) expert
pools, combine - and, for the multi-layer pipelined workloads, the
copy-engine prefetch of later layers' remote experts into the alternate
buffers.  Default workload: the DeepSeek-R1-shaped decode step (128 tokens,
H=7168, I=2048, 256 routed experts + 1 shared, top-8 of 8 groups / top-4,
bf16 weights, 64 local / 192 remote experts).

  python bench.py [--gpus N --steps K --warmup W] [--config 1..5] [--impl reference]

N > 1 (torchrun): N independent data-parallel replicas, one per GPU (the
block has no collective; each rank runs its own tokens): weak scaling,
value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at DeepSeek-R1 shape; % of HBM/tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "grouped_ffn_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", type=int, default=2)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-merge-ablation", action="store_true")
    p.add_argument("--prefetch-split", type=int, default=0, choices=(0, 1),
                   help="issue each layer's fetch in two halves in the windows between grouped GEMMs")
    p.add_argument("--act-dtype", choices=["bf16", "e4m3"], default="bf16",
                   help="activations the grouped GEMMs read (e4m3: opt-in fp8 tensor-core path, "
                        "e4m3-weight workloads only)")
    p.add_argument("--workloads", default="3,4,5",
                   help="further workloads measured in the same run (1 GPU only; '' for none)")
    p.add_argument("--workload-steps", type=int, default=5)
    p.add_argument("--gate-slots", type=int, default=8,
                   help="pipelined workloads: per-chunk readiness flags every N remote slots, "
                        "the grouped GEMM starting before the fetch ends (0: the compute stream "
                        "waits for the whole fetch)")
    p.add_argument("--pace-steps", type=int, default=0,
                   help="pipelined workloads with readiness flags: pace each fetch by the "
                        "previous grouped GEMM call's progress in N steps (0: unpaced)")
    p.add_argument("--pace-lead", type=int, default=2,
                   help="paced fetch: chunks issued before the first progress report")
    p.add_argument("--window-inter", type=int, default=12288,
                   help="intermediate size of the dense block that stands in for the attention "
                        "block in the prefetch-window measurement (0: skip it)")
    p.add_argument("--no-schedules", action="store_true",
                   help="pipelined workloads: measure only the configured prefetch schedule")
    p.add_argument("--measure-peaks", action="store_true",
                   help="measure the fp8 dense GEMM peak and the read-only HBM peak, print JSON")
    return p.parse_args(argv)


# ----------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


EXTRA_PEAKS = os.path.join(ROOT, "profiles", "peaks_fp8_hbm_read.json")
SUSTAINED_AFTER_S = 2.0   # timed regions at least this long are compared with the sustained peak


def load_extra_peaks():
    """fp8 dense TFLOP/s and read-only HBM GB/s measured by `bench.py
    --measure-peaks` on this machine's B200s (committed under profiles/)."""
    try:
        with open(EXTRA_PEAKS) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def tensor_peak(peaks, mma_kind: str, timed_s: float):
    """(peak TFLOP/s, its source) for the MMA kind the kernel issues: the burst
    figure for a timed region shorter than SUSTAINED_AFTER_S, else the
    sustained one.  kind::f16 takes the bf16 figures; kind::f8f6f4 the
    measured fp8 figure, else bf16 x 2 (the nominal ratio)."""
    sustained = timed_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks
    bf16 = float(peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"])
    which = "sustained" if sustained else "burst"
    if mma_kind == "f16":
        return bf16, f"bf16 dense, {which}"
    extra = load_extra_peaks()
    if "fp8_tflops" in extra:
        fp8 = float(extra["fp8_tflops"])
        if sustained:   # scale the measured burst figure like the bf16 one
            fp8 *= float(peaks["bf16_tflops_sustained"]) / float(peaks["bf16_tflops"])
        return fp8, f"fp8 dense measured (torch._scaled_mm 8192^3), {which}"
    return 2.0 * bf16, f"fp8 dense taken as 2 x bf16 {which} (nominal ratio)"


_COMMENTS = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def kernel_source_hash(files) -> str:
    """Hash of the kernel sources with comments and blank space taken out: a
    capture stays valid across an edit of the comments, not of the code."""
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "split_weight_b200", "csrc", name), encoding="utf-8") as f:
            code = " ".join(_COMMENTS.sub(" ", f.read()).split())
        h.update(code.encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, alg_bytes_per_layer: float):
    """DRAM bytes per layer of the grouped FFN (gate/up + down launches) from
    the committed ncu capture, if it was taken on the current kernel source.
    A full-size workload too large to capture is scaled from its reduced
    case by the ratio of algorithmic bytes (same tokens per expert)."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e:
        return None
    scale = 1.0
    if "scaled_from" in e:
        e = d.get(e["scaled_from"])
        if not e:
            return None
        scale = alg_bytes_per_layer / e["algorithmic_bytes_per_call"]
    if e.get("kernel_source_hash") != kernel_source_hash(e["kernel_files"]):
        return None
    return e["dram_bytes_per_call"] * scale


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while it runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def workload_desc(cfg) -> str:
    d = (f"{cfg.name}: T={cfg.T} tokens x {cfg.layers} layer(s), H={cfg.H}, I={cfg.I}, "
         f"E={cfg.E} routed" + (" + 1 shared" if cfg.has_shared else "") + f", top-{cfg.k} {cfg.score}")
    if cfg.score == "sigmoid":
        d += f" ({cfg.n_group} groups / top-{cfg.topk_group})"
    d += f", {cfg.w_dtype} weights, {cfg.local_count} local / {cfg.E - cfg.local_count} remote experts"
    return d


def roofline_figures(cfg, counts_per_layer, peaks):
    """Algorithmic FLOPs and bytes of the grouped FFN per step."""
    wbytes = 2 if cfg.w_dtype == "bf16" else 1
    act = 2
    flops = 0.0
    nbytes = 0.0
    for counts in counts_per_layer:
        touched = int((np.asarray(counts) > 0).sum()) + (1 if cfg.has_shared else 0)
        rows = cfg.A + (cfg.T if cfg.has_shared else 0)
        flops += rows * 6.0 * cfg.H * cfg.I
        nbytes += touched * 3.0 * cfg.H * cfg.I * wbytes + 2.0 * cfg.T * cfg.H * act
    return flops, nbytes


# ----------------------------------------------------------------------- our arm
def build_workload(cfg, args, dev, act_dtype):
    """Every layer of the workload resident in HBM; for multi-layer workloads
    the remote experts only in their peer stores, fetched by the pipeline."""
    import torch
    from moe_inputs import device as mdev
    dls = [mdev.build_layer(cfg, layer=l, device=dev, act_dtype=act_dtype)
           for l in range(cfg.layers)]
    pipe = None
    if cfg.layers > 1:
        from split_weight_b200 import PrefetchPipeline
        stores = [mdev.peer_store(cfg, l, dls[l].layer.weights, dev) for l in range(cfg.layers)]
        rbytes = dls[0].layer.weights.n_remote * dls[0].layer.weights.stride
        pipe = PrefetchPipeline([d.layer for d in dls], stores, rbytes, dev,
                                split=bool(args.prefetch_split), gate_slots=args.gate_slots,
                                pace_steps=args.pace_steps if args.gate_slots > 0 else 0,
                                pace_lead=args.pace_lead)
        for d in dls:  # the layers' own remote pools are not needed: the buffers replace them
            d.layer.weights.remote = torch.empty(1, dtype=torch.uint8, device=dev)
        torch.cuda.empty_cache()
        pipe.prime()
    torch.cuda.synchronize()
    return dls, pipe


def make_step(cfg, dls, pipe, stream):
    xs = [d.x for d in dls]
    h = stream.cuda_stream

    def step(timed_ffn=None, prefetch=True, inputs=None):
        inputs = xs if inputs is None else inputs
        if pipe is None:
            ml = dls[0].layer
            ml.route(inputs[0], h)
            ml.permute(inputs[0], h)
            if timed_ffn is not None:
                timed_ffn[0][0].record(stream)
            ml.grouped_ffn(h, x=inputs[0])
            if timed_ffn is not None:
                timed_ffn[0][1].record(stream)
            ml.combine(h)
            return
        for l in range(cfg.layers):
            pipe.run_layer(l, inputs[l], stream, prefetch=prefetch,
                           ffn_events=None if timed_ffn is None else timed_ffn[l])
    return step


def roofline_object(cfg, counts, act_dtype, ffn_ms, timed_s, peaks, peak_src):
    """The `roofline` object of the grouped FFN call (its two launches)."""
    flops, nbytes = roofline_figures(cfg, counts, peaks)
    hbm = float(peaks["hbm_gbs"])
    mma_kind = "f8f6f4" if act_dtype == "e4m3" else "f16"
    tc_peak, tc_src = tensor_peak(peaks, mma_kind, timed_s)
    t_hbm = nbytes / (hbm * 1e9)
    t_flop = flops / (tc_peak * 1e12)
    ffn_s = ffn_ms / 1e3
    if t_hbm >= t_flop:
        achieved = nbytes / ffn_s / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4)}
        read_peak = load_extra_peaks().get("hbm_read_gbs")
        if read_peak:
            roof["frac_of_read_peak"] = round(achieved / float(read_peak), 4)
            roof["read_peak_gbs"] = float(read_peak)
    else:
        achieved = flops / ffn_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(tc_peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4)}
        if mma_kind == "f16" and "bf16_tflops_sustained" in peaks:
            roof["frac_of_sustained"] = round(achieved / float(peaks["bf16_tflops_sustained"]), 4)
            roof["frac_of_burst"] = round(achieved / float(peaks["bf16_tflops"]), 4)
    traffic = profiled_traffic(cfg.name + ("" if act_dtype == "bf16" else "_" + act_dtype),
                               nbytes / cfg.layers)
    roof.update({
        "traffic": (round(traffic * cfg.layers) if traffic is not None else None),
        "kernel": "moe_grouped_ffn (gate/up + down launches)",
        "mma_kind": mma_kind,
        "peak_source": (f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})"
                        + (f"; tensor: {tc_src}" if roof["bound"] == "tensor" else "")),
        "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
        "kernel_ms_per_step": round(ffn_ms, 4),
        "roof_ms_per_step": round(max(t_hbm, t_flop) * 1e3, 4),
        "frac_of_roof": round(max(t_hbm, t_flop) / ffn_s, 4),
    })
    return roof


def time_steps(step, cfg, steps, stream, barrier, local_rank, sample_clocks=True):
    """Times `steps` steps on the compute stream; the grouped FFN of every
    layer is bracketed by its own events.  Returns (elapsed ms, FFN ms per
    step, launches, clocks summary)."""
    import torch
    from split_weight_b200 import _lib as L

    def events(n):
        return [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(cfg.layers)] for _ in range(n)]
    ffn_ev = events(steps)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank) if sample_clocks else None
    if clk is not None:
        clk.__enter__()
    try:
        launches0 = L.moe_kernel_launches()
        ev0.record(stream)
        for i in range(steps):
            step(ffn_ev[i])
        ev1.record(stream)
        launches = L.moe_kernel_launches() - launches0
        torch.cuda.synchronize()
    finally:
        if clk is not None:
            clk.__exit__(None, None, None)
    elapsed_ms = ev0.elapsed_time(ev1)
    ffn_ms = sum(a.elapsed_time(b) for st in ffn_ev for a, b in st) / steps
    return elapsed_ms, ffn_ms, launches, (clk.summary() if clk is not None else None)


def prefetch_overlap(cfg, pipe, step, stream, piped_ms, steps):
    """Exposed copy time per layer: the same steps without copies, and the
    copy of one layer's remote experts alone.  Also returns, under
    "_ffn_ms_no_copy", the grouped FFN's time per step in the steps without
    copies (the kernels alone, for the roofline)."""
    import torch
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(3, min(steps, 10))
    ffn_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(cfg.layers)] for _ in range(reps)]
    e0.record(stream)
    for i in range(reps):
        step(ffn_ev[i], prefetch=False)
    e1.record(stream)
    torch.cuda.synchronize()
    nocopy_ms = e0.elapsed_time(e1) / reps
    ffn_nocopy = sum(a.elapsed_time(b) for st in ffn_ev for a, b in st) / reps
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the baseline every schedule is measured against: the whole remote buffer of
    # one layer as one copy (the schedule's own chunking and flags excluded)
    from split_weight_b200 import _lib as L
    c0.record(pipe.copy_stream)
    L.check(L.moe_prefetch_layer(pipe.peer_stores[0].data_ptr(), pipe.bufs[0].data_ptr(),
                                 pipe.remote_bytes, 0, pipe.copy_stream.cuda_stream, None, None))
    c1.record(pipe.copy_stream)
    torch.cuda.synchronize()
    copy_ms = c0.elapsed_time(c1)
    # refill both buffers for the executions that come next (the execution
    # count keeps growing: readiness epochs must never repeat)
    pipe.prime()
    torch.cuda.synchronize()
    exposed = max(0.0, (piped_ms - nocopy_ms) / cfg.layers)
    return {
        "schedule": (("selective: predicted remote slots after the grouped GEMM, missed ones "
                      "before the next" if pipe.select else
                      f"paced by the grouped GEMM's progress ({pipe.pace_steps} steps, "
                      f"{pipe.pace_lead} chunks ahead)" if pipe.pace_steps else
                      "halves between grouped GEMMs" if pipe.split else "whole, after the grouped GEMM")
                     + (f"; readiness flags every {pipe.gate_slots} slots" if pipe.gate_slots else
                        "; compute waits for the whole fetch")
                     + ("; dense window block" if pipe.window_block is not None else "")),
        "remote_bytes_per_layer": pipe.remote_bytes,
        "copy_alone_ms_per_layer": round(copy_ms, 4),
        "step_ms_pipelined": round(piped_ms, 4),
        "step_ms_no_copy": round(nocopy_ms, 4),
        "exposed_copy_ms_per_layer": round(exposed, 4),
        "hidden_fraction": round(1.0 - exposed / copy_ms, 4) if copy_ms > 0 else None,
        "_ffn_ms_no_copy": ffn_nocopy,
    }


def prefetch_schedules(cfg, pipe, step, stream, args, dev):
    """Exposed copy time per layer under each prefetch schedule, measured on
    the same layers and buffers:
      events_halves   compute waits for each whole fetch, issued in halves
      flags_whole     the grouped GEMM starts at once and waits per chunk of
                      8 remote slots on the device (readiness flags); the
                      fetch is issued whole as soon as its buffer is free
      flags_halves    the same with the fetch in halves
      flags_paced     flags, the fetch of the next execution issued before
                      each grouped GEMM call and paced by its progress
                      reports (24 steps, 2 chunks ahead)
      selective       per-slot flags; only the remote slots predicted by a
                      look-ahead routing (the next layer's router on this
                      layer's input), then the ones it missed
      window_*        the same schedules with a dense compute block
                      (R1 attention FLOPs) before every MoE block, the
                      explainer's two-block window; its no-copy baseline runs
                      the block too
    Restores the pipeline's own schedule afterwards."""
    import torch
    from split_weight_b200 import DenseBlock
    from split_weight_b200 import _lib as L
    saved = (pipe.split, pipe.gate_slots, pipe.window_block, pipe.pace_steps, pipe.pace_lead,
             pipe.select)
    steps = max(3, args.workload_steps)

    def run(split, gate_slots, window, pace_steps=0, pace_lead=2, select=False):
        """One schedule; a kernel wait that ran out (or another device
        check) is reported in its entry, not raised."""
        torch.cuda.synchronize()
        pipe.configure(split=split, gate_slots=gate_slots, window_block=window,
                       pace_steps=pace_steps, pace_lead=pace_lead, select=select)
        pipe.select_stats = []
        pipe.prime()
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        st = L.moe_check_device()
        if st != L.MOE_OK:
            return {"error": f"{L.status_string(st)} in warm-up: {L.moe_last_error()}"}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        st = L.moe_check_device()
        if st != L.MOE_OK:
            return {"error": f"{L.status_string(st)}: {L.moe_last_error()}"}
        stats = list(pipe.select_stats)
        out = prefetch_overlap(cfg, pipe, step, stream, e0.elapsed_time(e1) / steps, steps)
        out.pop("_ffn_ms_no_copy", None)
        if select and stats:   # remote slots fetched per execution, after the first pass
            later = stats[cfg.layers:] or stats
            n_slots = pipe.remote_bytes // pipe.stride
            out["selective"] = {
                "remote_slots": n_slots,
                "touched_per_layer": round(float(np.mean([x["touched"] for x in later])), 2),
                "predicted_per_layer": round(float(np.mean([x.get("predicted_next", 0)
                                                            for x in later])), 2),
                "missed_per_layer": round(float(np.mean([x["missed"] for x in later])), 2),
            }
            f = out["selective"]
            f["fetched_fraction"] = round((f["predicted_per_layer"] + f["missed_per_layer"])
                                          / n_slots, 4)
        st = L.moe_check_device()
        if st != L.MOE_OK:
            out["error"] = f"{L.status_string(st)} in the no-copy or copy-alone runs"
        return out

    out = {"events_halves": run(True, 0, None), "flags_whole": run(False, 8, None),
           "flags_halves": run(True, 8, None), "flags_paced": run(False, 8, None, 24, 2),
           "selective": run(False, 1, None, select=True)}
    if args.window_inter > 0:
        block = DenseBlock(cfg.T, cfg.H, args.window_inter, dev)
        out["window_block"] = {"inter": args.window_inter,
                               "flop_per_token": 6.0 * cfg.H * args.window_inter}
        out["window_events_halves"] = run(True, 0, block)
        out["window_flags_whole"] = run(False, 8, block)
        out["window_flags_paced"] = run(False, 8, block, 24, 2)
        del block
    torch.cuda.synchronize()
    pipe.configure(split=saved[0], gate_slots=saved[1], window_block=saved[2],
                   pace_steps=saved[3], pace_lead=saved[4], select=saved[5])
    pipe.prime()
    torch.cuda.synchronize()
    return out


def pipelined_roofline(out, cfg, counts, act, ffn_ms_piped, timed_s, peaks, peak_src):
    """For a pipelined workload the grouped FFN's time in the pipelined steps
    includes waiting for chunks of a fetch in flight (readiness flags) and
    the copy's contention; the roofline takes the kernels alone, from the
    steps without copies, and keeps the pipelined figure beside it."""
    pre = out["prefetch"]
    ffn_alone = pre.pop("_ffn_ms_no_copy")
    roof = roofline_object(cfg, counts, act, ffn_alone, timed_s, peaks, peak_src)
    piped = roofline_object(cfg, counts, act, ffn_ms_piped, timed_s, peaks, peak_src)
    roof["kernel_timing"] = "grouped FFN in the steps without copies (the kernels alone)"
    roof["frac_with_fetch_in_flight"] = piped["frac"]
    roof["kernel_ms_per_step_with_fetch"] = piped["kernel_ms_per_step"]
    out["roofline"] = roof


def measure_extra_workload(cfg_id, args, dev, stream, peaks, peak_src):
    """Tokens/s, roofline and (multi-layer) prefetch overlap of another
    workload, measured in the same run with a few steps."""
    import gc
    import torch
    from moe_inputs import config
    from split_weight_b200 import _lib as L
    cfg = config(cfg_id)
    act = args.act_dtype if cfg.w_dtype == "e4m3" else "bf16"
    dls, pipe = build_workload(cfg, args, dev, act)
    step = make_step(cfg, dls, pipe, stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    L.check(L.moe_check_device())
    counts = [np.diff(d.layer.offsets.cpu().numpy()) for d in dls]
    elapsed_ms, ffn_ms, launches, clocks = time_steps(step, cfg, args.workload_steps, stream,
                                                      lambda: None, 0)
    L.check(L.moe_check_device())
    out = {"workload": workload_desc(cfg), "act_dtype": act, "steps": args.workload_steps,
           "ms_per_step": round(elapsed_ms / args.workload_steps, 4),
           "value": round(cfg.T * cfg.layers * args.workload_steps / (elapsed_ms / 1e3), 3),
           "unit": "tokens/s", "gpu_launches": int(launches),
           "roofline": roofline_object(cfg, counts, act, ffn_ms, elapsed_ms / 1e3, peaks, peak_src),
           "clocks": clocks}
    if pipe is not None:
        out["prefetch"] = prefetch_overlap(cfg, pipe, step, stream,
                                           elapsed_ms / args.workload_steps, args.workload_steps)
        pipelined_roofline(out, cfg, counts, act, ffn_ms, elapsed_ms / 1e3, peaks, peak_src)
        if not args.no_schedules:
            out["prefetch"]["schedules"] = prefetch_schedules(cfg, pipe, step, stream, args, dev)
    del dls, pipe, step
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    from moe_inputs import config

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = config(args.config)
    act_dtype = args.act_dtype if cfg.w_dtype == "e4m3" else "bf16"
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # ---- workload (resident in HBM before timing)
    dls, pipe = build_workload(cfg, args, dev, act_dtype)
    xs = [d.x for d in dls]
    step = make_step(cfg, dls, pipe, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    from split_weight_b200 import _lib as L
    L.check(L.moe_check_device())
    counts = [np.diff(d.layer.offsets.cpu().numpy()) for d in dls]

    # ---- device-timed region (FFN launches bracketed by their own events)
    elapsed_ms, ffn_ms, launches, clocks = time_steps(step, cfg, args.steps, stream, barrier,
                                                      local_rank)
    barrier()
    L.check(L.moe_check_device())

    # ---- pipelined workloads: exposed copy time per layer
    prefetch_info = None
    if pipe is not None:
        prefetch_info = prefetch_overlap(cfg, pipe, step, stream, elapsed_ms / args.steps,
                                         args.steps)
        ffn_alone_ms = prefetch_info.pop("_ffn_ms_no_copy")
        if world == 1 and not args.no_schedules:
            prefetch_info["schedules"] = prefetch_schedules(cfg, pipe, step, stream, args, dev)

    # ---- split-weight ablation: merge both pools into one buffer every step
    merge_info = None
    if pipe is None and not args.no_merge_ablation:
        merge_info = merge_ablation(cfg, dls[0], stream, elapsed_ms / args.steps,
                                    max(3, min(args.steps, 20)))

    # ---- end-to-end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and its outputs back; the
    # copies run on a second stream into alternate device buffers, so step
    # i+1's inputs and step i-1's outputs travel while step i computes.  All
    # copies are inside the timed region.
    e2e = None
    if not args.no_e2e:
        copy = torch.cuda.Stream(device=dev)
        x_host = [d.x.cpu().pin_memory() for d in dls]
        y_host = [torch.empty_like(d.layer.y[:cfg.T], device="cpu").pin_memory() for d in dls]
        x_dev = [[xs[l], torch.empty_like(xs[l])] for l in range(cfg.layers)]
        y_dev = [[d.layer.y, torch.empty_like(d.layer.y)] for d in dls]
        in_ready, x_free, y_ready, y_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))
        for e_ in x_free + y_free:  # so that the first waits are on recorded events
            e_.record(stream)

        def run_e2e(n):
            copy.wait_stream(stream)
            with torch.cuda.stream(copy):
                for l in range(cfg.layers):
                    x_dev[l][0].copy_(x_host[l], non_blocking=True)
                in_ready[0].record(copy)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    with torch.cuda.stream(copy):
                        copy.wait_event(x_free[1 - b])
                        for l in range(cfg.layers):
                            x_dev[l][1 - b].copy_(x_host[l], non_blocking=True)
                        in_ready[1 - b].record(copy)
                stream.wait_event(in_ready[b])
                stream.wait_event(y_free[b])
                for l, d in enumerate(dls):
                    d.layer.y = y_dev[l][b]
                step(inputs=[x_dev[l][b] for l in range(cfg.layers)])
                x_free[b].record(stream)
                y_ready[b].record(stream)
                with torch.cuda.stream(copy):
                    copy.wait_event(y_ready[b])
                    for l in range(cfg.layers):
                        y_host[l].copy_(y_dev[l][b][:cfg.T], non_blocking=True)
                    y_free[b].record(copy)
            stream.wait_stream(copy)

        run_e2e(2)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        run_e2e(args.steps)
        q1.record(stream)
        torch.cuda.synchronize()
        for l, d in enumerate(dls):
            d.layer.y = y_dev[l][0]
        e2e_ms = max_over_ranks(q0.elapsed_time(q1), world, dev)
        h2d = sum(t.numel() * t.element_size() for t in x_host)
        d2h = sum(t.numel() * t.element_size() for t in y_host)
        e2e = {"value": None, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "_ms": e2e_ms,
               "overlap": "inputs of step i+1 and outputs of step i-1 copied during step i"}
    barrier()

    max_ms = max_over_ranks(elapsed_ms, world, dev)
    tokens_per_step = cfg.T * cfg.layers
    total_tokens = sum_over_ranks(tokens_per_step * args.steps, world, dev)
    value = total_tokens / (max_ms / 1e3)
    if e2e is not None:
        e2e["value"] = round(total_tokens / (e2e.pop("_ms") / 1e3), 3)

    peaks, peak_src = load_peaks()
    roof = roofline_object(cfg, counts, act_dtype, ffn_ms, elapsed_ms / 1e3, peaks, peak_src)
    if prefetch_info is not None:
        holder = {"prefetch": dict(prefetch_info, _ffn_ms_no_copy=ffn_alone_ms)}
        pipelined_roofline(holder, cfg, counts, act_dtype, ffn_ms, elapsed_ms / 1e3, peaks, peak_src)
        roof = holder["roofline"]
    workload = cfg.name
    nbytes = roof["algorithmic_bytes"]
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.w_dtype, "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "tokens_per_rank_per_step": tokens_per_step,
                   "layers": cfg.layers, "parallelism": f"dp{world} replicas (no collective)",
                   "act_dtype": act_dtype,
                   "l2": "inputs larger than L2: %.1f GB of expert weights per step" % (nbytes / 1e9)},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks if rank == 0 else None,
    }
    if merge_info is not None:
        out["split_weight"] = merge_info
    if prefetch_info is not None:
        out["prefetch"] = prefetch_info

    # ---- further workloads in the same run (one GPU only)
    if world == 1 and args.workloads.strip():
        del dls, pipe, step, xs
        import gc
        gc.collect()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        extra = {}
        for w in args.workloads.split(","):
            w = int(w)
            if w == args.config:
                continue
            try:
                extra[config(w).name] = measure_extra_workload(w, args, dev, stream, peaks, peak_src)
            except Exception as exc:   # an extra measurement never costs the main line
                extra[config(w).name] = {"error": f"{type(exc).__name__}: {exc}"}
                gc.collect()
                torch.cuda.empty_cache()
        out["workloads"] = extra
    return out, cfg


def merge_ablation(cfg, dl, stream, split_step_ms: float, reps: int):
    """The alternative the explainer's split-weight figure argues against: copy
    the local and the remote experts into one contiguous buffer (expert order)
    before every grouped GEMM, then address it as a single pool.  Returns the
    merge copy time and the step time with it, next to the split-table step."""
    import numpy as np
    import torch
    from split_weight_b200 import SplitWeights
    from split_weight_b200 import _lib as L
    ml = dl.layer
    w = ml.weights
    merged = torch.empty(cfg.E * w.stride, dtype=torch.uint8, device=w.local.device)
    h = stream.cuda_stream

    def merge():
        # the default placement keeps experts in slot order in each pool:
        # local = experts [0, n_local), remote = the rest
        L.check(L.moe_prefetch_layer(w.local.data_ptr(), merged.data_ptr(), w.n_local * w.stride,
                                     0, h, None, None))
        L.check(L.moe_prefetch_layer(w.remote.data_ptr(), merged.data_ptr() + w.n_local * w.stride,
                                     w.n_remote * w.stride, 0, h, None, None))

    ps = np.arange(cfg.E, dtype=np.int64)
    mw = SplitWeights(w.H, w.I, w.w_dtype, ps.astype(np.int32), merged, cfg.E, merged[:1], 0,
                      w.shared)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    merge()
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        merge()
    ev[1].record(stream)
    saved = ml.weights
    ml.weights = mw
    try:
        ev[2].record(stream)
        for _ in range(reps):
            merge()
            ml.route(dl.x, h)
            ml.permute(dl.x, h)
            ml.grouped_ffn(h, x=dl.x)
            ml.combine(h)
        ev[3].record(stream)
        torch.cuda.synchronize()
    finally:
        ml.weights = saved
    merge_ms = ev[0].elapsed_time(ev[1]) / reps
    merged_step = ev[2].elapsed_time(ev[3]) / reps
    return {"merged_buffer_bytes": cfg.E * w.stride, "merge_copy_ms": round(merge_ms, 4),
            "step_ms_split_table": round(split_step_ms, 4),
            "step_ms_merge_then_gemm": round(merged_step, 4),
            "merge_overhead_fraction": round(merged_step / split_step_ms - 1.0, 4)}


# ----------------------------------------------------------------------- oracle
def oracle_sample(cfg, n_tokens: int, reps: int = 1):
    """Times the CPU oracle on the first n_tokens tokens of layer 0: routing,
    then the SwiGLU experts and combine for those tokens.  Expert weights are
    generated before the clock starts.  Returns (tokens/s, seconds, note)."""
    from moe_inputs import device as mdev, gen
    from oracle import workload as ow

    li = gen.layer_inputs(cfg, 0)
    toks = np.arange(min(n_tokens, cfg.T))
    sub = gen.LayerInputs(x=li.x[toks], x_bits=None, wg=li.wg, bias=li.bias)
    idx, w, _ = ow.route(cfg.with_(T=len(toks)), 0, sub)
    pool, slot = mdev.default_placement(cfg)
    cache = {}
    pools = ow.split_pools(cfg, 0, pool, slot, cache)
    for e in np.unique(idx):
        pools.expert(int(e))  # generate (untimed)
    t0 = time.perf_counter()
    for _ in range(reps):
        idx2, w2, _ = ow.route(cfg.with_(T=len(toks)), 0, sub)
        ow.layer_tokens(cfg.with_(T=len(toks)), 0, np.arange(len(toks)), idx2, w2, pool, slot,
                        sub, cache)
    dt = time.perf_counter() - t0
    return len(toks) * reps / dt, dt, f"first {len(toks)} token(s) of layer 0, {reps} pass(es)"


def cpu_cores() -> int:
    return len(os.sched_getaffinity(0))


def run_reference(args, rank, world):
    """The oracle as the reference arm.  One step is one ninth of one token's
    MoE block: the token's routing (on its first step) and one of its k
    routed experts or the shared expert, in fp64, accumulated into its output
    row.  Tokens cycle over the first few of the workload; their expert
    weights are generated before the clock starts."""
    from moe_inputs import config, device as mdev, gen
    from oracle import moe as om, workload as ow
    cfg = config(args.config)
    if rank != 0:
        return None
    parts = cfg.k + (1 if cfg.has_shared else 0)
    n_tok = max(1, min(4, cfg.T, -(-(args.steps + args.warmup) // parts)))
    li = gen.layer_inputs(cfg, 0)
    pool, slot = mdev.default_placement(cfg)
    cache = {}
    pools = ow.split_pools(cfg, 0, pool, slot, cache)
    sub_cfg = cfg.with_(T=1)
    routes = []
    for t in range(n_tok):
        sub = gen.LayerInputs(x=li.x[t:t + 1], x_bits=None, wg=li.wg, bias=li.bias)
        idx, w, _ = ow.route(sub_cfg, 0, sub)
        routes.append((sub, idx, w))
        for e in idx[0]:
            pools.expert(int(e))          # generated before timing

    def one_step(s):
        t = (s // parts) % n_tok
        part = s % parts
        sub, idx, w = routes[t]
        x64 = sub.x.astype(np.float64)
        if part == 0:
            ow.route(sub_cfg, 0, sub)
        if part < cfg.k:
            ex = pools.expert(int(idx[0, part]))
            return w[0, part] * om.swiglu_ffn(x64, ex.gu_f64(), ex.down_f64())
        return om.swiglu_ffn(x64, pools.shared.gu_f64(), pools.shared.down_f64())

    for s in range(args.warmup):
        one_step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        one_step(args.warmup + s)
    dt = time.perf_counter() - t0
    value = (args.steps / parts) / dt
    note = (f"each step: 1/{parts} of one token's block on the CPU oracle (routing over all "
            f"{cfg.E} experts on the token's first step, then one of its {cfg.k} routed experts "
            f"or the shared expert, fp64); tokens cycle over the first {n_tok}")
    return {
        "metric": METRIC, "value": round(value, 6), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / max(args.steps, 1) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_desc(cfg), "parallelism": "CPU oracle on rank 0"},
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": cpu_cores(),
                         "kind": "oracle", "sample": note},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------- peaks
def measure_peaks(reps: int = 10):
    """Denominators the driver's peak file does not carry, measured with
    library kernels on this GPU (CUDA events, best of `reps` after warm-up,
    no clock changes): the dense fp8 e4m3 GEMM (torch._scaled_mm at 8192^3,
    unit scales, bf16 out), the dense bf16 GEMM beside it (same shape), and
    the read-only HBM stream (torch.sum over 4 GiB of fp32) beside a copy."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def best(fn, warm=3):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return min(ts)

    n = 8192
    out = {}
    with ClockSampler(0) as clk:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()   # column-major
        one = torch.ones((), device=dev)
        ms = best(lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
        out["fp8_tflops"] = round(2.0 * n ** 3 / (ms * 1e-3) / 1e12, 1)
        del a, b
        a16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
        b16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
        ms = best(lambda: torch.matmul(a16, b16))
        out["bf16_tflops_same_run"] = round(2.0 * n ** 3 / (ms * 1e-3) / 1e12, 1)
        del a16, b16
        x = torch.rand(1 << 30, device=dev)                       # 4 GiB fp32
        ms = best(lambda: x.sum())
        out["hbm_read_gbs"] = round(x.numel() * 4 / (ms * 1e-3) / 1e9, 1)
        y = torch.empty_like(x)
        ms = best(lambda: y.copy_(x))
        out["hbm_copy_gbs_same_run"] = round(2 * x.numel() * 4 / (ms * 1e-3) / 1e9, 1)
        del x, y
        torch.cuda.synchronize()
    out["clocks"] = clk.summary()
    out["method"] = ("CUDA events, best of %d after 3 warm-up calls; fp8: torch._scaled_mm "
                     "e4m3 x e4m3 8192^3, unit fp32 scales, bf16 out; bf16: torch.matmul "
                     "8192^3; read: torch.sum over 2^30 fp32; copy: Tensor.copy_ of 4 GiB "
                     "(read + write bytes)" % reps)
    return out


# ----------------------------------------------------------------------- main
def main(argv=None):
    args = parse_args(argv)
    if args.measure_peaks:
        print(json.dumps(measure_peaks()), flush=True)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    out, cfg = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, note = oracle_sample(cfg, 6 if cfg.T > 64 else cfg.T)
        out["cpu_baseline"] = {"value": round(v, 6), "unit": "tokens/s", "cores": cpu_cores(),
                               "kind": "oracle", "sample": note + f" ({dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
