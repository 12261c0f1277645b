#!/usr/bin/env python
"""Benchmark of the B200 LatentMoE layer forward (tokens/s and roofline).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one latentmoe_forward call over the workload's T tokens: routing,
permutation, fc1 + shared up, expert up/down, combine, fc2 + shared down.
Inputs are seeded synthetic tensors already resident in HBM (x ~ N(0,1),
weights ~ N(0, 0.02) bf16, bias ~ U(-0.1, 0.1)); the ~22 GB of weights are far
larger than L2, so no flush is needed between steps (workloads whose weights
fit in L2, such as `tiny`, get a 256 MB overwrite between timed forwards and
are timed forward by forward). Timing: CUDA events on
the launching stream, W untimed warm-up steps, then exactly K steps between a
barrier + synchronize on both sides; the max over ranks. N > 1 runs N
independent replicas (each rank processes its own T tokens; no collective on
the data path), so `value` is the whole-job tokens/s and scaling is weak.

`--impl reference` times the fp64 CPU oracle on the host cores (the baseline
arm) on the same workload and metric, on a bounded sample of tokens per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LatentMoE layer fwd tokens/s on 1 B200; % of bf16 tensor peak / HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Stages between the library's profile events: "routing" is the statistics reset (plus the router GEMM
# where it cannot join the input GEMM launch); the router logits are the first problem of the fc1 +
# shared up launch, and the selection, the fp64 re-decision and the counting sort run on a second
# stream inside "input_gemm", next to the exact re-roundings of z and a_s.
STAGES = ["routing", "input_gemm", "gather", "expert_up_gemm", "expert_down_gemm", "combine", "output_gemm"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", self.gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ work accounting
def expert_gemm_work(w, distinct, nvfp4=False):
    """Algorithmic FLOPs and bytes of one expert GEMM launch (up or down)."""
    A = w.T * w.k
    flops = 2.0 * A * w.L * w.I
    weight_bytes = distinct * w.L * w.I * ((0.5 + 1.0 / 16) if nvfp4 else 2.0)
    act_bytes = 2.0 * A * w.L + 2.0 * A * w.I   # bf16 operand rows in, bf16 rows out (up) / fp32 out (down ~ same order)
    return flops, weight_bytes + act_bytes


def replica_x_offset(rank: int, shape) -> int:
    """First element of rank's x in the generator's x stream: replica r processes
    tokens r*T .. (r+1)*T - 1, so the ranks together process N*T distinct tokens."""
    return rank * shape.T * shape.H


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time (identity on one process)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ our arm
L2_BYTES = 126 << 20


def weight_bytes_of(shape):
    return 2 * (shape.E * 2 * shape.L * shape.I + shape.E * shape.H + 2 * shape.H * shape.L + 2 * shape.H * shape.Is)


def l2_resident(shape):
    """A 256 MB device buffer to overwrite between timed forwards when the
    layer's weights would otherwise stay in L2 (small workloads); else None."""
    import torch
    if weight_bytes_of(shape) > 2 * L2_BYTES:
        return None
    return torch.empty((256 << 20,), dtype=torch.uint8, device="cuda")


def l2_note(shape):
    gb = weight_bytes_of(shape) / 1e9
    if weight_bytes_of(shape) > 2 * L2_BYTES:
        return "inputs larger than L2 (%.1f GB of weights), no flush" % gb
    return ("weights fit in L2 (%.3f GB): 256 MB overwritten between timed forwards (L2 flushed); "
            "ms_per_step sums each forward's own CUDA-event time" % gb)


def measure(shape, steps, warmup, world, rank, local, dist, torch, nvfp4=False):
    import latentmoe_layer_b200 as lm
    import synth

    dev = synth.device_inputs(shape, 0)
    if rank > 0:  # each replica processes its own tokens: rows rank*T .. (rank+1)*T of the x stream
        lib = synth._gpu_lib()
        import ctypes
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        n = shape.T * shape.H
        off = replica_x_offset(rank, shape)
        if shape.x_f32:
            lib.synth_cuda_fill_normal_f32(dev["x"].data_ptr(), n, 0, synth.TID_X, 1.0, off, stream)
        else:
            lib.synth_cuda_fill_normal_bf16(dev["x"].data_ptr(), n, 0, synth.TID_X, 1.0, off, stream)
        if shape.skew_hot:
            dev["x"][:, 0] = 1.0
    if nvfp4:  # expert weights converted once, before any timing
        q = {}
        q["up_w"], q["up_sf"], q["up_gs"] = lm.quantize_nvfp4(dev["up_w"])
        q["down_w"], q["down_sf"], q["down_gs"] = lm.quantize_nvfp4(dev["down_w"])
        layer = lm.LatentMoE(shape, dict(dev, **q), shape.T, x_f32=shape.x_f32, expert_format=lm.LMOE_EXPERTS_NVFP4)
        dev["nvfp4"] = q
    else:
        layer = lm.LatentMoE(shape, dev, shape.T, x_f32=shape.x_f32)
    x = dev["x"]
    y = torch.empty((shape.T, shape.H), dtype=torch.float32, device="cuda")
    layer.workspace(shape.T)
    for _ in range(warmup):
        layer.forward(x, y)
    torch.cuda.synchronize()

    # stage events, created up front (one set of 8 per step)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(steps)]
    for row in evs:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    import ctypes
    handles = [(ctypes.c_void_p * 8)(*[e.cuda_event for e in row]) for row in evs]

    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local] if os.environ.get("CUDA_VISIBLE_DEVICES") \
        else str(local)
    clocks = ClockSampler(gpu_id)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    flush = l2_resident(shape)
    t_start.record()
    for i in range(steps):
        if flush is not None:
            flush.zero_()  # between timed forwards: evicts the layer's weights from L2
        lm.latentmoe_set_profile_events(layer.h, ctypes.cast(handles[i], ctypes.c_void_p), 8)
        layer.forward(x, y)
    t_end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    lm.latentmoe_set_profile_events(layer.h, None, 0)
    if flush is None:
        ms = max_over_ranks(t_start.elapsed_time(t_end), dist, "cuda")
    else:  # the forwards alone: each one's first and last stage markers
        ms = max_over_ranks(sum(evs[i][0].elapsed_time(evs[i][-1]) for i in range(steps)), dist, "cuda")
    stage_ms = {name: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps))
                for j, name in enumerate(STAGES)}
    st = layer.stats()
    # expert loads of this batch (one more, untimed forward that also writes the counts)
    counts = torch.empty((shape.E,), dtype=torch.int32, device="cuda")
    layer.forward(x, y, counts=counts)
    cnt = counts.cpu().tolist()
    loads = {"load_imbalance": round(max(cnt) / (shape.T * shape.k / shape.E), 3)}
    if shape.skew_hot:
        loads["hot_share"] = round(sum(cnt[:shape.skew_hot]) / float(shape.T * shape.k), 4)

    # End to end through the public call with host buffers: every step copies its
    # x from pinned host memory to the device, runs the layer and copies y back.
    # Copies run on their own streams, double-buffered, so step i's compute
    # overlaps step i+1's upload and step i-1's download (as a serving loop would):
    # pipelined throughput. e2e_serial_run times the same steps with each step's
    # upload, forward and download in sequence on one stream (per-call latency).
    xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    xh.copy_(x)
    yh = torch.empty((shape.T, shape.H), dtype=torch.float32, pin_memory=True)
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        h2d_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        d2h_done = [torch.cuda.Event() for _ in range(2)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(comp)
        up.wait_event(start)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(comp_done[b])
                xd[b].copy_(xh, non_blocking=True)
                h2d_done[b].record(up)
            comp.wait_event(h2d_done[b])
            if i >= 2:
                comp.wait_event(d2h_done[b])
            layer.forward(xd[b], yd[b])
            comp_done[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[b])
                yh.copy_(yd[b], non_blocking=True)
                d2h_done[b].record(down)
        comp.wait_stream(down)
        end.record(comp)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    def e2e_serial_run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(comp)
        for i in range(n):
            xd[0].copy_(xh, non_blocking=True)
            layer.forward(xd[0], yd[0])
            yh.copy_(yd[0], non_blocking=True)
        end.record(comp)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    e2e_run(max(2, warmup))
    e_steps = max(2, min(steps, 50))
    if dist is not None:
        dist.barrier()
    e_ms = max_over_ranks(e2e_run(e_steps), dist, "cuda")
    e2e_serial_run(2)
    if dist is not None:
        dist.barrier()
    es_ms = max_over_ranks(e2e_serial_run(e_steps), dist, "cuda")
    res = {
        "ms": ms, "stage_ms": stage_ms, "stats": st, "loads": loads, "clocks": clk, "e2e_ms": e_ms, "e2e_serial_ms": es_ms,
        "e2e_steps": e_steps,
        "h2d": x.numel() * x.element_size(), "d2h": y.numel() * 4, "layer": layer, "dev": dev,
    }
    return res


# DRAM bytes per assignment of the expert up GEMM, from an ncu capture of this
# kernel on the probe_e64 workload (1.978 GB for 45 056 assignments; the same
# tile shapes and rows per expert as ultra_prefill). Traffic grows with the
# assignments (rows) and, at ~704 rows per expert, with the experts in the same
# ratio. Reset to None when that kernel changes.
UP_GEMM_DRAM_BYTES_PER_ASSIGNMENT = (1.529e9 + 0.449e9) / 45056


def roofline_for(shape, res, peaks, peak_src, prefill: bool, nvfp4=False):
    st = res["stats"]
    flops, byts = expert_gemm_work(shape, st.distinct_experts, nvfp4)
    up_ms, dn_ms = res["stage_ms"]["expert_up_gemm"], res["stage_ms"]["expert_down_gemm"]
    name, kms = ("expert_up_gemm", up_ms) if up_ms >= dn_ms else ("expert_down_gemm", dn_ms)
    if prefill:
        ach = flops / (kms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        return {"kernel": name, "bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "peak_kind": "%s burst bf16 (the target denominator)" % peak_src,
                "frac_of_sustained_peak": round(ach / peaks["bf16_tflops_sustained"], 4),
                "traffic": (round(UP_GEMM_DRAM_BYTES_PER_ASSIGNMENT * shape.T * shape.k)
                            if name == "expert_up_gemm" and UP_GEMM_DRAM_BYTES_PER_ASSIGNMENT else None),
                "traffic_note": "ncu capture of the same kernel on probe_e64, scaled by assignments",
                "algorithmic_per_launch": flops, "launch_ms": round(kms, 4)}
    ach = byts / (kms * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
            "frac": round(ach / peak, 4), "peak_kind": "%s HBM copy" % peak_src, "traffic": None,
            "algorithmic_per_launch": byts, "launch_ms": round(kms, 4)}


def target_of(shape, summary, prefill):
    """The layer-level target the throughput is held to: >= 60% of the bf16 tensor
    peak (burst) at large token counts, >= 70% of HBM bandwidth over the touched
    weights at decode sizes. A layer whose weights fit in L2 is latency-bound:
    reported, with no target."""
    if weight_bytes_of(shape) < L2_BYTES:
        return {"metric": None, "value": None, "target": None, "met": None,
                "note": "latency-bound (the weights fit in L2): reported only"}
    key, goal = ("layer_frac_of_burst_bf16", 0.60) if prefill else ("layer_frac_of_hbm", 0.70)
    return {"metric": key, "value": summary[key], "target": goal, "met": bool(summary[key] >= goal)}


def layer_summary(shape, res, peaks, peak_src, steps, nvfp4=False):
    import latentmoe_layer_b200.accounting as acc
    st = res["stats"]
    ms_step = res["ms"] / steps
    tok_s = shape.T / (ms_step * 1e-3)
    layer_flops = acc.flops_per_token(shape) * shape.T
    layer_bytes = acc.min_bytes_per_call(shape, st.distinct_experts, nvfp4)
    return {
        "ms_per_step": round(ms_step, 4), "tokens_per_s": round(tok_s, 1),
        "layer_tflops": round(layer_flops / (ms_step * 1e-3) / 1e12, 1),
        "layer_frac_of_sustained_bf16": round(layer_flops / (ms_step * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"], 4),
        "layer_frac_of_burst_bf16": round(layer_flops / (ms_step * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
        "layer_gbs_min_bytes": round(layer_bytes / (ms_step * 1e-3) / 1e9, 1),
        "layer_frac_of_hbm": round(layer_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "stage_ms": {k: round(v, 4) for k, v in res["stage_ms"].items()},
        "distinct_experts": st.distinct_experts, "max_expert_tokens": st.max_expert_tokens,
        "flagged_tokens": st.flagged_tokens, **res["loads"],
    }


def cpu_baseline(shape, dev, target_s=15.0):
    """The oracle as it stands, on the host cores, over a bounded token sample."""
    import numpy as np
    import oracle
    import torch

    def bits(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    cores = os.cpu_count() or 1
    need = min(shape.T, max(cores, 8))
    wts = {k: bits(dev[k]) for k in ("router_w", "fc1_w", "fc2_w", "shared_up_w", "shared_down_w")}
    wts["e_bias"] = dev["e_bias"].cpu().numpy()
    up = bits(dev["up_w"]) if shape.E * shape.I * shape.L <= 4 << 30 else None
    dn = bits(dev["down_w"]) if up is not None else None
    if up is None:  # per-expert host copies (bf16 bits), ~22 GB at the Ultra shape
        up = [bits(dev["up_w"][e]) for e in range(shape.E)]
        dn = [bits(dev["down_w"][e]) for e in range(shape.E)]
    wts["up_w"], wts["down_w"] = up, dn
    xs = dev["x"].cpu().numpy() if shape.x_f32 else bits(dev["x"])
    cfg = oracle.make_cfg(shape)
    t0 = time.time()
    oracle.forward(cfg, xs[:need], wts)
    t1 = time.time()
    per_tok = (t1 - t0) / need
    more = int(min(shape.T - need, max(0, target_s - (t1 - t0)) / max(per_tok, 1e-9)))
    more = max(0, (more // cores) * cores)
    done = need
    if more > 0:
        oracle.forward(cfg, xs[need:need + more], wts)
        done += more
    t2 = time.time()
    return {"value": round(done / (t2 - t0), 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "first %d of %d tokens of the workload, full layer per token (fp64, OpenMP over tokens)" %
                      (done, shape.T), "seconds": round(t2 - t0, 2)}, wts


def cpu_baseline_one_core(shape, wts, dev, target_s=8.0):
    """The same oracle on one host core (its OpenMP runtime limited to one
    thread for this measurement, then restored), over a smaller token sample."""
    import ctypes
    import numpy as np
    import oracle
    import torch
    gomp = ctypes.CDLL("libgomp.so.1")
    gomp.omp_get_max_threads.restype = ctypes.c_int
    before = gomp.omp_get_max_threads()
    xs = dev["x"].cpu().numpy() if shape.x_f32 else dev["x"].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    cfg = oracle.make_cfg(shape)
    gomp.omp_set_num_threads(1)
    try:
        t0 = time.time()
        oracle.forward(cfg, xs[:1], wts)
        t1 = time.time()
        more = int(min(shape.T - 1, max(0.0, target_s - (t1 - t0)) / max(t1 - t0, 1e-9)))
        if more > 0:
            oracle.forward(cfg, xs[1:1 + more], wts)
        t2 = time.time()
    finally:
        gomp.omp_set_num_threads(before)
    done = 1 + max(more, 0)
    return {"value": round(done / (t2 - t0), 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "first %d of %d tokens of the workload, full layer per token (fp64, one thread)" %
                      (done, shape.T), "seconds": round(t2 - t0, 2)}


def run_ours(args):
    import torch
    import synth
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    peaks, peak_src = load_peaks()
    shape = synth.WORKLOADS[args.workload]
    prefill = shape.T * shape.k > 64 * shape.E
    nv = args.experts == "nvfp4"
    res = measure(shape, args.steps, args.warmup, world, rank, local, dist, torch, nvfp4=nv)
    ms_step = res["ms"] / args.steps
    value = world * shape.T / (ms_step * 1e-3)
    e2e_value = world * shape.T * res["e2e_steps"] / (res["e2e_ms"] * 1e-3)
    summary = layer_summary(shape, res, peaks, peak_src, args.steps, nvfp4=nv)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; x~N(0,1), weights~N(0,0.02) bf16)",
        "config": {"workload": shape.name, "T": shape.T, "H": shape.H, "L": shape.L, "E": shape.E, "k": shape.k,
                   "n_group": shape.G, "topk_group": shape.Gk, "I": shape.I, "Is": shape.Is,
                   "global_batch": shape.T * world, "parallelism": "replicas" if world > 1 else "single",
                   "experts": args.experts,
                   "l2": l2_note(shape)},
        "roofline": roofline_for(shape, res, peaks, peak_src, prefill, nvfp4=nv),
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"],
                "mode": "pipelined: pinned-host copies double-buffered on their own streams, overlapping compute",
                "serial_value": round(world * shape.T * res["e2e_steps"] / (res["e2e_serial_ms"] * 1e-3), 1),
                "serial_mode": "each step's upload, forward and download in sequence on one stream"},
        "gpu_launches": res["stats"].kernel_launches * args.steps,
        "clocks": res["clocks"],
        "layer": summary,
        "target": target_of(shape, summary, prefill),
    }
    layer, dev = res["layer"], res["dev"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not nv:
        cb, wts = cpu_baseline(shape, dev)
        line["cpu_baseline"] = cb
        line["cpu_baseline_1core"] = cpu_baseline_one_core(shape, wts, dev)
    layer.close()
    del res, layer, dev
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and args.secondary not in ("", "none") and args.secondary != shape.name:
        s2 = synth.WORKLOADS[args.secondary]
        r2 = measure(s2, args.secondary_steps, args.warmup, 1, 0, local, None, torch)
        line["secondary"] = {"workload": s2.name, "value": round(s2.T / (r2["ms"] / args.secondary_steps * 1e-3), 1),
                             "unit": "tokens/s", "steps": args.secondary_steps,
                             "roofline": roofline_for(s2, r2, peaks, peak_src, s2.T * s2.k > 64 * s2.E),
                             "layer": layer_summary(s2, r2, peaks, peak_src, args.secondary_steps),
                             "clocks": r2["clocks"]}
        line["secondary"]["target"] = target_of(s2, line["secondary"]["layer"], s2.T * s2.k > 64 * s2.E)
        r2["layer"].close()
        del r2
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and args.nvfp4_workload not in ("", "none"):
        # the same layer with NVFP4 routed-expert weights (dense weights stay bf16)
        s3 = synth.WORKLOADS[args.nvfp4_workload]
        r3 = measure(s3, args.secondary_steps, args.warmup, 1, 0, local, None, torch, nvfp4=True)
        line["nvfp4_experts"] = {
            "workload": s3.name, "value": round(s3.T / (r3["ms"] / args.secondary_steps * 1e-3), 1),
            "unit": "tokens/s", "steps": args.secondary_steps,
            "roofline": roofline_for(s3, r3, peaks, peak_src, s3.T * s3.k > 64 * s3.E, nvfp4=True),
            "layer": layer_summary(s3, r3, peaks, peak_src, args.secondary_steps, nvfp4=True),
            "clocks": r3["clocks"]}
        line["nvfp4_experts"]["target"] = target_of(s3, line["nvfp4_experts"]["layer"], s3.T * s3.k > 64 * s3.E)
        r3["layer"].close()
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 oracle on the host cores: same workload and metric, bounded token sample per step."""
    world, rank, local = dist_setup()
    if rank != 0:
        return
    import numpy as np
    import oracle
    import synth
    shape = synth.WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:  # inputs made by the device generator, copied to the host (input generation only)
        torch.cuda.set_device(local)
        dev = synth.device_inputs(shape, 0)

        def bits(t):
            return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        wts = {k: bits(dev[k]) for k in ("router_w", "fc1_w", "fc2_w", "shared_up_w", "shared_down_w")}
        wts["e_bias"] = dev["e_bias"].cpu().numpy()
        wts["up_w"] = [bits(dev["up_w"][e]) for e in range(shape.E)]
        wts["down_w"] = [bits(dev["down_w"][e]) for e in range(shape.E)]
        xs = dev["x"].cpu().numpy() if shape.x_f32 else bits(dev["x"])
        del dev
        torch.cuda.empty_cache()
    else:
        wts = synth.host_inputs(shape, 0)
        xs = wts["x"]
    cfg = oracle.make_cfg(shape)
    per_step = min(shape.T, cores * args.ref_tokens_per_core)
    pos = 0
    for _ in range(args.warmup):
        oracle.forward(cfg, xs[pos:pos + per_step], wts)
        pos = (pos + per_step) % max(1, shape.T - per_step + 1)
    t0 = time.time()
    for _ in range(args.steps):
        oracle.forward(cfg, xs[pos:pos + per_step], wts)
        pos = (pos + per_step) % max(1, shape.T - per_step + 1)
    dt = time.time() - t0
    value = per_step * args.steps / dt
    sample = "%d of %d tokens per step (full layer per token, fp64, OpenMP over tokens)" % (per_step, shape.T)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": shape.name, "T": shape.T},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ultra_prefill")
    ap.add_argument("--secondary", default="ultra_decode", help="second workload reported under 'secondary'")
    ap.add_argument("--secondary-steps", type=int, default=200)
    ap.add_argument("--experts", choices=["bf16", "nvfp4"], default="bf16",
                    help="routed-expert weight format of the main measurement")
    ap.add_argument("--nvfp4-workload", default="ultra_decode",
                    help="workload measured again with NVFP4 expert weights ('none' to skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens-per-core", type=int, default=2)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
