"""Benchmark: packed-ternary decode GEMV (with the FWHT-1024 rotation) on B200.

One step = one decode token through the 5120x5120 / 5120x17408 / 17408x5120
triple at M = 1: one bt_gemv_batched call takes the three matrices, each with
its own bf16 activation, rotates each activation block-wise (R = H_1024 S / 32)
and multiplies by the base-3 packed ternary weights with g128 FP16 scales. The weights are synthetic and seeded (the pages' 27B model
is not available); twelve distinct copies of the triple (537 MB, over four
times the 126 MB L2) are used in turn so every step streams from HBM.

`value` = packed weight bytes (codes + scales) per step / device time per step.
The same JSON line carries the prefill GEMM (pp512: M = 512 on the same
triple) in TFLOP/s, the 2-bit layout twin, the end-to-end figure through the
public API with host buffers, a roofline block and the CPU oracle baseline.

`--impl reference` times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload and prints the same metric.
Multi-GPU (`--gpus N` under torchrun): independent replicas, weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "packed-ternary GEMV weight GB/s (% of HBM peak); pp512 GEMM TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
# DRAM bytes (read + write) per launch of the table-lookup kernel over the
# decode triple (one bt_gemv_batched call), from an ncu capture of the current
# kernel (dram__bytes_read.sum + dram__bytes_write.sum); None when the kernel
# has changed since the counters were taken.
TRAFFIC_PER_LAUNCH = 44_860_160
STEPS_PER_GRAPH = 4


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs", 6545.0), "bf16_tflops": d.get("bf16_tflops", 1627.8),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", 1395.0), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self._t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
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
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------- multi-rank timing ---

def max_over_ranks(ms: float, world: int, dist=None, device=None) -> float:
    """The slowest rank's time: every rank calls this once per timed region."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, ms: float, world: int) -> float:
    """Units per second over all ranks (weak scaling: each rank does its own units)."""
    return units_per_rank * world / (ms * 1e-3)


# ----------------------------------------------------------------- inputs ---

def _layer_tensors(bt, torch, dev, layout, idx, L, with_x=False):
    import workloads
    inp = workloads.layer_inputs("C1", L, index=idx, with_x=with_x)
    codes = bt.pack(torch.from_numpy(inp["trits"]).to(dev), layout)
    scales = torch.from_numpy(inp["scales"].view(np.int16)).to(dev)
    return codes, scales, inp


def _weight_bytes(L, layout):
    if layout == 2:  # continuous base-3: ceil(K/5) bytes rounded up to 16, plus the scales
        return L.N * (((L.K + 4) // 5 + 15) // 16 * 16 + (L.K // 128) * 2)
    per_group = (26 if layout == 0 else 32) + 2
    return L.N * (L.K // 128) * per_group


# ---------------------------------------------------------------- GPU arm ---

def run_gpu(args, rank, world):
    import torch
    import torch.distributed as dist
    import ternary_weight_fwht1024_b200 as bt
    import workloads

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    bt.load()
    peaks = _peaks()
    triple = workloads.TRIPLE
    sign = torch.from_numpy(workloads.sign1024()).to(dev)
    copies = max(4, math.ceil(4 * L2_BYTES / sum(_weight_bytes(L, 0) for L in triple)))

    def build(layout):
        base = [_layer_tensors(bt, torch, dev, layout, i, L)[:2] for i, L in enumerate(triple)]
        reps = [[(c.clone(), s.clone()) for c, s in base] for _ in range(copies)]
        del base
        return reps

    stream = torch.cuda.Stream(device=dev)
    M = 1
    g = workloads.rng(2 * 1_000_003 + 99)
    xs_host = [torch.from_numpy(workloads.activations_bf16_bits(g, M, L.K, True).view(np.int16)).pin_memory()
               for L in triple]
    xs = [h.to(dev).view(torch.bfloat16) for h in xs_host]
    ys = [torch.empty((M, L.N), dtype=torch.float32, device=dev) for L in triple]
    probs_of = lambda reps, r, xs_, ys_: [dict(codes=reps[r][i][0], scales=reps[r][i][1], x=xs_[i], y=ys_[i],  # noqa: E731
                                               N=L.N, K=L.K) for i, L in enumerate(triple)]
    ws = torch.empty(max([bt.gemv_workspace_bytes(l, M, L.N, L.K) for L in triple for l in (0, 1)] +
                         [bt.gemv_batched_workspace_bytes(l, [dict(N=L.N, K=L.K) for L in triple]) for l in (0, 1)]),
                     dtype=torch.uint8, device=dev)

    # Steps are replayed from CUDA graphs of STEPS_PER_GRAPH consecutive steps
    # (each step its own bt_gemv_batched call on the next weight copy), so the
    # host's graph launches keep ahead of the device.
    spg = STEPS_PER_GRAPH if copies % STEPS_PER_GRAPH == 0 else 1

    def graphs_for(reps, layout, with_events=False):
        gs = []
        with torch.cuda.stream(stream):
            for r in range(copies):  # warm the code path before capture
                bt.gemv_batched(probs_of(reps, r, xs, ys), sign, layout, ws=ws)
            torch.cuda.synchronize()
            for r0 in range(0, copies, spg):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    for r in range(r0, r0 + spg):
                        bt.gemv_batched(probs_of(reps, r, xs, ys), sign, layout, ws=ws)
                gs.append(gr)
        return gs

    def timed(gs, steps, warmup, per_call_events=False, per_graph=1):
        """K steps from graphs of `per_graph` steps each (K a multiple of it)."""
        assert steps % per_graph == 0
        warmup = -(-warmup // per_graph)
        steps_r = steps // per_graph
        with torch.cuda.stream(stream):
            for w in range(warmup):
                gs[w % len(gs)].replay()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            st = torch.cuda.Event(enable_timing=True)
            en = torch.cuda.Event(enable_timing=True)
            st.record(stream)
            for k in range(steps_r):
                gs[(warmup + k) % len(gs)].replay()
            en.record(stream)
            torch.cuda.synchronize()
        return max_over_ranks(st.elapsed_time(en) / steps, world, dist, dev)

    if args.steps % spg:
        spg = 1

    # ---- base-3 (headline) ----
    reps3 = build(0)
    gs3 = graphs_for(reps3, 0)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.5)  # let the sampler start before the timed region
        ms3 = timed(gs3, args.steps, args.warmup, per_graph=spg)
    bytes3 = sum(_weight_bytes(L, 0) for L in triple)
    io_bytes = sum(M * L.K * 2 + M * L.N * 4 for L in triple)

    # per-call durations of single bt_gemv calls (context: each call is a main
    # kernel and a reduction), from a CUDA graph of `copies` calls of one layer
    # over the rotating weight copies
    per_layer_us = []
    with torch.cuda.stream(stream):
        for i, L in enumerate(triple):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for r in range(copies):
                    bt.gemv(reps3[r][i][0], reps3[r][i][1], xs[i], sign, L.N, 0, out=ys[i], ws=ws)
            for _ in range(3):
                gr.replay()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            reps_t = 20
            a.record(stream)
            for _ in range(reps_t):
                gr.replay()
            b.record(stream)
            torch.cuda.synchronize()
            per_layer_us.append(a.elapsed_time(b) * 1e3 / (reps_t * copies))
            del gr
    del gs3

    # ---- e2e through the public API with host buffers ----
    # Each step copies the step's activations from pinned host memory, makes
    # the step's bt_gemv_batched call and reads the outputs back into pinned
    # host memory. "graph": the step as a serving loop would run it, captured once
    # as a CUDA graph of those API calls and copies and replayed per step.
    # "eager": the same calls issued from Python every step.
    # one pinned host buffer per direction: a step is one H2D copy of the three
    # activation rows and one D2H copy of the three outputs
    x_host_all = torch.cat([h.view(-1) for h in xs_host]).pin_memory()
    x_dev_all = torch.empty_like(x_host_all, device=dev)
    y_dev_all = torch.empty(sum(M * L.N for L in triple), dtype=torch.float32, device=dev)
    y_host_all = torch.empty_like(y_dev_all, device="cpu").pin_memory()
    xo = [0]
    yo = [0]
    for L in triple:
        xo.append(xo[-1] + M * L.K)
        yo.append(yo[-1] + M * L.N)
    xs_e = [x_dev_all[xo[i]:xo[i + 1]].view(torch.bfloat16).view(M, L.K) for i, L in enumerate(triple)]
    ys_e = [y_dev_all[yo[i]:yo[i + 1]].view(M, L.N) for i, L in enumerate(triple)]

    def e2e_step(r):
        x_dev_all.copy_(x_host_all, non_blocking=True)
        bt.gemv_batched(probs_of(reps3, r, xs_e, ys_e), sign, 0, ws=ws)
        y_host_all.copy_(y_dev_all, non_blocking=True)

    def e2e_timed(run_step):
        with torch.cuda.stream(stream):
            for w in range(args.warmup):
                run_step(w % copies)
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            st = torch.cuda.Event(enable_timing=True)
            en = torch.cuda.Event(enable_timing=True)
            st.record(stream)
            for k in range(args.steps):
                run_step((args.warmup + k) % copies)
            en.record(stream)
            torch.cuda.synchronize()
        return max_over_ranks(st.elapsed_time(en) / args.steps, world, dist, dev)

    e2e_eager_ms = e2e_timed(e2e_step)
    e2e_graphs = []
    with torch.cuda.stream(stream):
        for r in range(copies):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                e2e_step(r)
            e2e_graphs.append(gr)
    e2e_serial_ms = e2e_timed(lambda r: e2e_graphs[r].replay())
    del e2e_graphs

    # Pipelined: a serving loop keeps the copy engines and the SMs busy at once.
    # Two device buffers per direction; step t's H2D copy runs while step t-1
    # computes, and step t's D2H copy while step t+1 computes; events keep each
    # buffer's reuse in order. Every step still
    # copies its activations in and its outputs out. Captured as graphs of
    # STEPS_PER_GRAPH steps.
    cs_in = torch.cuda.Stream(device=dev)
    cs_out = torch.cuda.Stream(device=dev)
    x_dev2 = [torch.empty_like(x_host_all, device=dev) for _ in range(2)]
    y_dev2 = [torch.empty_like(y_dev_all) for _ in range(2)]
    y_host2 = [torch.empty_like(y_dev_all, device="cpu").pin_memory() for _ in range(2)]
    xs2 = [[x_dev2[b][xo[i]:xo[i + 1]].view(torch.bfloat16).view(M, L.K) for i, L in enumerate(triple)]
           for b in range(2)]
    ys2 = [[y_dev2[b][yo[i]:yo[i + 1]].view(M, L.N) for i, L in enumerate(triple)] for b in range(2)]
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "out", "free_x", "free_y")}

    def e2e_pipelined(r0, nsteps):
        # on `stream` (the capture stream): fork the copy streams, run nsteps, join.
        # H2D copies on cs_in, D2H copies on cs_out, so neither direction waits
        # behind the other.
        for b in range(2):
            ev["free_x"][b].record(stream)
            ev["free_y"][b].record(stream)
        cs_in.wait_stream(stream)
        cs_out.wait_stream(stream)
        for t in range(nsteps):
            b = t % 2
            with torch.cuda.stream(cs_in):
                cs_in.wait_event(ev["free_x"][b])
                x_dev2[b].copy_(x_host_all, non_blocking=True)
                ev["in"][b].record(cs_in)
            stream.wait_event(ev["in"][b])
            stream.wait_event(ev["free_y"][b])
            bt.gemv_batched(probs_of(reps3, (r0 + t) % copies, xs2[b], ys2[b]), sign, 0, ws=ws)
            ev["free_x"][b].record(stream)
            ev["out"][b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev["out"][b])
                y_host2[b].copy_(y_dev2[b], non_blocking=True)
                ev["free_y"][b].record(cs_out)
        stream.wait_stream(cs_in)
        stream.wait_stream(cs_out)

    pgraphs = []
    with torch.cuda.stream(stream):
        e2e_pipelined(0, spg)  # warm the path before capture
        torch.cuda.synchronize()
        for r0 in range(0, copies, spg):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                e2e_pipelined(r0, spg)
            pgraphs.append(gr)
    e2e_ms = timed(pgraphs, args.steps, args.warmup, per_graph=spg)
    del pgraphs
    del reps3

    # ---- 2-bit layout twin ----
    reps2 = build(1)
    gs2 = graphs_for(reps2, 1)
    ms2 = timed(gs2, args.steps, args.warmup, per_graph=spg)
    bytes2 = sum(_weight_bytes(L, 1) for L in triple)
    del gs2, reps2

    # ---- continuous base-3 twin (1.725 bit: no per-group byte padding) ----
    reps_c = build(2)
    gs_c = graphs_for(reps_c, 2)
    ms_c = timed(gs_c, args.steps, args.warmup, per_graph=spg)
    bytes_c = sum(_weight_bytes(L, 2) for L in triple)
    del gs_c, reps_c

    # ---- GEMV / GEMM crossover on the triple (base-3) ----
    crossover = None
    if not args.no_sweep:
        try:
            crossover = run_crossover(bt, torch, dev, stream, sign)
        except Exception as e:
            crossover = {"error": str(e)[:200]}

    # ---- prefill GEMM pp512, both layouts (seeded C3 / C4 inputs) ----
    gemm = {}
    for layout, cfg, name in ((0, "C3", "base-3"), (1, "C4", "2-bit")):
        try:
            gemm[name] = run_gemm(bt, torch, dev, stream, sign, layout, cfg, args, timed, peaks)
        except Exception as e:  # the prefill path is reported, not required for the headline
            gemm[name] = {"value": None, "error": str(e)[:200]}

    # ---- 27B-equivalent decode sweep: 64 stacks x 2 triples = 384 matrices
    sweep = None
    if not args.no_sweep:
        sweep = {}
        for layout, name in ((0, "base-3"), (1, "2-bit")):
            try:
                sweep[name] = run_sweep(bt, torch, dev, stream, sign, args, world, dist, layout)
            except Exception as e:
                sweep[name] = {"error": str(e)[:200]}

    # ---- standalone rotation sweep: graphs of calls over distinct buffers; where
    # one call's input + output is large, enough buffers that the set exceeds 4x L2
    fwht = {}
    try:
        fwht = run_fwht_sweep(bt, torch, dev, stream, sign)
    except Exception as e:
        fwht = {"error": str(e)[:200]}

    gbs = whole_job_rate(bytes3, ms3, world) / 1e9
    # the dominant launch pair is the step's own bt_gemv_batched call: its
    # algorithmic bytes are the triple's weights and scales plus activations in
    # and outputs out; its duration is the device time of the step
    dom_bytes = sum(_weight_bytes(L, 0) + M * L.K * 2 + M * L.N * 4 for L in triple)
    achieved = dom_bytes / (ms3 * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",  # M = 1: FP32 table entries (partial dot products), FP32 scale products and sums
        "data": "synthetic (seeded trits P(0)=0.4, g128 fp16 scales, bf16 activations with 0.1% x20 outliers)",
        "config": {"workload": "decode GEMV M=1 on the 5120x5120 / 5120x17408 / 17408x5120 triple, base-3 g128, "
                               "FWHT-1024 fused",
                   "M": M, "layout": "base-3 5 trits/byte, 26 B + 2 B scale per 128 weights",
                   "l2": f"{copies} distinct weight copies rotated ({copies * bytes3 / 1e6:.0f} MB > 126 MB L2)",
                   "graph": f"each step is one bt_gemv_batched call (the three matrices); {spg} consecutive steps per "
                            "CUDA graph replay",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": round(100 * gbs / world / peaks["hbm_gbs"], 2),
        "per_call_us": {L.name: round(u, 2) for L, u in zip(triple, per_layer_us)},
        "layout_2bit": {"value": round(bytes2 / (ms2 * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
                        "ms_per_step": round(ms2, 5), "bytes_per_step": bytes2},
        "layout_b3_continuous": {"value": round(bytes_c / (ms_c * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
                                 "ms_per_step": round(ms_c, 5), "bytes_per_step": bytes_c,
                                 "bits_per_weight": round(8 * bytes_c / sum(L.N * L.K for L in triple), 4)},
        "crossover_gemv_gemm": crossover,
        "tokens_per_s_triple": round(1e3 / ms3 * world, 1),
        "gemm": gemm.get("base-3"),
        "gemm_2bit": gemm.get("2-bit"),
        "sweep_27b": sweep,
        "fwht_sweep": fwht,
        "e2e": {"value": round(bytes3 / (e2e_ms * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": sum(M * L.K * 2 for L in triple),
                "d2h_bytes_per_step": sum(M * L.N * 4 for L in triple),
                "mode": f"pipelined serving loop: each step's H2D and D2H copies on copy streams overlap the "
                        f"neighbouring steps' compute (double buffers, events); graphs of {spg} steps",
                "serial": {"value": round(bytes3 / (e2e_serial_ms * 1e-3) / 1e9 * world, 2),
                           "ms_per_step": round(e2e_serial_ms, 5),
                           "mode": "copy in, call, copy out on one stream; one graph per step"},
                "eager": {"value": round(bytes3 / (e2e_eager_ms * 1e-3) / 1e9 * world, 2),
                          "ms_per_step": round(e2e_eager_ms, 5)}},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     # dram__bytes_read.sum + dram__bytes_write.sum of the table-lookup kernel per
                     # launch (one ncu capture of this kernel build)
                     "traffic": TRAFFIC_PER_LAUNCH,
                     "algorithmic_bytes_per_launch": int(dom_bytes),
                     "kernel": "the step's bt_gemv_batched call: gemv_lut_kernel over the three matrices "
                               "and gemv_lut_reduce_kernel, timed together (CUDA events on the launching stream)",
                     "peak_kind": f"HBM copy, {peaks['src']}"},
        "gpu_launches": args.steps * 2,  # table-lookup kernel + reduction kernel per bt_gemv_batched call
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return out


def run_gemm(bt, torch, dev, stream, sign, layout, cfg, args, timed, peaks):
    """pp512: M = 512 seeded activations (with their outliers) through the triple,
    one CUDA graph of three bt_gemm calls per step."""
    import workloads
    triple = workloads.TRIPLE
    Mg = 512
    ins = [workloads.layer_inputs(cfg, L, M=Mg, index=i) for i, L in enumerate(triple)]
    gm = [(bt.pack(torch.from_numpy(c["trits"]).to(dev), layout), torch.from_numpy(c["scales"].view(np.int16)).to(dev))
          for c in ins]
    Xs = [torch.from_numpy(c["x"].view(np.int16)).to(dev).view(torch.bfloat16) for c in ins]
    del ins
    Ys = [torch.empty((Mg, L.N), dtype=torch.bfloat16, device=dev) for L in triple]
    wsg = torch.zeros(max(bt.gemm_workspace_bytes(layout, Mg, L.N, L.K) for L in triple), dtype=torch.uint8,
                      device=dev)
    with torch.cuda.stream(stream):
        for i, L in enumerate(triple):
            bt.gemm(gm[i][0], gm[i][1], Xs[i], sign, L.N, layout, out=Ys[i], ws=wsg)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for i, L in enumerate(triple):
                bt.gemm(gm[i][0], gm[i][1], Xs[i], sign, L.N, layout, out=Ys[i], ws=wsg)
        with ClockSampler(dev.index) as clk:
            time.sleep(0.3)  # let the sampler start before the timed region
            gms = timed([gr], args.steps, args.warmup)
        del gr
    flops = sum(2.0 * Mg * L.N * L.K for L in triple)
    tf = flops / (gms * 1e-3) / 1e12
    return {"value": round(tf, 2), "unit": "TFLOP/s", "ms_per_step": round(gms, 4),
            "workload": f"pp512 triple, {'base-3' if layout == 0 else '2-bit'}, seeded {cfg} activations",
            "frac_of_peak": round(tf / peaks["bf16_tflops"], 4), "peak": peaks["bf16_tflops"],
            "peak_kind": f"bf16 burst, {peaks['src']}",
            # the timed loop is back-to-back GEMMs for about half a second: the
            # fraction of the sustained (power-capped) figure, and the clocks seen
            "frac_of_sustained_peak": round(tf / peaks["bf16_tflops_sustained"], 4),
            "sustained_peak": peaks["bf16_tflops_sustained"],
            "clocks": clk.summary(),
            "l2": "weights (21-26 MB per matrix) re-read from L2 across steps; the activations dominate traffic"}


def run_crossover(bt, torch, dev, stream, sign):
    """Decode GEMV against the prefill GEMM on the base-3 triple for M = 1 .. 64
    activation rows: the GEMV at M = 1 (one batched call) and M = 2, 4, 8, 16
    (three bt_gemv calls), above 16 as M / 16 such calls; the GEMM at M = 128,
    the smallest M it takes (a caller pads M rows up to it). Device time per
    triple from CUDA graphs over weight copies that exceed L2; tokens/s = M /
    time. The crossover is the smallest M at which the padded GEMM is faster."""
    import workloads
    triple = workloads.TRIPLE
    copies = max(4, math.ceil(4 * L2_BYTES / sum(_weight_bytes(L, 0) for L in triple)))
    base = [_layer_tensors(bt, torch, dev, 0, i, L)[:2] for i, L in enumerate(triple)]
    reps = [[(c.clone(), s.clone()) for c, s in base] for _ in range(copies)]
    del base

    def per_triple_us(step):
        with torch.cuda.stream(stream):
            for r in range(copies):
                step(r)
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for r in range(copies):
                    step(r)
            for _ in range(3):
                gr.replay()
            torch.cuda.synchronize()
            a_ = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            n = 10
            a_.record(stream)
            for _ in range(n):
                gr.replay()
            b_.record(stream)
            torch.cuda.synchronize()
        return a_.elapsed_time(b_) * 1e3 / (n * copies)

    g = workloads.rng(4 * 1_000_003 + 7)
    gemv_us = {}
    for M in (1, 2, 4, 8, 16):
        xs = [torch.from_numpy(workloads.activations_bf16_bits(g, M, L.K, True).view(np.int16)).to(dev)
              .view(torch.bfloat16) for L in triple]
        ys = [torch.empty((M, L.N), device=dev) for L in triple]
        if M == 1:
            ws = torch.empty(bt.gemv_batched_workspace_bytes(0, [dict(N=L.N, K=L.K) for L in triple]),
                             dtype=torch.uint8, device=dev)
            step = lambda r: bt.gemv_batched([dict(codes=reps[r][i][0], scales=reps[r][i][1], x=xs[i], y=ys[i],  # noqa: E731
                                                   N=L.N, K=L.K) for i, L in enumerate(triple)], sign, 0, ws=ws)
        else:
            ws = torch.empty(max(bt.gemv_workspace_bytes(0, M, L.N, L.K) for L in triple), dtype=torch.uint8,
                             device=dev)
            step = lambda r: [bt.gemv(reps[r][i][0], reps[r][i][1], xs[i], sign, L.N, 0, out=ys[i], ws=ws)  # noqa: E731
                              for i, L in enumerate(triple)]
        gemv_us[M] = per_triple_us(step)
    Mg = 128
    Xg = [torch.from_numpy(workloads.activations_bf16_bits(g, Mg, L.K, True).view(np.int16)).to(dev)
          .view(torch.bfloat16) for L in triple]
    Yg = [torch.empty((Mg, L.N), dtype=torch.bfloat16, device=dev) for L in triple]
    wsg = torch.empty(max(bt.gemm_workspace_bytes(0, Mg, L.N, L.K) for L in triple), dtype=torch.uint8, device=dev)
    gemm_us = per_triple_us(lambda r: [bt.gemm(reps[r][i][0], reps[r][i][1], Xg[i], sign, L.N, 0, out=Yg[i], ws=wsg)
                                       for i, L in enumerate(triple)])
    del reps
    rows = {}
    cross = None
    for M in (1, 2, 4, 8, 16, 32, 64):
        gv = gemv_us[M] if M <= 16 else gemv_us[16] * (M // 16)
        rows[f"M{M}"] = {"gemv_us": round(gv, 2), "gemm_padded_us": round(gemm_us, 2),
                         "gemv_tokens_per_s": round(M / gv * 1e6, 1), "gemm_tokens_per_s": round(M / gemm_us * 1e6, 1)}
        if cross is None and gemm_us <= gv:
            cross = M
    return {"triple": "5120x5120 / 5120x17408 / 17408x5120, base-3", "gemm_M": Mg, "rows": rows,
            "crossover_M": cross, "note": "GEMV above M = 16 is M/16 calls of 16 rows"}


def run_fwht_sweep(bt, torch, dev, stream, sign):
    """bt_fwht1024 at M in {1, 16, 512} x K in {1024, 5120, 17408}, FP32 output: per
    size, a CUDA graph of calls over distinct input/output buffers (as many as
    keep the set above 4x L2, at most 20). GB/s counts bf16 in + FP32 out."""
    import workloads
    out = {}
    for Mf in (1, 16, 512):
        for Kf in (1024, 5120, 17408):
            per = Mf * Kf * 6
            nbuf = max(1, min(20, math.ceil(4 * L2_BYTES / per)))
            resident = nbuf * per > 4 * L2_BYTES
            g = workloads.rng(5 * 1_000_003 + Mf * 7 + Kf)
            xb = torch.from_numpy(workloads.activations_bf16_bits(g, Mf, Kf, True).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            xs = [xb.clone() for _ in range(nbuf)]
            os_ = [torch.empty((Mf, Kf), dtype=torch.float32, device=dev) for _ in range(nbuf)]
            calls = 20
            with torch.cuda.stream(stream):
                bt.fwht1024(xs[0], sign, out=os_[0])
                torch.cuda.synchronize()
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    for c in range(calls):
                        bt.fwht1024(xs[c % nbuf], sign, out=os_[c % nbuf])
                gr.replay()
                torch.cuda.synchronize()
                a_ = torch.cuda.Event(enable_timing=True)
                b_ = torch.cuda.Event(enable_timing=True)
                a_.record(stream)
                for _ in range(10):
                    gr.replay()
                b_.record(stream)
                torch.cuda.synchronize()
                del gr
            us = a_.elapsed_time(b_) * 1e3 / (10 * calls)
            out[f"M{Mf}xK{Kf}"] = {"us": round(us, 2), "GB/s": round(per / (us * 1e-6) / 1e9, 1),
                                   "buffers": nbuf, "hbm_resident": resident}
            del xs, os_
    return out


def run_sweep(bt, torch, dev, stream, sign, args, world, dist, layout=0):
    """Decode token through 64 stacks x 2 triples (384 matrices, 26.2e9 weights, 5.7 GB
    base-3 / 7.0 GB 2-bit): one seeded triple generated on the host and cloned on the
    device to 128 distinct copies at distinct addresses.

    M = 1: the chained decode step -- each matrix's bf16 output is the next matrix's
    input (5120 -> 5120 -> 17408 -> 5120 -> 5120 -> ...), as in a layer stack: two
    bt_gemv_batched calls of 192 chained matrices (the second starts from the first's
    last output), captured in one CUDA graph per token.
    M = 4, 16: 384 bt_gemv calls per token, the three activations of the triple reused,
    replayed from CUDA graphs."""
    import workloads
    triple = workloads.TRIPLE
    uniq = []
    for i, L in enumerate(triple):
        inp = workloads.layer_inputs("C2", L, index=i, with_x=False)
        uniq.append((bt.pack(torch.from_numpy(inp["trits"]).to(dev), layout),
                     torch.from_numpy(inp["scales"].view(np.int16)).to(dev)))
    n_triples = 128
    mats = [[(c.clone(), s.clone()) for c, s in uniq] for _ in range(n_triples)]
    del uniq
    weight_bytes = n_triples * sum(_weight_bytes(L, layout) for L in triple)
    out = {"weights": int(n_triples * sum(L.N * L.K for L in triple)), "bytes_per_token": weight_bytes,
           "matrices": 3 * n_triples}

    def time_graphs(graphs, tokens=3):
        with torch.cuda.stream(stream):
            for gr in graphs:
                gr.replay()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a_ = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            for _ in range(tokens):
                for gr in graphs:
                    gr.replay()
            b_.record(stream)
            torch.cuda.synchronize()
        return max_over_ranks(a_.elapsed_time(b_) / tokens, world, dist, dev)

    # ---- M = 1, chained
    n_mat = 3 * n_triples
    per_call = n_mat // 2
    g = workloads.rng(3 * 1_000_003 + 1000 + 1)
    x0 = torch.from_numpy(workloads.activations_bf16_bits(g, 1, triple[0].K, True).view(np.int16)).to(dev) \
        .view(torch.bfloat16)
    ychain = [torch.empty((1, triple[j % 3].N), dtype=torch.bfloat16, device=dev) for j in range(n_mat)]
    calls = []
    for c0 in range(0, n_mat, per_call):
        probs = []
        for j in range(c0, c0 + per_call):
            L = triple[j % 3]
            p = dict(codes=mats[j // 3][j % 3][0], scales=mats[j // 3][j % 3][1], y=ychain[j], N=L.N, K=L.K)
            if j == c0:
                p["x"] = x0 if j == 0 else ychain[j - 1]
            else:
                p["x_from"] = j - 1 - c0
            probs.append(p)
        calls.append(probs)
    wsc = torch.empty(max(bt.gemv_batched_workspace_bytes(layout, pr) for pr in calls), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for pr in calls:
            bt.gemv_batched(pr, sign, layout, y_dtype=bt.BF16, ws=wsc)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for pr in calls:
                bt.gemv_batched(pr, sign, layout, y_dtype=bt.BF16, ws=wsc)
    ms = time_graphs([gr])
    out["M1"] = {"ms_per_token_step": round(ms, 3), "tokens_per_s": round(whole_job_rate(1, ms, world), 1),
                 "weight_GB/s": round(whole_job_rate(weight_bytes, ms, world) / 1e9, 1),
                 "chained": True, "calls_per_token": len(calls)}
    del gr, wsc, ychain

    # ---- M = 4, 16
    for M in (4, 16):
        g = workloads.rng(3 * 1_000_003 + 1000 + M)
        xs = [torch.from_numpy(workloads.activations_bf16_bits(g, M, L.K, True).view(np.int16)).to(dev)
              .view(torch.bfloat16) for L in triple]
        ys = [torch.empty((M, L.N), device=dev) for L in triple]
        ws = torch.empty(max(bt.gemv_workspace_bytes(layout, M, L.N, L.K) for L in triple), dtype=torch.uint8,
                         device=dev)
        graphs = []
        with torch.cuda.stream(stream):
            for i, L in enumerate(triple):
                bt.gemv(mats[0][i][0], mats[0][i][1], xs[i], sign, L.N, layout, out=ys[i], ws=ws)
            torch.cuda.synchronize()
            per_graph = 16
            for g0 in range(0, n_triples, per_graph):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    for t in range(g0, g0 + per_graph):
                        for i, L in enumerate(triple):
                            bt.gemv(mats[t][i][0], mats[t][i][1], xs[i], sign, L.N, layout, out=ys[i], ws=ws)
                graphs.append(gr)
        ms = time_graphs(graphs)
        out[f"M{M}"] = {"ms_per_token_step": round(ms, 3), "tokens_per_s": round(whole_job_rate(M, ms, world), 1),
                        "weight_GB/s": round(whole_job_rate(weight_bytes, ms, world) / 1e9, 1)}
        del graphs
    out["roofline_tokens_per_s_M1"] = round(_peaks()["hbm_gbs"] * 1e9 / weight_bytes, 1)
    out["M1_frac_of_roofline"] = round(out["M1"]["tokens_per_s"] / world / out["roofline_tokens_per_s_M1"], 4)
    del mats
    return out


# ---------------------------------------------------------------- CPU arm ---

def cpu_baseline(budget_s: float):
    """The FP64 oracle (rotation + dense dequantise + naive matmul) on host cores,
    on the decode triple: full passes (or a row sample of each matrix when one
    pass would exceed the budget), repeated until about `budget_s` seconds of
    CPU work; GB/s of packed weights."""
    import oracle
    import workloads
    oracle.build()
    inputs = [workloads.layer_inputs("C1", L, index=i) for i, L in enumerate(workloads.TRIPLE)]
    per_row = []
    for inp in inputs:
        xr = oracle.rotate_bf16(inp["x"], inp["sign"])
        t0 = time.perf_counter()
        oracle.gemv(inp["trits"][:32], inp["scales"][:32], xr)        # calibration
        per_row.append((time.perf_counter() - t0) / 32)
    rows = reference_rows(per_row, [L.N for L in workloads.TRIPLE], budget_s)
    t_total, b_total, passes = 0.0, 0, 0
    while t_total < budget_s or passes == 0:
        for inp, L, r in zip(inputs, workloads.TRIPLE, rows):
            t0 = time.perf_counter()
            xr = oracle.rotate_bf16(inp["x"], inp["sign"])
            oracle.gemv(inp["trits"][:r], inp["scales"][:r], xr)
            t_total += time.perf_counter() - t0
            b_total += _weight_bytes(workloads.Layer(L.name, L.K, r), 0)
        passes += 1
    sample = ("decode triple M=1 incl. rotation of x, rows per pass " +
              ", ".join(f"{L.name}:{r}/{L.N}" for L, r in zip(workloads.TRIPLE, rows)) +
              f", {passes} passes, {t_total:.1f} s")
    # the same oracle on one host thread, on a row sample of each matrix
    cores = oracle.threads()
    oracle.set_threads(1)
    try:
        r1 = [max(8, r // max(1, cores)) for r in rows]
        t1, b1 = 0.0, 0
        for inp, L, r in zip(inputs, workloads.TRIPLE, r1):
            t0 = time.perf_counter()
            xr = oracle.rotate_bf16(inp["x"], inp["sign"])
            oracle.gemv(inp["trits"][:r], inp["scales"][:r], xr)
            t1 += time.perf_counter() - t0
            b1 += _weight_bytes(workloads.Layer(L.name, L.K, r), 0)
    finally:
        oracle.set_threads(cores)
    return {"value": round(b_total / t_total / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "sample": sample, "cpu_model": _cpu_model(),
            "one_thread": {"value": round(b1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                           "sample": "rows per matrix " + ", ".join(f"{L.name}:{r}" for L, r in
                                                                   zip(workloads.TRIPLE, r1)) + f", {t1:.1f} s"}}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def reference_rows(per_row_s, Ns, step_budget_s):
    """Rows of each matrix one oracle step covers: the whole matrix when the
    step fits its time budget, else the same fraction of every matrix."""
    full = sum(p * n for p, n in zip(per_row_s, Ns))
    frac = min(1.0, step_budget_s / max(full, 1e-12))
    return [max(8, min(n, int(n * frac))) for n in Ns]


def run_reference(args):
    """The CPU oracle as the reference arm, on the same metric and workload:
    each step is the rotation of x plus the FP64 GEMV of a row sample of every
    matrix, sized so that warm-up plus timed steps take about `ref_seconds`."""
    import oracle
    import workloads
    oracle.build()
    triple = workloads.TRIPLE
    inputs = [workloads.layer_inputs("C1", L, index=i) for i, L in enumerate(triple)]
    per_row = []
    for inp in inputs:
        xr = oracle.rotate_bf16(inp["x"], inp["sign"])
        t0 = time.perf_counter()
        oracle.gemv(inp["trits"][:64], inp["scales"][:64], xr)
        per_row.append((time.perf_counter() - t0) / 64)
    rows = reference_rows(per_row, [L.N for L in triple], args.ref_seconds / (args.steps + args.warmup))

    def step():
        b = 0
        for inp, L, r in zip(inputs, triple, rows):
            xr = oracle.rotate_bf16(inp["x"], inp["sign"])
            oracle.gemv(inp["trits"][:r], inp["scales"][:r], xr)
            b += _weight_bytes(workloads.Layer(L.name, L.K, r), 0)
        return b
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    tot = 0
    for _ in range(args.steps):
        tot += step()
    dt = time.perf_counter() - t0
    v = tot / dt / 1e9
    sample = ("decode triple M=1 incl. rotation of x, rows per step " +
              ", ".join(f"{L.name}:{r}/{L.N}" for L, r in zip(triple, rows)))
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", 1)),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode GEMV M=1 on the 5120x5120 / 5120x17408 / 17408x5120 triple, base-3 g128, "
                               "FWHT-1024 fused", "M": 1},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample, "cpu_model": _cpu_model()},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "FP64 CPU oracle on rank 0's host cores; other ranks exit without work",
    }


def run_case(case: str, reps: int):
    """One small workload for a profiler capture (one kernel of interest, a few
    launches, a few GB on the device at most); prints one line and exits."""
    import torch
    import ternary_weight_fwht1024_b200 as bt
    import workloads
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sign = torch.from_numpy(workloads.sign1024()).to(dev)
    if case.startswith("gemv"):
        # gemv_m<M>_<layout>: the three decode layers at M rows, seeded C2 inputs
        M = int(case.split("_")[1][1:])
        layout = 1 if case.endswith("2bit") else 0
        for i, L in enumerate(workloads.TRIPLE):
            inp = workloads.layer_inputs("C2", L, M=M, index=i)
            codes = bt.pack(torch.from_numpy(inp["trits"]).to(dev), layout)
            sc = torch.from_numpy(inp["scales"].view(np.int16)).to(dev)
            x = torch.from_numpy(inp["x"].view(np.int16)).to(dev).view(torch.bfloat16)
            for _ in range(reps):
                bt.gemv(codes, sc, x, sign, L.N, layout)
    elif case.startswith("batched"):
        # batched[_2bit]: the decode triple in one bt_gemv_batched launch, seeded C1 inputs
        layout = 1 if case.endswith("2bit") else 0
        probs = []
        for i, L in enumerate(workloads.TRIPLE):
            inp = workloads.layer_inputs("C1", L, index=i)
            probs.append(dict(codes=bt.pack(torch.from_numpy(inp["trits"]).to(dev), layout),
                              scales=torch.from_numpy(inp["scales"].view(np.int16)).to(dev),
                              x=torch.from_numpy(inp["x"].view(np.int16)).to(dev).view(torch.bfloat16),
                              y=torch.empty((1, L.N), device=dev), N=L.N, K=L.K))
        for _ in range(reps):
            bt.gemv_batched(probs, sign, layout)
    elif case.startswith("gemm"):
        # gemm[_2bit]: pp512 on the 5120x5120 layer; gemm_triple[_2bit]: on
        # all three layers, one bt_gemm call each per rep
        layout = 1 if case.endswith("2bit") else 0
        idxs = range(len(workloads.TRIPLE)) if "triple" in case else [0]
        calls = []
        for i in idxs:
            L = workloads.TRIPLE[i]
            inp = workloads.layer_inputs("C3", L, M=512, index=i)
            calls.append((bt.pack(torch.from_numpy(inp["trits"]).to(dev), layout),
                          torch.from_numpy(inp["scales"].view(np.int16)).to(dev),
                          torch.from_numpy(inp["x"].view(np.int16)).to(dev).view(torch.bfloat16), L.N))
        for _ in range(reps):
            for codes, sc, x, n in calls:
                bt.gemm(codes, sc, x, sign, n, layout)
    elif case == "fwht":
        # 512 x 17408 (53 MB in + out) over distinct buffers: 10 of them exceed 4x L2
        g = workloads.rng(77)
        xs = [torch.from_numpy(workloads.activations_bf16_bits(g, 512, 17408, True).view(np.int16)).to(dev)
              .view(torch.bfloat16) for _ in range(10)]
        outs = [torch.empty((512, 17408), dtype=torch.float32, device=dev) for _ in range(10)]
        for r in range(reps):
            for x, o in zip(xs, outs):
                bt.fwht1024(x, sign, out=o)
    else:
        raise SystemExit(f"unknown case {case}")
    torch.cuda.synchronize()
    print(json.dumps({"case": case, "reps": reps, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="CPU time the reference arm spends over warm-up + timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 384-matrix 27B-equivalent sweep")
    ap.add_argument("--case", default=None,
                    help="run one small workload for a profiler capture (gemv_m<M>[_2bit], batched[_2bit], "
                         "gemm[_triple][_2bit], fwht)")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.case:
        run_case(args.case, args.reps)
        return
    args.warmup = max(3, args.warmup)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out = run_gpu(args, rank, world)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
