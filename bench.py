#!/usr/bin/env python
"""Benchmark of the selective scan (S6) forward on B200.

One step = one selective-scan forward pass (softplus, discretisation, scan,
readout, D skip, SiLU gate, final state) over one batch of the workload,
launched through the C ABI. Default workload: the long-context layer (batch 1,
d_inner 5120, N 16, L 131072, bf16 inputs, fp32 state), the largest
single-GPU configuration; the other layer shapes (Mamba-130M- and
Mamba-1.4B-shaped) are timed as legs of the same run, each with its own
roofline, beside the decode step, the convolution prologue, the trapezoidal
rule, the backward pass and the Mamba-2 SSD forward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the fp64 CPU oracle, timed on host cores)

Prints one JSON line on rank 0. Metric: scan elements (batch*dim*L*N) per
second, whole job (all ranks). Under torchrun every rank runs an independent
replica on its own batch (weak scaling, no data-path collective); the barrier
and the max-over-ranks reduction of the elapsed device time use NCCL.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_27_b200.inputs import (DECODE_WORKLOADS, SCAN_WORKLOADS,  # noqa: E402
                                                  make_decode_state, make_decode_step, make_scan_inputs)

METRIC = "selective-scan B·D·L·N elems/s at 1 B200; % of HBM/MUFU roofline"
UNIT = "elem/s"
L2_BYTES = 126 * 1024 * 1024
ROTATE = 3  # input sets cycled through so that each step reads inputs not resident in L2

# B200 unit counts for the arithmetic rooflines (per SM per clock): MUFU
# transcendental results 16, FP32 lanes 128.
SMS_B200 = 148
MUFU_PER_CLK = 16
# DRAM bytes (read + write) per launch from one ncu capture of the kernel and
# plan (scan: workload, plan configuration, CTAs) on that workload; profiles/
# holds the summaries. Any other kernel, plan or workload reports traffic null.
# The long-context layer was captured at 16,384 of its 131,072 steps (same rows,
# same plan): its traffic is proportional to the steps, so the capture is scaled
# by 8.
NCU_TRAFFIC = {("long_context_131k", 10, 148): (505176320 + 150065408) * 8,
               ("mamba130m_layer", 10, 296): 152307456 + 32844800,
               ("mamba1p4b_layer", 10, 444): 813864448 + 252678912,
               ("mamba2_layer_d2048", "ssd_kernel"): 565090000 + 247200000,
               ("decode_b256_d5120", "state_update_vec_kernel"): 92157440 + 29935104}
FP32_PER_CLK = 128
# FP32 operations of one exponential on the FMA pipe (the combined MUFU + FMA bound)
EXP_FMA_OPS = 8
# decode: layers whose states the timed steps cycle through (4 x 84 MB > L2),
# and the steps captured in one CUDA graph for that timing
DECODE_LAYERS = 4
# end-to-end leg: host-to-device copy streams (the large inputs go out in parallel)
E2E_COPY_STREAMS = 3
DECODE_GRAPH_STEPS = 40


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_context_131k", choices=sorted(SCAN_WORKLOADS))
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the headline workload's sequence length (0: the workload's own); used for "
                         "profiler captures of a shortened long-context layer")
    ap.add_argument("--leg-workloads", default="mamba130m_layer,mamba1p4b_layer",
                    help="other scan workloads timed as legs (comma separated; empty: none)")
    ap.add_argument("--leg-steps", type=int, default=50, help="timed steps of each scan-workload leg")
    ap.add_argument("--segments-leg", type=int, default=8,
                    help="also time the headline workload with this many forced time segments per row (0: skip)")
    ap.add_argument("--side-workload", default="mamba130m_layer", choices=sorted(SCAN_WORKLOADS),
                    help="workload of the convolution-prologue, trapezoidal and backward legs")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: seconds of oracle work for the whole warm-up + timed run")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU-baseline budget (seconds of oracle work on rank 0)")
    ap.add_argument("--prologue-steps", type=int, default=200,
                    help="steps of the scan with the fused convolution prologue (0 skips the leg)")
    ap.add_argument("--trap-steps", type=int, default=200,
                    help="steps of the exponential-trapezoidal scan (0 skips the leg)")
    ap.add_argument("--bwd-steps", type=int, default=20,
                    help="steps of the scan backward (0 skips the leg)")
    ap.add_argument("--ssd-steps", type=int, default=50,
                    help="steps of the Mamba-2 chunked SSD forward on its (4, 8192, 64 heads) layer (0 skips)")
    ap.add_argument("--decode-steps", type=int, default=1000,
                    help="decode state-update steps timed on the (256, 5120, 16) decode workload (0: skip)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------
# distributed plumbing

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, value: float, device=None) -> float:
        if not self.pg:
            return value
        import torch
        import torch.distributed as dist
        t = torch.tensor([value], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ----------------------------------------------------------------------------
# algorithmic counts (per scan pass)

def algorithmic_counts(w, in_bytes: int):
    """Bytes, MUFU and FP32 operations the scan needs, independent of the kernel.

    Bytes: u, delta, z read once; B, C read once; A, D, delta_bias read once;
    y written once; final state written once.
    MUFU: exp(delta A) per (b, d, t, n); softplus (exp + log) and the gate
    (exp + reciprocal) per (b, d, t).
    FP32: delta*A, delta*B*u, the state FMA and the readout FMA per element;
    about 8 per (b, d, t) for softplus, skip and gate.
    """
    rows_t = w.batch * w.dim * w.seqlen
    elems = rows_t * w.dstate
    n_in = 3 if w.has_z else 2
    bytes_ = (n_in * rows_t * in_bytes + 2 * w.batch * w.dstate * w.seqlen * in_bytes
              + w.dim * w.dstate * 4 + 2 * w.dim * 4
              + rows_t * in_bytes + w.batch * w.dim * w.dstate * 4)
    mufu = elems + rows_t * (2 + (2 if w.has_z else 0))
    fp32 = 4 * elems + 8 * rows_t
    return {"elements": elems, "bytes": bytes_, "mufu": mufu, "fp32": fp32}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "bf16_tflops": float(d.get("bf16_tflops", 1590.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw_slowdown": parts[5], "hw_thermal": parts[6],
                             "sw_thermal": parts[7], "sw_power_cap": parts[8]})
            except ValueError:
                continue
        if not rows:
            return None
        # keep samples at load (the timed region keeps the SMs busy)
        top = max(r["sm"] for r in rows)
        busy = [r for r in rows if r["power"] > 0.5 * max(r2["power"] for r2 in rows)] or rows
        reasons = set()
        for r in busy:
            for k in ("hw_slowdown", "hw_thermal", "sw_thermal", "sw_power_cap"):
                if r[k].lower() == "active":
                    reasons.add({"hw_thermal": "hw_thermal_slowdown",
                                 "sw_thermal": "sw_thermal_slowdown"}.get(k, k))
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": busy[0]["max"],
                "sm_mhz_peak_seen": top, "samples": len(busy),
                "power_w_median": statistics.median(r["power"] for r in busy),
                "reasons": sorted(reasons)}


def physical_gpu(local_rank: int) -> str:
    """nvidia-smi index (or UUID) of this rank's GPU."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ----------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of the workload

def cpu_rate(w, inp, seconds: float, rows_cap=None):
    """Time the fp64 oracle on a seeded sample of rows; returns (elem/s, threads, sample)."""
    import oracle
    threads = oracle.max_threads()
    total_rows = w.batch * w.dim
    g = np.random.default_rng(12345)
    n = min(total_rows, max(threads, 32))
    t = time.perf_counter()
    oracle.scan(**_oracle_kw(inp), rows=np.sort(g.choice(total_rows, n, replace=False)))
    dt = time.perf_counter() - t
    per_row = dt / n
    n = int(min(total_rows, max(n, seconds / max(per_row, 1e-9))))
    if rows_cap:
        n = min(n, rows_cap)
    rows = np.sort(g.choice(total_rows, n, replace=False))
    t = time.perf_counter()
    oracle.scan(**_oracle_kw(inp), rows=rows)
    dt = time.perf_counter() - t
    elems = n * w.seqlen * w.dstate
    return elems / dt, threads, f"{n} of {total_rows} rows (seeded), full L={w.seqlen}, N={w.dstate}", dt


def _oracle_kw(inp):
    return dict(u=inp["u"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"],
                z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True, dtype=inp["dtype"])


# ----------------------------------------------------------------------------

def workload_config(w, extra=None):
    cfg = {"workload": w.name, "batch": w.batch, "d_inner": w.dim, "d_state": w.dstate,
           "seq_len": w.seqlen, "in_dtype": w.dtype, "state_dtype": "f32", "gate": w.has_z,
           "l2": l2_note(w), "parallelism": "replicas (independent batch per GPU)"}
    if extra:
        cfg.update(extra)
    return cfg


def run_reference(args, dist: Dist):
    """The fp64 CPU oracle as the reference arm: rank 0 only."""
    if dist.rank != 0:
        return 0
    import oracle
    w = SCAN_WORKLOADS[args.workload]
    inp = make_scan_inputs(w)
    threads = oracle.max_threads()
    total_rows = w.batch * w.dim
    # size each step so the whole warm-up + timed run takes about --ref-seconds
    rate, _, _, _ = cpu_rate(w, inp, min(1.0, args.ref_seconds), rows_cap=4096)
    per_step_budget = args.ref_seconds / max(1, args.steps + args.warmup)
    n = int(max(1, min(total_rows, per_step_budget * rate / (w.seqlen * w.dstate))))
    g = np.random.default_rng(777)
    samples = [np.sort(g.choice(total_rows, n, replace=False)) for _ in range(4)]
    kw = _oracle_kw(inp)
    for s in range(args.warmup):
        oracle.scan(**kw, rows=samples[s % 4])
    t = time.perf_counter()
    for s in range(args.steps):
        oracle.scan(**kw, rows=samples[s % 4])
    dt = time.perf_counter() - t
    elems = args.steps * n * w.seqlen * w.dstate
    value = elems / dt
    sample = f"{n} of {total_rows} rows per step (seeded), full L={w.seqlen}, N={w.dstate}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": workload_config(w, {"l2": l2_note(w)}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rotate_count(w) -> int:
    """Input sets cycled through so that every step reads inputs that are not
    resident in L2: one set when a set alone is several times the L2."""
    in_bytes = 4 if w.dtype == "f32" else 2
    set_bytes = (3 if w.has_z else 2) * w.batch * w.dim * w.seqlen * in_bytes
    return 1 if set_bytes > 4 * L2_BYTES else ROTATE


def l2_note(w) -> str:
    n = rotate_count(w)
    return ("inputs larger than L2 (one set)" if n == 1 else
            f"inputs rotated over {n} resident copies (> L2 of 126 MB)")


class ScanSetup:
    """Seeded inputs of one scan workload on the device, the C-ABI argument
    structs of its rotating input sets, the workspace and the launch plan."""

    def __init__(self, w, dev, rank, pin=False, force_segments=0):
        import torch
        import selective_state_space_27_b200 as ms
        self.w = w
        self.force_segments = force_segments
        self.in_bytes = 4 if w.dtype == "f32" else 2
        self.tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        self.inp = make_scan_inputs(w, seed=w.seed + 1000 * rank)

        def host(a):
            t = torch.from_numpy(np.ascontiguousarray(a))
            return t.view(torch.bfloat16) if (a.dtype == np.uint16) else t

        self.names = ["u", "delta", "B", "C"] + (["z"] if w.has_z else [])
        src = {k: host(self.inp[k]) for k in self.names}
        self.pinned = {k: v.pin_memory() for k, v in src.items()} if pin else None
        self.params = {k: torch.from_numpy(self.inp[k]).to(dev) for k in ("A", "D", "delta_bias")}
        self.rotate = rotate_count(w)
        self.sets = [{k: v.to(dev) for k, v in (self.pinned or src).items()} for _ in range(self.rotate)]
        self.y = torch.empty((w.batch, w.dim, w.seqlen), dtype=self.tdt, device=dev)
        self.hT = torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
        self.args = [self.scan_args(st, self.y, self.hT) for st in self.sets]
        self.plan = ms.scan_plan(self.args[0])
        self.ws = torch.empty(max(ms.scan_workspace_size(self.args[0]), 256), dtype=torch.uint8, device=dev)
        kind = {c: k for c, _, _, _, k in ms.scan_configs()}[self.plan.config]
        self.kernel = (f"rec_kernel<{'bf16' if w.dtype == 'bf16' else 'f32'}, {self.plan.lanes}>" if kind == 1
                       else "scan_kernel")
        self.kernel_desc = (
            f"{self.kernel} (sequential, warp-specialised, {self.plan.lanes} lanes per row, "
            f"{self.plan.warps_per_cta - 4} I/O warps, config {self.plan.config}, "
            + (f"persistent schedule over {self.plan.ctas} CTAs)" if self.plan.ctas else "one CTA per block of rows)")
            if kind == 1 else
            f"scan_kernel (chunked, config {self.plan.config}, {self.plan.warps_per_cta} warps, "
            f"{self.plan.segments} segments)")
        self.launches_per_step = 2 if (kind == 0 and self.plan.segments > 1) else 1
        self.counts = algorithmic_counts(w, self.in_bytes)
        torch.cuda.synchronize()

    def scan_args(self, st, y, hT):
        import selective_state_space_27_b200 as ms
        return ms.build_scan_args(st["u"], st["delta"], self.params["A"], st["B"], st["C"], y, D=self.params["D"],
                                  z=st.get("z"), delta_bias=self.params["delta_bias"], final_state=hT,
                                  force_segments=self.force_segments)

    def step(self, lib, i, stream, args=None):
        import ctypes
        import selective_state_space_27_b200 as ms
        a = args if args is not None else self.args[i % self.rotate]
        rc = lib.mamba_scan_fwd(ctypes.byref(a), self.ws.data_ptr(), self.ws.numel(), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())


def time_steps(fn, n, stream):
    """CUDA-event time (ms) of n calls of fn() on `stream`, synchronized on both sides."""
    import torch
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def scan_roofline(setup, us, mufu, peaks):
    """Roofline of one scan launch: the binding bound is the MUFU (one ex2 per
    element + the softplus and gate transcendentals per (b, d, t)), against the
    MUFU throughput measured on this device; HBM and FP32 fractions beside."""
    c = setup.counts
    t = us * 1e-6
    fp32_peak = SMS_B200 * FP32_PER_CLK * peaks["sm_max_mhz"] * 1e6
    t_bounds = {"hbm": c["bytes"] / (peaks["hbm_gbs"] * 1e9), "mufu": c["mufu"] / mufu["measured_per_s"],
                "fp32": c["fp32"] / fp32_peak}
    # The combined bound: a share a of the MUFU operations evaluated on the FMA
    # pipe instead (2^x by argument reduction and a degree-5 polynomial, about
    # EXP_FMA_OPS FP32 operations each), chosen so that both pipes finish
    # together. The measured offload was slower (the kernels are bound by issue
    # slots and latency), so the MUFU-only bound stays the roofline; this one
    # is reported beside it.
    e_t, f_t = t_bounds["mufu"], t_bounds["fp32"]
    k_t = c["mufu"] * EXP_FMA_OPS / fp32_peak
    share = max(0.0, (e_t - f_t) / (e_t + k_t))
    t_comb = max((1.0 - share) * e_t, f_t + share * k_t)
    return {
        "bound": "alu", "unit": "Tmufu/s", "achieved": c["mufu"] / t / 1e12, "peak": mufu["measured_per_s"] / 1e12,
        "frac": c["mufu"] / t / mufu["measured_per_s"],
        "traffic": NCU_TRAFFIC.get((setup.w.name, setup.plan.config, setup.plan.ctas)),
        "kernel": setup.kernel_desc,
        "peak_note": (f"measured: ex2.approx throughput of this device ({mufu['measured_per_clk_per_sm']:.2f} per clk "
                      f"per SM, mamba_probe_unit_throughput); nominal {SMS_B200} SMs x {MUFU_PER_CLK}/clk x "
                      f"{peaks['sm_max_mhz']:.0f} MHz = {mufu['nominal_per_s'] / 1e12:.3f} T/s"),
        "frac_of_nominal": c["mufu"] / t / mufu["nominal_per_s"],
        "algorithmic_per_launch": c,
        "hbm": {"achieved_gbs": c["bytes"] / t / 1e9, "peak_gbs": peaks["hbm_gbs"],
                "frac": c["bytes"] / t / 1e9 / peaks["hbm_gbs"], "peak_source": peaks["source"]},
        "bound_times_us": {k: v * 1e6 for k, v in t_bounds.items()},
        "mufu_plus_fma": {"bound_us": t_comb * 1e6, "frac": t_comb / t, "fma_share_of_exponentials": share,
                          "fp32_ops_per_exponential": EXP_FMA_OPS},
        "kernel_us": us,
        "roofline_elem_per_s": c["elements"] / max(t_bounds.values()),
    }


def measure_mufu(peaks):
    import selective_state_space_27_b200 as ms
    per_s, per_clk = ms.probe_unit_throughput("ex2")
    tanh_s, _ = ms.probe_unit_throughput("tanh")
    return {"measured_per_s": per_s, "measured_per_clk_per_sm": per_clk, "tanh_per_s": tanh_s,
            "nominal_per_s": SMS_B200 * MUFU_PER_CLK * peaks["sm_max_mhz"] * 1e6}


def run_scan_leg(args, dist, dev, w, mufu, peaks, lib, stream, force_segments=0):
    """Time another scan workload through mamba_scan_fwd: its own plan,
    rotating input sets when they fit in L2, and roofline. With
    force_segments > 1 the call forces that many time segments per row (the
    chunked kernels' multi-block carry), timed against the same algorithmic
    bound."""
    setup = ScanSetup(w, dev, dist.rank, force_segments=force_segments)
    for i in range(max(3, args.warmup)):
        setup.step(lib, i, stream)
    n = args.leg_steps
    ms_ = dist.max(time_steps(lambda i: setup.step(lib, i, stream), n, stream), dev)
    us = ms_ * 1e3 / n
    cfg = {"l2": l2_note(w)}
    if force_segments:
        cfg["force_segments"] = force_segments
    out = {"workload": w.name, "config": workload_config(w, cfg), "steps": n, "us_per_step": us,
           "value": dist.world * setup.counts["elements"] / (us * 1e-6), "unit": UNIT,
           "roofline": scan_roofline(setup, us, mufu, peaks), "gpu_launches": n * setup.launches_per_step}
    del setup
    return out


def run_e2e(args, dist, dev, setup, lib, stream):
    """The same step end to end through the C ABI from pinned host buffers:
    every step copies its inputs host -> device and y and the final state
    device -> host. Steps are pipelined over two device buffer sets on three
    streams (copy in, compute, copy out), so the copy-in of step i+1, the
    scan of step i and the copy-out of step i-1 overlap; the timed region runs
    from the first copy-in to the last copy-out."""
    import torch
    w = setup.w
    s_ins = [torch.cuda.Stream(dev) for _ in range(E2E_COPY_STREAMS)]   # one copy-in stream per large input
    s_in, s_out = s_ins[0], torch.cuda.Stream(dev)
    bufs = [setup.sets[0], {k: torch.empty_like(v) for k, v in setup.sets[0].items()}]
    ys = [setup.y, torch.empty_like(setup.y)]
    hs = [setup.hT, torch.empty_like(setup.hT)]
    argl = [setup.scan_args(bufs[j], ys[j], hs[j]) for j in range(2)]
    y_host = torch.empty(setup.y.shape, dtype=setup.tdt).pin_memory()
    h_host = torch.empty(setup.hT.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in setup.pinned.values())
    # the inputs, largest first, dealt round-robin over the copy-in streams
    in_names = sorted(setup.pinned, key=lambda k: -setup.pinned[k].numel() * setup.pinned[k].element_size())
    d2h = y_host.numel() * y_host.element_size() + h_host.numel() * 4

    def run(n):
        ev_in = [[torch.cuda.Event() for _ in s_ins] for _ in range(n)]
        ev_cmp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for cs in s_ins[1:]:
            cs.wait_event(t0)
        for i in range(n):
            j = i % 2
            for m, cs in enumerate(s_ins):
                with torch.cuda.stream(cs):
                    if i >= 2:
                        cs.wait_event(ev_cmp[i - 2])    # the scan of step i-2 has read buffer j
                    for k in in_names[m::len(s_ins)]:
                        bufs[j][k].copy_(setup.pinned[k], non_blocking=True)
                    ev_in[i][m].record(cs)
            for e in ev_in[i]:
                stream.wait_event(e)
            if i >= 2:
                stream.wait_event(ev_out[i - 2])        # step i-2's outputs have left buffer j
            setup.step(lib, 0, stream, args=argl[j])
            ev_cmp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                y_host.copy_(ys[j], non_blocking=True)
                h_host.copy_(hs[j], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    run(2)
    dist.barrier()
    n = args.e2e_steps
    e2e_ms = dist.max(run(n), dev)
    return {"value": setup.counts["elements"] * n * dist.world / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / n,
            "pipeline": (f"copy-in ({E2E_COPY_STREAMS} streams), scan and copy-out of consecutive steps overlap "
                         "(2 buffer sets)")}


def cpu_single_core(w_name, seconds):
    """The oracle on one host core over a seeded sample of rows of `w_name`."""
    import oracle
    w = SCAN_WORKLOADS[w_name]
    inp = make_scan_inputs(w)
    total_rows = w.batch * w.dim
    g = np.random.default_rng(4321)
    t = time.perf_counter()
    oracle.scan(**_oracle_kw(inp), rows=np.sort(g.choice(total_rows, 4, replace=False)), threads=1)
    per_row = (time.perf_counter() - t) / 4
    n = int(min(total_rows, max(4, seconds / max(per_row, 1e-9))))
    rows = np.sort(g.choice(total_rows, n, replace=False))
    t = time.perf_counter()
    oracle.scan(**_oracle_kw(inp), rows=rows, threads=1)
    dt = time.perf_counter() - t
    return {"workload": w_name, "value": n * w.seqlen * w.dstate / dt, "unit": UNIT, "cores": 1,
            "sample": f"{n} of {total_rows} rows (seeded), full L={w.seqlen}, N={w.dstate}", "seconds": dt}


def run_ours(args, dist: Dist):
    import torch
    import selective_state_space_27_b200 as ms

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the product path has no CPU fallback)")
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    w = SCAN_WORKLOADS[args.workload]
    if args.seqlen:
        w = dataclasses.replace(w, seqlen=args.seqlen)
    peaks = load_peaks()
    mufu = measure_mufu(peaks)
    lib = ms.load_library()
    stream = torch.cuda.current_stream()
    setup = ScanSetup(w, dev, dist.rank, pin=args.e2e_steps > 0)

    for i in range(args.warmup):
        setup.step(lib, i, stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(physical_gpu(dist.local_rank))
    if dist.rank == 0:
        sampler.start()
    dist.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    sampler.mark_begin()
    ev[0].record(stream)
    for i in range(args.steps):
        setup.step(lib, i, stream)
    ev[1].record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    dist.barrier()
    elapsed_ms = ev[0].elapsed_time(ev[1])
    clocks = sampler.stop() if dist.rank == 0 else None
    elapsed_ms = dist.max(elapsed_ms, dev)
    if setup.plan.ctas and ms.scan_status(setup.ws) != 0:
        raise SystemExit("bench.py: a persistent scan reported a failed carry wait")

    counts = setup.counts
    total_elems = counts["elements"] * args.steps * dist.world
    value = total_elems / (elapsed_ms / 1e3)
    ms_per_step = elapsed_ms / args.steps
    roofline = scan_roofline(setup, ms_per_step * 1e3, mufu, peaks)

    e2e = run_e2e(args, dist, dev, setup, lib, stream) if args.e2e_steps > 0 else None
    launches = args.steps * setup.launches_per_step
    del setup
    torch.cuda.empty_cache()

    legs = {}
    for name in [s for s in args.leg_workloads.split(",") if s]:
        if name != w.name:
            legs[name] = run_scan_leg(args, dist, dev, SCAN_WORKLOADS[name], mufu, peaks, lib, stream)
            torch.cuda.empty_cache()

    segmented = None
    if args.segments_leg > 1:
        segmented = run_scan_leg(args, dist, dev, w, mufu, peaks, lib, stream, force_segments=args.segments_leg)
        torch.cuda.empty_cache()

    decode = run_decode(args, dist, dev) if args.decode_steps > 0 else None
    side = None
    if args.prologue_steps > 0 or args.trap_steps > 0 or args.bwd_steps > 0:
        side = ScanSetup(SCAN_WORKLOADS[args.side_workload], dev, dist.rank)
    mufu_peak = mufu["measured_per_s"]
    prologue = (run_prologue(args, dist, dev, side.w, side.sets, side.params, side.y, side.hT, side.counts, mufu_peak)
                if args.prologue_steps > 0 else None)
    trap = (run_trap(args, dist, dev, side.w, side.sets, side.params, side.y, side.hT, side.counts, mufu_peak)
            if args.trap_steps > 0 else None)
    bwd = run_bwd(args, dist, dev, side.w, side.sets, side.params, side.counts, mufu_peak) if args.bwd_steps > 0 else None
    del side
    torch.cuda.empty_cache()
    ssd = run_ssd(args, dist, dev, peaks) if args.ssd_steps > 0 else None

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        rate, threads, sample, secs = cpu_rate(w, make_scan_inputs(w), args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
               "seconds": secs, "single_core": cpu_single_core("mamba130m_layer", min(5.0, args.cpu_seconds))}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded)", "config": workload_config(w, {"l2": l2_note(w)}),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "mufu_probe": mufu, "scan_legs": legs,
        "segmented": segmented,
        "decode": decode, "conv_prologue": prologue, "trapezoidal": trap, "backward": bwd, "ssd": ssd,
        "gpu_launches": launches, "clocks": clocks,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.close()
    return 0


def run_prologue(args, dist: Dist, dev, w, sets, params, y, hT, counts, mufu_peak):
    """Time the scan with the causal depthwise convolution + SiLU prologue
    fused in front (width 4, seeded taps): the same workload and rotating input
    sets as the headline step, with u read as the convolution input x."""
    import ctypes

    import torch
    import selective_state_space_27_b200 as ms
    from selective_state_space_27_b200.inputs import make_conv_params

    conv_np = make_conv_params(w.dim, 4, seed=w.seed + 77)
    conv_t = {k: torch.from_numpy(v).to(dev) for k, v in conv_np.items()}
    conv = ms.build_conv_args(conv_t["conv_w"], conv_t["conv_b"], True)
    argl = [ms.build_scan_args(s["u"], s["delta"], params["A"], s["B"], s["C"], y, D=params["D"], z=s.get("z"),
                               delta_bias=params["delta_bias"], final_state=hT) for s in sets]
    lib = ms.load_library()
    stream = torch.cuda.current_stream()
    nbytes = ctypes.c_size_t(0)
    rc = lib.mamba_conv_scan_workspace_size(ctypes.byref(argl[0]), ctypes.byref(conv), None, ctypes.byref(nbytes))
    if rc != 0:
        raise ms.MambaScanError(rc, lib.mamba_last_error().decode())
    workspace = torch.empty(max(1, nbytes.value), dtype=torch.uint8, device=dev)

    def step(i):
        rc = lib.mamba_conv_scan_fwd_ws(ctypes.byref(argl[i % len(argl)]), ctypes.byref(conv), None,
                                        workspace.data_ptr() if nbytes.value else None, nbytes.value,
                                        stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    n = args.prologue_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max(e0.elapsed_time(e1) * 1e3 / n, dev)
    rows_t = w.batch * w.dim * w.seqlen
    mufu = counts["mufu"] + 2 * rows_t          # + exp and reciprocal of the prologue's SiLU
    return {
        "workload": w.name, "width": 4, "silu": True, "steps": n,
        "metric": "conv prologue + selective scan B*D*L*N elems/s", "unit": UNIT,
        "value": dist.world * counts["elements"] / (us * 1e-6), "us_per_step": us,
        "roofline": {"bound": "alu", "unit": "Tmufu/s", "achieved": mufu / (us * 1e-6) / 1e12,
                     "peak": mufu_peak / 1e12, "frac": mufu / (us * 1e-6) / mufu_peak,
                     "algorithmic_mufu": mufu,
                     "note": "bytes as the plain scan (x replaces u); the convolution adds 4 FMA per (b, d, t)"},
        "gpu_launches": n,
    }


def run_trap(args, dist: Dist, dev, w, sets, params, y, hT, counts, mufu_peak):
    """Time the exponential-trapezoidal scan (Mamba-3) on the headline workload
    and input sets, with a seeded lambda_raw ~ N(0, 1) per (b, d, t)."""
    import ctypes

    import torch
    import selective_state_space_27_b200 as ms
    from selective_state_space_27_b200.inputs import make_lambda_raw

    lam_np = make_lambda_raw(w.batch, w.dim, w.seqlen, w.dtype, seed=w.seed + 1000 * dist.rank + 91)
    lam = torch.from_numpy(lam_np)
    lam = (lam.view(torch.bfloat16) if w.dtype == "bf16" else lam).to(dev)
    argl = [ms.build_scan_args(s["u"], s["delta"], params["A"], s["B"], s["C"], y, D=params["D"], z=s.get("z"),
                               delta_bias=params["delta_bias"], final_state=hT) for s in sets]
    lib = ms.load_library()
    stream = torch.cuda.current_stream()
    lam_args = (lam.data_ptr(), lam.stride(0), lam.stride(1))
    nbytes = ctypes.c_size_t(0)
    rc = lib.mamba_trap_scan_workspace_size(ctypes.byref(argl[0]), *lam_args, None, ctypes.byref(nbytes))
    if rc != 0:
        raise ms.MambaScanError(rc, lib.mamba_last_error().decode())
    workspace = torch.empty(max(1, nbytes.value), dtype=torch.uint8, device=dev)

    def step(i):
        rc = lib.mamba_trap_scan_fwd_ws(ctypes.byref(argl[i % len(argl)]), *lam_args, None,
                                        workspace.data_ptr() if nbytes.value else None, nbytes.value,
                                        stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    n = args.trap_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max(e0.elapsed_time(e1) * 1e3 / n, dev)
    mufu = counts["mufu"] + 2 * w.batch * w.dim * w.seqlen      # + exp and reciprocal of lambda's sigmoid
    return {
        "workload": w.name, "steps": n, "metric": "trapezoidal selective scan B*D*L*N elems/s", "unit": UNIT,
        "value": dist.world * counts["elements"] / (us * 1e-6), "us_per_step": us,
        "roofline": {"bound": "alu", "unit": "Tmufu/s", "achieved": mufu / (us * 1e-6) / 1e12,
                     "peak": mufu_peak / 1e12, "frac": mufu / (us * 1e-6) / mufu_peak, "algorithmic_mufu": mufu,
                     "note": "bytes as the plain scan + lambda_raw read once"},
        "gpu_launches": n,
    }


def run_bwd(args, dist: Dist, dev, w, sets, params, counts, mufu_peak):
    """Time the scan backward (gradients for a seeded dy, recomputing the
    states from 8-step checkpoints) on the side workload, through the C ABI
    with preallocated outputs and workspace."""
    import ctypes

    import torch
    import selective_state_space_27_b200 as ms
    from selective_state_space_27_b200.inputs import bf16_bits_from_f32

    g = np.random.default_rng(w.seed + 1000 * dist.rank + 5)
    dy_np = g.normal(size=(w.batch, w.dim, w.seqlen)).astype(np.float32)
    dy = torch.from_numpy(dy_np if w.dtype == "f32" else bf16_bits_from_f32(dy_np))
    dy = (dy.view(torch.bfloat16) if w.dtype == "bf16" else dy).to(dev)
    s0 = sets[0]
    args0 = ms.build_scan_args(s0["u"], s0["delta"], params["A"], s0["B"], s0["C"], s0["u"], D=params["D"],
                               z=s0.get("z"), delta_bias=params["delta_bias"])
    f32 = dict(device=dev, dtype=torch.float32)
    outs = {"du": torch.empty_like(s0["u"]), "ddelta": torch.empty_like(s0["u"]),
            "dz": torch.empty_like(s0["u"]) if w.has_z else None, "dA": torch.empty((w.dim, w.dstate), **f32),
            "dB": torch.empty((w.batch, w.dstate, w.seqlen), **f32),
            "dC": torch.empty((w.batch, w.dstate, w.seqlen), **f32), "dD": torch.empty(w.dim, **f32),
            "ddelta_bias": torch.empty(w.dim, **f32)}
    gb = ms.ScanBwdArgs()
    gb.dy, gb.dy_batch_stride, gb.dy_dim_stride = dy.data_ptr(), dy.stride(0), dy.stride(1)
    for k in ("du", "ddelta", "dz"):
        if outs[k] is not None:
            setattr(gb, k, outs[k].data_ptr())
            setattr(gb, f"{k}_batch_stride", outs[k].stride(0))
            setattr(gb, f"{k}_dim_stride", outs[k].stride(1))
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        setattr(gb, k, outs[k].data_ptr())
    lib = ms.load_library()
    n_ws = ctypes.c_size_t(0)
    lib.mamba_scan_bwd_workspace_size(ctypes.byref(args0), ctypes.byref(n_ws))
    ws = torch.empty(max(n_ws.value, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        rc = lib.mamba_scan_bwd(ctypes.byref(args0), ctypes.byref(gb), ws.data_ptr(), ws.numel(), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n = args.bwd_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max(e0.elapsed_time(e1) * 1e3 / n, dev)

    # The training pair: the forward keeps the states of every 8th step
    # (mamba_scan_fwd_checkpointed) and the backward recomputes from them
    # (mamba_scan_bwd_checkpointed) instead of sweeping the sequence first.
    y_buf = torch.empty_like(s0["u"])
    hT_buf = torch.empty((w.batch, w.dim, w.dstate), **f32)
    fargs = ms.build_scan_args(s0["u"], s0["delta"], params["A"], s0["B"], s0["C"], y_buf, D=params["D"],
                               z=s0.get("z"), delta_bias=params["delta_bias"], final_state=hT_buf)
    ck = torch.empty(max(n_ws.value // 4, 64), dtype=torch.float32, device=dev)
    fws = torch.empty(max(ms.scan_workspace_size(fargs), 256), dtype=torch.uint8, device=dev)

    def fwd_plain():
        rc = lib.mamba_scan_fwd(ctypes.byref(fargs), fws.data_ptr(), fws.numel(), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    def fwd_ck():
        rc = lib.mamba_scan_fwd_checkpointed(ctypes.byref(fargs), ck.data_ptr(), ck.numel() * 4, fws.data_ptr(),
                                             fws.numel(), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    def bwd_ck():
        rc = lib.mamba_scan_bwd_checkpointed(ctypes.byref(args0), ctypes.byref(gb), ck.data_ptr(), ck.numel() * 4,
                                             stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return dist.max(e0.elapsed_time(e1) * 1e3 / n, dev)

    fwd_ck()
    fwd_plain_us, fwd_ck_us, bwd_ck_us = timed(fwd_plain), timed(fwd_ck), timed(bwd_ck)
    rows_t = w.batch * w.dim * w.seqlen
    mufu = 2 * counts["elements"] + 6 * rows_t   # forward sweep + recompute ex2 per element; softplus, gates per (b,d,t)
    mufu_ck = counts["elements"] + 6 * rows_t     # the recompute only
    return {
        "workload": w.name, "steps": n, "metric": "scan backward B*D*L*N elems/s", "unit": UNIT,
        "value": dist.world * counts["elements"] / (us * 1e-6), "us_per_step": us,
        "roofline": {"bound": "alu", "unit": "Tmufu/s", "achieved": mufu / (us * 1e-6) / 1e12,
                     "peak": mufu_peak / 1e12, "frac": mufu / (us * 1e-6) / mufu_peak, "algorithmic_mufu": mufu,
                     "note": "two ex2 per element: the checkpoint sweep and the per-chunk recomputation"},
        "checkpointed": {
            "note": "forward with 8-step checkpoints (mamba_scan_fwd_checkpointed), backward from them "
                    "(mamba_scan_bwd_checkpointed)",
            "fwd_plain_us": fwd_plain_us, "fwd_checkpointed_us": fwd_ck_us, "bwd_us": bwd_ck_us,
            "pair_us": fwd_ck_us + bwd_ck_us, "pair_without_checkpoints_us": fwd_plain_us + us,
            "bwd_roofline": {"bound": "alu", "unit": "Tmufu/s", "achieved": mufu_ck / (bwd_ck_us * 1e-6) / 1e12,
                             "peak": mufu_peak / 1e12, "frac": mufu_ck / (bwd_ck_us * 1e-6) / mufu_peak,
                             "algorithmic_mufu": mufu_ck,
                             "note": "one ex2 per element (the recomputation) plus the per-(b,d,t) terms"},
        },
        "gpu_launches": 6 * n + 3 * (n + 3) + 1,
    }


def ssd_counts(w, chunk=128):
    """Algorithmic work of one SSD forward pass.

    Bytes: x, z and dt read once, B and C read once, y written once, the
    final state written once, A, D and dt_bias read once. Tensor FLOPs of the
    chunked form per (token, head): 2 Q N for C B^T, 2 Q P for the masked
    product with X, and 2 N P each for the chunk state and the state readout.
    """
    tok = w.batch * w.seqlen
    th = tok * w.nheads
    bytes_ = (th * w.headdim * 2 * (3 if w.has_z else 2) + th * 2 + 2 * tok * w.ngroups * w.dstate * 2
              + 3 * w.nheads * 4 + w.batch * w.nheads * w.headdim * w.dstate * 4)
    flops = th * (2 * chunk * w.dstate + 2 * chunk * w.headdim + 4 * w.dstate * w.headdim)
    return {"elements": w.elements, "bytes": bytes_, "tensor_flops": flops}


def run_ssd(args, dist: Dist, dev, peaks):
    """Time the Mamba-2 chunked SSD forward (tcgen05 kernel) on the page's
    layer: batch 4, 8192 tokens, 64 heads of 64 channels, d_state 128, one
    group, bf16, with gate. Its inputs (about 560 MB) exceed the L2."""
    import ctypes

    import torch
    import selective_state_space_27_b200 as ms
    from selective_state_space_27_b200.inputs import SSD_WORKLOADS, make_ssd_inputs

    w = SSD_WORKLOADS["mamba2_layer_d2048"]
    inp = make_ssd_inputs(w, seed=w.seed + 1000 * dist.rank)

    def dev_t(a, bf16):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if bf16 else t).to(dev)

    t = {k: dev_t(inp[k], True) for k in ("x", "dt", "B", "C", "z")}
    prm = {k: dev_t(inp[k], False) for k in ("A", "D", "dt_bias")}
    y = torch.empty_like(t["x"])
    hT = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=dev)
    a = ms.build_ssd_args(t["x"], t["dt"], prm["A"], t["B"], t["C"], y, D=prm["D"], z=t["z"],
                          dt_bias=prm["dt_bias"], final_state=hT)
    lib = ms.load_library()
    stream = torch.cuda.current_stream()
    nbytes = ctypes.c_size_t(0)
    rc = lib.mamba_ssd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes))
    if rc != 0:
        raise ms.MambaScanError(rc, lib.mamba_last_error().decode())
    status = torch.zeros(nbytes.value, dtype=torch.uint8, device=dev)   # status word (+ hand-over slots)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    schedule = (f"persistent: {sms} CTAs over {w.batch * w.nheads} (batch, head) sequences"
                if nbytes.value > ms.SSD_WORKSPACE_BYTES else "one CTA per (batch, head)")

    def step():
        rc = lib.mamba_ssd_fwd(ctypes.byref(a), status.data_ptr(), status.numel(), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    n = args.ssd_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms.ssd_check(status)
    us = dist.max(e0.elapsed_time(e1) * 1e3 / n, dev)
    c = ssd_counts(w)
    gbs = c["bytes"] / (us * 1e-6) / 1e9
    tflops = c["tensor_flops"] / (us * 1e-6) / 1e12
    return {
        "workload": w.name, "steps": n, "metric": "Mamba-2 SSD forward B*L*H*P*N state elems/s", "unit": UNIT,
        "value": dist.world * c["elements"] / (us * 1e-6), "us_per_step": us,
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": 128, "dtype": "bf16",
                   "l2": "inputs larger than L2", "schedule": schedule},
        "roofline": {"bound": "hbm", "unit": "GB/s", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "frac": gbs / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC.get((w.name, "ssd_kernel")),
                     "peak_source": peaks["source"], "algorithmic_per_launch": c,
                     "tensor": {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
                                "frac": tflops / peaks["bf16_tflops"]},
                     "bound_times_us": {"hbm": c["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6,
                                        "tensor": c["tensor_flops"] / (peaks["bf16_tflops"] * 1e12) * 1e6}},
        "gpu_launches": n,
    }


def run_decode(args, dist: Dist, dev):
    """Time the single-token state update on the decode workload (batch 256,
    d_inner 5120, N 16, fp32 state, bf16 tokens): ``--decode-steps``
    sequential steps cycling over 8 pre-uploaded seeded token sets, launched
    through the C ABI. Three timings:
    - layers cycled (the roofline's): each step updates the state of the next
      of DECODE_LAYERS layers (4 x 84 MB, more than the 126 MB L2), so every
      step reads a state that is not in L2 and the previous step's writes
      leave L2 during it, as when a token passes through a model's layers;
    - back to back on one state, which then stays in L2 (one layer alone);
    - one state behind a 256 MB write between steps (the write is outside the
      per-step events, but its dirty lines are written back during the step)."""
    import ctypes

    import torch
    import selective_state_space_27_b200 as ms

    w = DECODE_WORKLOADS["decode_b256_d5120"]
    st0 = make_decode_state(w, seed=w.seed + 1000 * dist.rank)
    states = [torch.from_numpy(st0["h0"]).to(dev) for _ in range(DECODE_LAYERS)]
    prm = {k: torch.from_numpy(st0[k]).to(dev) for k in ("A", "D", "delta_bias")}
    toks = []
    for s in range(8):
        t = make_decode_step(w, s, seed=w.seed + 1000 * dist.rank)
        toks.append({k: torch.from_numpy(v).view(torch.bfloat16).to(dev) for k, v in t.items()})
    y = torch.empty((w.batch, w.dim), dtype=torch.bfloat16, device=dev)
    argl = [[ms.build_update_args(st, t["x"], t["delta"], prm["A"], t["B"], t["C"], y, D=prm["D"], z=t["z"],
                                  delta_bias=prm["delta_bias"]) for t in toks] for st in states]
    lib = ms.load_library()
    stream = torch.cuda.current_stream()

    def step(i, layer=0):
        rc = lib.mamba_state_update(ctypes.byref(argl[layer][i % 8]), stream.cuda_stream)
        if rc != 0:
            raise ms.MambaScanError(rc, lib.mamba_last_error().decode())

    for i in range(20):
        step(i, i % DECODE_LAYERS)
    torch.cuda.synchronize()
    n = args.decode_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # layers cycled: DECODE_GRAPH_STEPS calls through the C ABI captured once in
    # a CUDA graph (as a serving loop replays a token's layers), replayed until
    # n steps have run, so that the host's per-call cost does not starve the GPU
    reps = max(1, n // DECODE_GRAPH_STEPS)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            cap = torch.cuda.current_stream()
            for i in range(DECODE_GRAPH_STEPS):
                rc = lib.mamba_state_update(ctypes.byref(argl[i % DECODE_LAYERS][i % 8]), cap.cuda_stream)
                if rc != 0:
                    raise ms.MambaScanError(rc, lib.mamba_last_error().decode())
    stream.wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    cyc_us = e0.elapsed_time(e1) * 1e3 / (reps * DECODE_GRAPH_STEPS)
    del graph
    # back to back on one state
    e0.record(stream)
    for i in range(n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    hot_us = e0.elapsed_time(e1) * 1e3 / n
    # one state behind a 256 MB write
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    nf = min(n, 200)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nf)]
    for i in range(nf):
        flush.zero_()
        evs[i][0].record(stream)
        step(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    cold_us = sum(a.elapsed_time(b) for a, b in evs) * 1e3 / nf
    cyc_us = dist.max(cyc_us, dev)
    hot_us = dist.max(hot_us, dev)
    cold_us = dist.max(cold_us, dev)
    rows = w.batch * w.dim
    bytes_step = 2 * rows * w.dstate * 4 + 4 * rows * 2 + 2 * w.batch * w.dstate * 2 + w.dim * (w.dstate + 2) * 4
    peaks = load_peaks()
    elems = rows * w.dstate
    del flush
    return {
        "workload": w.name, "batch": w.batch, "d_inner": w.dim, "d_state": w.dstate, "steps": n,
        "metric": "decode state-update B*D*N elems/s", "unit": UNIT,
        "value": dist.world * elems / (cyc_us * 1e-6), "us_per_step": cyc_us,
        "timing": f"each step on the next of {DECODE_LAYERS} layers' states ({DECODE_LAYERS} x "
                  f"{w.batch * w.dim * w.dstate * 4 / 1e6:.0f} MB > L2); {DECODE_GRAPH_STEPS} C-ABI calls captured "
                  f"in a CUDA graph, replayed {reps} times",
        "value_back_to_back": dist.world * elems / (hot_us * 1e-6), "us_per_step_back_to_back": hot_us,
        "value_l2_flushed": dist.world * elems / (cold_us * 1e-6), "us_per_step_l2_flushed": cold_us,
        "tokens": "8 seeded token sets cycled",
        "kernel": "state_update_vec_kernel (dstate 16, two threads per row, two batch entries per thread)",
        "roofline": {"bound": "hbm", "unit": "GB/s", "algorithmic_bytes_per_step": bytes_step,
                     "achieved": bytes_step / (cyc_us * 1e-6) / 1e9,
                     "achieved_back_to_back": bytes_step / (hot_us * 1e-6) / 1e9,
                     "achieved_l2_flushed": bytes_step / (cold_us * 1e-6) / 1e9,
                     "peak": peaks["hbm_gbs"], "frac": bytes_step / (cyc_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                     "peak_source": peaks["source"],
                     "traffic": NCU_TRAFFIC.get((w.name, "state_update_vec_kernel")),
                     "note": "frac uses the layers-cycled timing; the L2-flushed step also pays the write-back of "
                             "the flush buffer's dirty lines"},
        "gpu_launches": reps * DECODE_GRAPH_STEPS + n + nf,
    }


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    return run_ours(args, dist)


if __name__ == "__main__":
    sys.exit(main())
