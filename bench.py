#!/usr/bin/env python
"""Benchmark of the block-scaled FP4 hot path on B200.

One step = one pass of the whole path over one batch: the NVFP4 Fprop of the
Llama-3.1-8B QKV projection at 8192 tokens -- rotated-tensor amax and fused
H16-rotate/scale/round/pack quantization of X [8192, 4096] and of
W [6144, 4096] (bf16), then the block-scaled FP4 GEMM Y = X W^T
(8192 x 6144 x 4096, bf16 out).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4|reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under torchrun,
each rank runs its own independent problem (weak scaling, no collective on the
data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp4_block_scaled_h16_b200 import workloads  # noqa: E402

METRIC = "FP4 quantize GB/s and block-scaled FP4 GEMM TFLOPS (% of B200 roofline)"
M, N, K = workloads.TOKENS, workloads.QKV_OUT, workloads.HIDDEN
WORKLOAD = "nvfp4_fprop_qkv_%dx%dx%d" % (M, N, K)
GEMM_FLOP = 2.0 * M * N * K
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one gemm_kernel
# launch on this workload, from one ncu capture of the current kernel: 36.3 MB
# read (the 33 MB of operands cross DRAM once) and 49.5 MB written (the rest of
# the 100.7 MB of C was still in L2 when the kernel ended)
GEMM_TRAFFIC_BYTES = 36_268_032 + 49_481_728


class L2Flush:
    """Evicts L2 (126 MB on B200) between timed steps: a 256 MiB write, then a
    256 MiB read, so that the lines left behind are clean and the next timed
    kernel does not pay for writing the flush buffer back to HBM."""

    def __init__(self, device):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self.sink = torch.zeros((), dtype=torch.int32, device=device)

    def __call__(self):
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.sink)
# algorithmic bytes per element (bf16 in): amax pass reads 2 B; the quantize
# pass reads 2 B and writes 0.5 B of codes + 1/16 B of E4M3 scale
AMAX_BPE = 2.0
QUANT_BPE = 2.0 + 0.5 + 1.0 / 16.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": names}


# ------------------------------------------------------------------------ GPU arm

class Fprop:
    """Device buffers and the step of the NVFP4 Fprop workload."""

    def __init__(self, fp4, X, W, device):
        self.fp4 = fp4
        self.X, self.W = X.to(device), W.to(device)
        self.qx = fp4.alloc_qtensor(M, K, fp4.FP4_NVFP4, device=device)
        self.qw = fp4.alloc_qtensor(N, K, fp4.FP4_NVFP4, device=device)
        self.ax = torch.empty(1, dtype=torch.float32, device=device)
        ws = fp4.fp4_quantize_workspace_size(fp4.FP4_NVFP4, False, False)
        self.wsx = torch.empty(ws, dtype=torch.uint8, device=device)
        self.wsw = torch.empty(ws, dtype=torch.uint8, device=device)
        self.C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        # quantize X (amax pass + quantize pass in one launch), the same for W, GEMM
        self.launches_per_step = 3

    def quant(self, x, q, ws):
        f = self.fp4
        f.quantize(x, f.FP4_NVFP4, f.FP4_RTNE, f.FP4_ROT_H16, axis=1, out=q, workspace=ws)

    def gemm(self):
        self.fp4.gemm(self.qx, self.qw, self.fp4.FP4_OUT_BF16, out=self.C)

    def step(self, ev=None):
        if ev:
            ev[0].record()
        self.quant(self.X, self.qx, self.wsx)
        if ev:
            ev[1].record()
        self.quant(self.W, self.qw, self.wsw)
        if ev:
            ev[2].record()
        self.gemm()
        if ev:
            ev[3].record()


def run_gpu(args, rank, world, device):
    from fp4_block_scaled_h16_b200 import fp4
    peaks = measured_peaks()
    d = workloads.nvfp4_fprop_qkv(seed=rank)
    w = Fprop(fp4, d["X"], d["W"], device)
    flush = L2Flush(device)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        w.step()
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK

    # optionally the step as one CUDA graph (its 3 kernels and 2 workspace
    # memsets), captured on a side stream after the eager warm-up
    graph = None
    if args.graph:
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            w.step()
            torch.cuda.synchronize()
            with torch.cuda.graph(graph, stream=side):
                w.step()
        torch.cuda.current_stream(device).wait_stream(side)
        torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clocks:
        for i in range(args.steps):
            flush()                       # L2 flush, outside the timed events
            evs[i][0].record()
            if graph is not None:
                graph.replay()
            else:
                w.step()
            evs[i][1].record()
        torch.cuda.synchronize()
    barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = sum(step_ms)
    status = fp4.fp4_last_error()

    # the step's kernels one by one (eager, events between them)
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(max(3, min(args.steps, 20)))]
    for e in evk:
        flush()
        w.step(e)
    torch.cuda.synchronize()
    qx = [e[0].elapsed_time(e[1]) for e in evk]
    qw = [e[1].elapsed_time(e[2]) for e in evk]
    gm = [e[2].elapsed_time(e[3]) for e in evk]

    # the two passes as separate kernels (fp4_amax, then fp4_quantize given the
    # amax), timed on a second pass: each kernel against its own bytes
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    amax_ms, quant_ms = [], []
    for _ in range(max(3, min(args.steps, 20))):
        flush()
        ev_a[0].record()
        fp4.fp4_amax(w.X, fp4.FP4_IN_BF16, M, K, K, fp4.FP4_ROT_H16, 1, 0, w.ax)
        ev_a[1].record()
        fp4.quantize(w.X, fp4.FP4_NVFP4, fp4.FP4_RTNE, fp4.FP4_ROT_H16, axis=1, tensor_amax=w.ax, out=w.qx)
        ev_a[2].record()
        torch.cuda.synchronize()
        amax_ms.append(ev_a[0].elapsed_time(ev_a[1]))
        quant_ms.append(ev_a[1].elapsed_time(ev_a[2]))

    # end to end through the public API: every step copies its inputs from
    # pinned host memory and its whole result back.  Two sets of device
    # buffers and three streams (host->device, compute, device->host) let
    # step i+1's inputs and step i-1's result cross PCIe, in both directions,
    # while step i computes; the timed region spans all the steps.
    e2e_steps = max(4, min(args.steps, 20))
    hX = d["X"].pin_memory()
    hW = d["W"].pin_memory()
    hC = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    slots = [w, Fprop(fp4, d["X"], d["W"], device)]
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "run", "out")}
    for k in ev:                                  # every slot starts free
        for e in ev[k]:
            e.record()
    torch.cuda.synchronize()
    flush()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in (s_run, s_out):
        _.wait_stream(s_in)
    for i in range(e2e_steps):
        k = i % 2
        f = slots[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["run"][k])         # step i-2 is done reading this slot
            f.X.copy_(hX, non_blocking=True)
            f.W.copy_(hW, non_blocking=True)
            ev["in"][k].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev["in"][k])
            s_run.wait_event(ev["out"][k])        # step i-2's result has left this slot
            f.step()
            ev["run"][k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][k])
            hC[k].copy_(f.C, non_blocking=True)
            ev["out"][k].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = [e0.elapsed_time(e1) / e2e_steps]
    del slots[1]

    t = torch.tensor([total_ms, statistics.mean(e2e_ms)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    total_max, e2e_max = float(t[0]), float(t[1])
    if rank != 0:
        return None

    ms_per_step = total_max / args.steps
    value = world * args.steps * GEMM_FLOP / (total_max * 1e-3) / 1e12
    gemm_ms = statistics.mean(gm)
    fp4_peak = peaks["bf16"] * 4.0      # nominal dense fp4 / bf16 ratio (9 / 2.25 PFLOP/s)
    achieved = GEMM_FLOP / (gemm_ms * 1e-3) / 1e12
    bpe_x = M * K
    comp = {
        "amax_X": {"ms": statistics.mean(amax_ms), "gbs": AMAX_BPE * bpe_x / (statistics.mean(amax_ms) * 1e6),
                   "kernel": "fp4_amax alone"},
        "quantize_X": {"ms": statistics.mean(quant_ms), "gbs": QUANT_BPE * bpe_x / (statistics.mean(quant_ms) * 1e6),
                       "kernel": "fp4_quantize given the amax"},
        "amax+quantize_X": {"ms": statistics.mean(qx), "gbs_2read": (AMAX_BPE + QUANT_BPE) * M * K / (statistics.mean(qx) * 1e6),
                            "gbs_1read": QUANT_BPE * M * K / (statistics.mean(qx) * 1e6),
                            "kernel": "fp4_quantize, internal amax: one launch (as timed in the step)"},
        "amax+quantize_W": {"ms": statistics.mean(qw), "gbs_2read": (AMAX_BPE + QUANT_BPE) * N * K / (statistics.mean(qw) * 1e6),
                            "gbs_1read": QUANT_BPE * N * K / (statistics.mean(qw) * 1e6),
                            "kernel": "fp4_quantize, internal amax: one launch (as timed in the step)"},
        "gemm": {"ms": gemm_ms, "tflops": achieved},
    }
    for k in ("amax_X", "quantize_X"):
        comp[k]["frac_hbm"] = comp[k]["gbs"] / peaks["hbm"]
    for k in ("amax+quantize_X", "amax+quantize_W"):
        comp[k]["frac_hbm"] = comp[k]["gbs_2read"] / peaks["hbm"]
        comp[k]["frac_hbm_1read"] = comp[k]["gbs_1read"] / peaks["hbm"]
    comp["gemm"]["frac_fp4"] = achieved / fp4_peak
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 scales) -> f32 accumulate; quantizer f32",
        "data": "synthetic (seeded: X N(0,1) with 8 outlier channels x64, W N(0,0.02); bf16)",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "format": "NVFP4",
                   "rotation": "H16", "rounding": "RTNE", "out": "bf16",
                   "value_is": "GEMM FLOP of the step / whole step time (quantize X and W, each with its tensor amax, + GEMM)",
                   "l2": "flushed between steps (256 MiB write, then 256 MiB read, outside the timed events)",
                   "launch": "the step replayed as one CUDA graph" if args.graph else "eager launches",
                   "parallelism": "independent problem per GPU" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "kernel": "gemm_kernel (NVFP4, 128x256 tile)",
                     "achieved": round(achieved, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / fp4_peak, 4), "traffic": GEMM_TRAFFIC_BYTES,
                     "traffic_is": "ncu dram read + write bytes of one launch (algorithmic: 33.0 MB read, 100.7 MB written)",
                     "peak_is": "%s bf16 burst %.1f TFLOP/s x 4 (nominal fp4/bf16)" % (peaks["src"], peaks["bf16"])},
        "components": comp,
        "e2e": {"value": round(world * GEMM_FLOP / (e2e_max * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(d["X"].numel() * 2 + d["W"].numel() * 2),
                "d2h_bytes_per_step": int(M * N * 2), "ms_per_step": round(e2e_max, 4),
                "how": "fp4.quantize / fp4.gemm on inputs copied from pinned host memory each step, the whole "
                       "bf16 result copied back; two buffer sets on 3 streams overlap the copies of "
                       "neighbouring steps with each other and with compute"},
        "gpu_launches": w.launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "device_status": fp4.fp4_status_string(status),
    }
    return line


# ------------------------------------------------------------------------ every config

def _median_ms(fn, flush, reps):
    """Median CUDA-event time of fn() over reps runs, L2 flushed before each."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    ts = []
    for _ in range(reps):
        flush()
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def _qbytes(x, fmt, db):
    """Algorithmic bytes of one quantize call: read once, codes + scales (+ outer) written."""
    n = x.numel()
    blk = 32 if fmt == 0 else 16
    return n * x.element_size() + n / 2 + n / blk + (n / 128 * 4 if db else 0)


CONFIG_NAMES = ("tiny", "wgrad", "dgrad_db", "layer")


def measure_configs(fp4, device, peaks, reps=10, only=CONFIG_NAMES):
    """Per-kernel timings of every workload (or of those named in `only`):
    quantize GB/s and GEMM TFLOP/s with their fractions of the measured HBM
    and derived FP4 peaks."""
    flush = L2Flush(device)
    fp4_peak = peaks["bf16"] * 4.0
    out = {}

    def quant_entry(x, **kw):
        fmt, db = kw["fmt"], kw.get("double_block", False)
        axis = kw.get("axis", 1)
        R, C = x.shape
        q = fp4.alloc_qtensor(R if axis else C, C if axis else R, fmt, db, device)
        ws = torch.empty(256, dtype=torch.uint8, device=device)
        ms = _median_ms(lambda: fp4.quantize(x, out=q, workspace=ws, **kw), flush, reps)
        gb = _qbytes(x, fmt, db) + (x.numel() * x.element_size() if (fmt != 0 and not db) else 0)
        return q, {"ms": ms, "gbs": gb / (ms * 1e6), "frac_hbm": gb / (ms * 1e6) / peaks["hbm"],
                   "bytes": "2 reads (amax pass + quantize)" if (fmt != 0 and not db) else "1 read"}

    def gemm_entry(qa, qb, out_dtype):
        M, N, K = qa["lines"], qb["lines"], qa["K"]
        C = torch.empty((M, N), dtype=torch.bfloat16 if out_dtype else torch.float32, device=device)
        ms = _median_ms(lambda: fp4.gemm(qa, qb, out_dtype, out=C), flush, reps)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        return {"ms": ms, "tflops": tf, "frac_fp4": tf / fp4_peak, "shape": [M, N, K]}

    NV, MX, UF = fp4.FP4_NVFP4, fp4.FP4_MXFP4, fp4.FP4_UFP4
    BF, F32 = fp4.FP4_OUT_BF16, fp4.FP4_OUT_F32

    if "tiny" in only:
        d = workloads.tiny_mxfp4()
        A, B = d["A"].to(device), d["B"].to(device)
        qa, ea = quant_entry(A, fmt=MX, axis=1)
        qb, eb = quant_entry(B, fmt=MX, axis=0)
        out["tiny_mxfp4_256x256x512"] = {"quantize_A": ea, "quantize_B": eb, "gemm": gemm_entry(qa, qb, F32),
                                         "note": "launch-bound; outside the roofline targets"}

    if "wgrad" in only:
        d = workloads.mxfp4_wgrad_down()
        dY, H = d["dY"].to(device), d["H"].to(device)
        kw = dict(fmt=MX, rounding=fp4.FP4_SR, rotation=fp4.FP4_ROT_RH32, axis=0, seed=0)
        qa, ea = quant_entry(dY, tensor_id=1, **kw)
        qb, eb = quant_entry(H, tensor_id=2, **kw)
        out["mxfp4_wgrad_down_4096x14336x8192"] = {"quantize_dY": ea, "quantize_H": eb,
                                                   "gemm": gemm_entry(qa, qb, F32)}
        del dY, H, qa, qb

    if "dgrad_db" in only:
        d = workloads.nvfp4_dgrad_down()
        dY, Wd = d["dY"].to(device), d["Wd"].to(device)
        kw = dict(fmt=NV, rounding=fp4.FP4_SR, double_block=True, seed=0)
        qa, ea = quant_entry(dY, axis=1, tensor_id=1, **kw)
        qb, eb = quant_entry(Wd, axis=0, tensor_id=2, **kw)
        entry = {"quantize_Wd": eb, "quantize_dY": ea, "gemm": gemm_entry(qa, qb, BF)}
        # tensor alignment: the forward-quantized weight W^ (rows) re-quantized
        # along the columns for this GEMM, instead of quantizing bf16 Wd again
        fwd = fp4.quantize(Wd, NV, fp4.FP4_RTNE, axis=1, double_block=True)
        back = fp4.alloc_qtensor(Wd.shape[1], Wd.shape[0], NV, True, device)
        ms = _median_ms(lambda: fp4.requantize(fwd, NV, fp4.FP4_SR, double_block=True, seed=0, tensor_id=2,
                                               out=back), flush, reps)
        n = Wd.numel()
        gb = 2 * (n // 2 + n // 16 + 4 * (n // 128))     # codes + scales + outer, read and written
        entry["requantize_Wd_hat"] = {"ms": ms, "gbs": gb / (ms * 1e6), "frac_hbm": gb / (ms * 1e6) / peaks["hbm"],
                                      "bytes": "FP4 source read + FP4 result written"}
        out["nvfp4_dgrad_down_db_8192x14336x4096"] = entry
        del dY, Wd, qa, qb, fwd, back
    if "layer" not in only:
        return out

    # the decoder layer: Fprop, Dgrad, Wgrad of each linear in NVFP4 with H16
    # (SR on the Wgrad operands), then the UFP4 quantizer on the same operands
    layer = {"quantize_nvfp4_ms": 0.0, "quantize_ufp4_ms": 0.0, "quantize_bytes": 0.0, "gemm_ms": 0.0,
             "gemm_flop": 0.0, "linears": {}}
    for name, _, _, _ in workloads.LAYER_LINEARS:
        d = workloads.layer_linear(name)
        X, W, dY = d["X"].to(device), d["W"].to(device), d["dY"].to(device)
        H16, SR, RT = fp4.FP4_ROT_H16, fp4.FP4_SR, fp4.FP4_RTNE
        ops = {"X_ax1": (X, 1, RT), "W_ax1": (W, 1, RT), "dY_ax1": (dY, 1, RT), "W_ax0": (W, 0, RT),
               "dY_ax0": (dY, 0, SR), "X_ax0": (X, 0, SR)}
        lin = {}
        qs = {}
        for role, (t, axis, rnd) in ops.items():
            qs[role], e = quant_entry(t, fmt=NV, rounding=rnd, rotation=H16, axis=axis, seed=0, tensor_id=len(qs))
            _, u = quant_entry(t, fmt=UF, rounding=rnd, rotation=H16, axis=axis, seed=0, tensor_id=len(qs))
            lin["nv_" + role], lin["uf_" + role] = e, u
            layer["quantize_nvfp4_ms"] += e["ms"]
            layer["quantize_ufp4_ms"] += u["ms"]
            layer["quantize_bytes"] += e["gbs"] * e["ms"] * 1e6
        for gname, (a_, b_, od) in {"fprop": ("X_ax1", "W_ax1", BF), "dgrad": ("dY_ax1", "W_ax0", BF),
                                    "wgrad": ("dY_ax0", "X_ax0", F32)}.items():
            g = gemm_entry(qs[a_], qs[b_], od)
            lin[gname] = g
            layer["gemm_ms"] += g["ms"]
            layer["gemm_flop"] += 2.0 * g["shape"][0] * g["shape"][1] * g["shape"][2]
        layer["linears"][name] = lin
        del X, W, dY, qs
        torch.cuda.empty_cache()
    layer["gemm_tflops"] = layer["gemm_flop"] / (layer["gemm_ms"] * 1e-3) / 1e12
    layer["gemm_frac_fp4"] = layer["gemm_tflops"] / fp4_peak
    layer["quantize_nvfp4_gbs"] = layer["quantize_bytes"] / (layer["quantize_nvfp4_ms"] * 1e6)
    layer["quantize_nvfp4_frac_hbm"] = layer["quantize_nvfp4_gbs"] / peaks["hbm"]
    out["llama8b_layer_linears_t8192"] = layer
    return out


# ------------------------------------------------------------------------ oracle arm

def oracle_slab_time(d, rows):
    """Oracle time of the step restricted to `rows` rows of X and of W,
    extrapolated to the whole workload (seconds), and the threads it used."""
    import oracle
    X = workloads.bf16_bits(d["X"][:rows])
    W = workloads.bf16_bits(d["W"][:rows])
    t0 = time.perf_counter()
    ax = oracle.tensor_amax(X, 1, oracle.ROT_H16)
    t1 = time.perf_counter()
    qx = oracle.quantize(X, oracle.NVFP4, rotation=oracle.ROT_H16, amax=ax)
    t2 = time.perf_counter()
    aw = oracle.tensor_amax(W, 1, oracle.ROT_H16)
    t3 = time.perf_counter()
    qw = oracle.quantize(W, oracle.NVFP4, rotation=oracle.ROT_H16, amax=aw)
    t4 = time.perf_counter()
    oracle.gemm(qx, qw)
    t5 = time.perf_counter()
    full = ((t2 - t0) * M / rows + (t4 - t2) * N / rows + (t5 - t4) * (M * N) / (rows * rows))
    return full, oracle.default_threads()


def cpu_baseline(d, target_s=10.0):
    rows = 64
    t, cores = oracle_slab_time(d, rows)
    # grow the slab towards ~target_s of CPU work
    spent = t * rows / M
    if spent < target_s / 4:
        rows = int(min(1024, rows * target_s / 2 / max(spent, 1e-3)))
        rows = max(64, rows - rows % 16)
        t, cores = oracle_slab_time(d, rows)
    value = GEMM_FLOP / t / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": "%d rows of X and of W: amax + quantize (NVFP4, H16) and the float64 GEMM of "
                      "the %dx%d slab, each part extrapolated to the full 8192x6144x4096 step" % (rows, rows, rows)}


def run_reference(args):
    """The oracle, as it stands, timed on the host cores on a bounded sample."""
    d = workloads.nvfp4_fprop_qkv(seed=0)
    budget_s = 120.0                              # wall time of the whole run
    steps = args.steps + args.warmup
    # calibrate on a 64-row slab, then take the largest slab (a multiple of 16
    # rows, at most 1024) whose steps fit the budget: small slabs are
    # dominated by fixed costs and understate the oracle's rate
    t0 = time.perf_counter()
    oracle_slab_time(d, 64)
    wall64 = time.perf_counter() - t0
    rows = int(64 * budget_s / (steps * max(wall64, 1e-4)))
    rows = max(16, min(1024, rows - rows % 16))
    times = []
    for i in range(args.warmup + args.steps):
        t, cores = oracle_slab_time(d, rows)
        if i >= args.warmup:
            times.append(t)
    ms = statistics.mean(times) * 1e3
    value = GEMM_FLOP / (ms * 1e-3) / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer, f64 GEMM (CPU oracle)",
        "data": "synthetic (same seeded workload)",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "format": "NVFP4", "rotation": "H16",
                   "rounding": "RTNE", "out": "f64"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: %d rows of X and W through the whole step, extrapolated" % rows},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fp4", "reference"], default="fp4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config kernel table")
    ap.add_argument("--graph", action="store_true",
                    help="time the step replayed as one CUDA graph (measured equal to eager launches)")
    ap.add_argument("--configs", default=",".join(CONFIG_NAMES),
                    help="comma-separated workloads of the per-config table: " + ", ".join(CONFIG_NAMES))
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    line = run_gpu(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_configs:
            from fp4_block_scaled_h16_b200 import fp4 as _fp4
            only = tuple(c for c in args.configs.split(",") if c)
            unknown = [c for c in only if c not in CONFIG_NAMES]
            if unknown:
                raise SystemExit("unknown --configs entries: %s" % ", ".join(unknown))
            line["configs"] = measure_configs(_fp4, device, measured_peaks(), only=only)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(workloads.nvfp4_fprop_qkv(seed=0))
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
