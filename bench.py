#!/usr/bin/env python
"""Benchmark of the block-scaled FP4 hot path on B200.

One step = one pass of the whole path over the linears of one Llama-3.1-8B
decoder layer at 8192 tokens: QKV 4096 -> 6144, O 4096 -> 4096, fused
gate+up 4096 -> 28672, down 14336 -> 4096.  For each linear the six operands
of its Fprop, Dgrad and Wgrad GEMMs are quantized to NVFP4 with H16 (rotated
tensor amax, rotate, block scale, round, pack; stochastic rounding on the
Wgrad operands; the Dgrad and Wgrad operands along the transposed axis) and
the three block-scaled FP4 GEMMs run: 24 quantize calls and 12 GEMMs,
10.72 TFLOP of GEMM work per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4|reference]

Prints one JSON line (rank 0).  `value` is the step's GEMM FLOP over the whole
step time (quantization included).  Multi-GPU: one process per GPU under
torchrun, each rank runs its own independent layer (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
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
WORKLOAD = "llama31_8b_layer_linears_t8192_nvfp4_h16"
T = workloads.TOKENS
L2_FLUSH_BYTES = 256 << 20
OPERANDS = workloads.LAYER_OPERANDS
GEMMS = workloads.LAYER_GEMMS
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per GEMM launch,
# averaged over the 12 GEMM launches of one layer step, from one ncu capture of
# the current kernel (profiles/gemm_layer_llama8b_t8192.md); the algorithmic
# bytes (operands read once, C written once) average 241.7 MB
GEMM_TRAFFIC_BYTES_PER_LAUNCH = 276_598_528
# the same for the step's 12 both-axes quantize launches (profiles/quant_both_axes_layer_llama8b_t8192.md);
# their algorithmic bytes (input read twice, both outputs written) average 336.8 MB
QUANT_BOTH_TRAFFIC_BYTES_PER_LAUNCH = 246_176_917


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


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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


def qbytes(numel, elem_bytes, fmt, db=False, reads=1):
    """Algorithmic bytes of one quantize call: the input read `reads` times,
    codes + scales (+ outer scales) written."""
    blk = 32 if fmt == 0 else 16
    return reads * numel * elem_bytes + numel / 2 + numel / blk + (numel / 128 * 4 if db else 0)


def quantize_kernels(axis, internal_amax):
    """Kernels one fp4_quantize call launches: one on either axis (with an
    internal tensor amax, the amax and quantize passes run as one cooperative
    kernel)."""
    return 1


# ------------------------------------------------------------------------ GPU arm

class LayerStep:
    """Device buffers and the step of the layer workload: per linear, the six
    NVFP4 + H16 operands and the Fprop, Dgrad and Wgrad GEMMs."""

    def __init__(self, fp4, device, seed=0, fmt=None, host=None, both_axes=True):
        self.fp4 = fp4
        self.fmt = fp4.FP4_NVFP4 if fmt is None else fmt
        self.device = device
        self.linears = []
        self.flop = 0.0
        self.quant_bytes = 0.0
        self.ws = torch.empty(256, dtype=torch.uint8, device=device)
        self.launches = 0
        for index, (name, d_in, d_out, _) in enumerate(workloads.LAYER_LINEARS):
            d = host[index] if host is not None else workloads.layer_linear(name, seed=seed)
            t = {k: v.to(device) for k, v in d.items()}
            qs, calls = [], []
            for role, (tn, axis, sr) in enumerate(OPERANDS):
                R, C = t[tn].shape
                L, K = (R, C) if axis == 1 else (C, R)
                qs.append(fp4.alloc_qtensor(L, K, self.fmt, device=device))
                calls.append(dict(x=tn, axis=axis, rounding=fp4.FP4_SR if sr else fp4.FP4_RTNE,
                                  tensor_id=workloads.layer_tensor_id(index, role), name="%s_ax%d" % (tn, axis)))
                self.quant_bytes += qbytes(R * C, 2, self.fmt, reads=2)
            outs = []
            for gname, ra, rb, bf16 in GEMMS:
                M, N, K = qs[ra]["lines"], qs[rb]["lines"], qs[ra]["K"]
                outs.append(torch.empty((M, N), dtype=torch.bfloat16 if bf16 else torch.float32, device=device))
                self.flop += 2.0 * M * N * K
            # both-axes calls: each tensor once, its row operand and its column operand together
            both = []
            for tn in dict.fromkeys(c["x"] for c in calls):
                rrole = next(r for r, c in enumerate(calls) if c["x"] == tn and c["axis"] == 1)
                crole = next(r for r, c in enumerate(calls) if c["x"] == tn and c["axis"] == 0)
                both.append(dict(x=tn, rows=rrole, cols=crole, name="%s_both" % tn))
            self.linears.append(dict(name=name, t=t, qs=qs, calls=calls, both=both, outs=outs))
        self.set_both_axes(both_axes)

    def set_both_axes(self, on):
        """Quantize each tensor along both axes in one call (fp4_quantize_both_axes,
        3 calls per linear) or each operand on its own (fp4_quantize, 6 calls)."""
        self.both_axes = bool(on)
        n_lin = len(self.linears)
        self.launches = n_lin * (3 if self.both_axes else len(OPERANDS)) + n_lin * len(GEMMS)

    def quantize_both(self, lin, k):
        b = lin["both"][k]
        cr, cc = lin["calls"][b["rows"]], lin["calls"][b["cols"]]
        self.fp4.quantize_both_axes(lin["t"][b["x"]], self.fmt, self.fp4.FP4_ROT_H16, seed=0,
                                    rounding_rows=cr["rounding"], tensor_id_rows=cr["tensor_id"],
                                    rounding_cols=cc["rounding"], tensor_id_cols=cc["tensor_id"],
                                    out_rows=lin["qs"][b["rows"]], out_cols=lin["qs"][b["cols"]], workspace=self.ws)

    def quantize(self, lin, role):
        c = lin["calls"][role]
        self.fp4.quantize(lin["t"][c["x"]], self.fmt, c["rounding"], self.fp4.FP4_ROT_H16, axis=c["axis"],
                          seed=0, tensor_id=c["tensor_id"], out=lin["qs"][role], workspace=self.ws)

    def gemm(self, lin, g):
        _, ra, rb, bf16 = GEMMS[g]
        self.fp4.gemm(lin["qs"][ra], lin["qs"][rb], self.fp4.FP4_OUT_BF16 if bf16 else self.fp4.FP4_OUT_F32,
                      out=lin["outs"][g])

    def calls(self):
        """The step's calls in order: (kind, linear name, call name, fn)."""
        out = []
        for lin in self.linears:
            if self.both_axes:
                for k, b in enumerate(lin["both"]):
                    out.append(("quant_both", lin["name"], b["name"], k, lin))
            else:
                for role in range(len(OPERANDS)):
                    kind = "quant_rows" if lin["calls"][role]["axis"] == 1 else "quant_cols"
                    out.append((kind, lin["name"], lin["calls"][role]["name"], role, lin))
            for g in range(len(GEMMS)):
                out.append(("gemm", lin["name"], GEMMS[g][0], g, lin))
        return out

    def run_call(self, c):
        kind, _, _, i, lin = c
        if kind == "gemm":
            self.gemm(lin, i)
        elif kind == "quant_both":
            self.quantize_both(lin, i)
        else:
            self.quantize(lin, i)

    def step(self):
        for lin in self.linears:
            if self.both_axes:
                for k in range(len(lin["both"])):
                    self.quantize_both(lin, k)
            else:
                for role in range(len(OPERANDS)):
                    self.quantize(lin, role)
            for g in range(len(GEMMS)):
                self.gemm(lin, g)


def time_steps(fn, flush, n):
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for e in evs:
        flush()
        e[0].record()
        fn()
        e[1].record()
    torch.cuda.synchronize()
    return [e[0].elapsed_time(e[1]) for e in evs]


def _median_ms(fn, flush, reps):
    """Median CUDA-event time of fn() over reps runs, L2 flushed before each."""
    fn()
    return statistics.median(time_steps(fn, flush, reps))


def per_call_split(layer, flush, reps, peaks):
    """Each call of the step timed on its own (events between the calls of
    eager steps), with its algorithmic rate and fraction of peak."""
    calls = layer.calls()
    ms = [[] for _ in calls]
    for _ in range(reps):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        evs[0].record()
        for i, c in enumerate(calls):
            layer.run_call(c)
            evs[i + 1].record()
        torch.cuda.synchronize()
        for i in range(len(calls)):
            ms[i].append(evs[i].elapsed_time(evs[i + 1]))
    fp4_peak = peaks["bf16"] * 4.0
    table, fam = {}, {}
    for c, m in zip(calls, ms):
        kind, lname, cname, i, lin = c
        t = statistics.mean(m)
        if kind == "gemm":
            _, ra, rb, _ = GEMMS[i]
            M, N, K = lin["qs"][ra]["lines"], lin["qs"][rb]["lines"], lin["qs"][ra]["K"]
            work = 2.0 * M * N * K
            e = {"ms": t, "tflops": work / (t * 1e-3) / 1e12, "frac_fp4": work / (t * 1e-3) / 1e12 / fp4_peak,
                 "shape": [M, N, K], "launches": 1}
        elif kind == "quant_both":
            b = lin["both"][i]
            x = lin["t"][b["x"]]
            # the input read twice (amax pass, quantize pass) for both axes; both outputs written
            work = 2 * x.numel() * 2 + 2 * (qbytes(x.numel(), 2, layer.fmt, reads=0))
            e = {"ms": t, "gbs": work / (t * 1e6), "frac_hbm": work / (t * 1e6) / peaks["hbm"],
                 "bytes": "2 reads (amax pass + quantize, both axes at once) + both outputs", "launches": 1,
                 "rounding": "rows %s, columns %s" % tuple("SR" if lin["calls"][b[a]]["rounding"] else "RTNE"
                                                            for a in ("rows", "cols"))}
        else:
            x = lin["t"][lin["calls"][i]["x"]]
            work = qbytes(x.numel(), 2, layer.fmt, reads=2)
            axis = lin["calls"][i]["axis"]
            e = {"ms": t, "gbs": work / (t * 1e6), "frac_hbm": work / (t * 1e6) / peaks["hbm"],
                 "bytes": "2 reads (amax pass + quantize)", "launches": quantize_kernels(axis, True),
                 "rounding": "SR" if lin["calls"][i]["rounding"] else "RTNE"}
        table.setdefault(lname, {})[cname] = e
        f = fam.setdefault(kind, {"ms": 0.0, "work": 0.0, "launches": 0})
        f["ms"] += t
        f["work"] += work
        f["launches"] += e["launches"]
    for kind, f in fam.items():
        if kind == "gemm":
            f["tflops"] = f["work"] / (f["ms"] * 1e-3) / 1e12
            f["frac_fp4"] = f["tflops"] / fp4_peak
        else:
            f["gbs"] = f["work"] / (f["ms"] * 1e6)
            f["frac_hbm"] = f["gbs"] / peaks["hbm"]
    return table, fam


class Fprop:
    """The NVFP4 Fprop of the QKV projection (8192 x 6144 x 4096): quantize X
    and W (each with its tensor amax, one launch), then the GEMM."""

    def __init__(self, fp4, X, W, device):
        self.fp4 = fp4
        self.X, self.W = X.to(device), W.to(device)
        M, K = self.X.shape
        N = self.W.shape[0]
        self.shape = (M, N, K)
        self.qx = fp4.alloc_qtensor(M, K, fp4.FP4_NVFP4, device=device)
        self.qw = fp4.alloc_qtensor(N, K, fp4.FP4_NVFP4, device=device)
        self.ws = torch.empty(256, dtype=torch.uint8, device=device)
        self.C = torch.empty((M, N), dtype=torch.bfloat16, device=device)

    def step(self):
        f = self.fp4
        f.quantize(self.X, f.FP4_NVFP4, f.FP4_RTNE, f.FP4_ROT_H16, axis=1, out=self.qx, workspace=self.ws)
        f.quantize(self.W, f.FP4_NVFP4, f.FP4_RTNE, f.FP4_ROT_H16, axis=1, out=self.qw, workspace=self.ws)
        f.gemm(self.qx, self.qw, f.FP4_OUT_BF16, out=self.C)


def fprop_component(fp4, device, flush, peaks, reps):
    d = workloads.nvfp4_fprop_qkv(seed=0)
    w = Fprop(fp4, d["X"], d["W"], device)
    M, N, K = w.shape
    step = _median_ms(w.step, flush, reps)
    gemm = _median_ms(lambda: fp4.gemm(w.qx, w.qw, fp4.FP4_OUT_BF16, out=w.C), flush, reps)
    flop = 2.0 * M * N * K
    out = {"workload": "nvfp4_fprop_qkv_%dx%dx%d" % (M, N, K),
           "step_ms": step, "step_tflops": flop / (step * 1e-3) / 1e12,
           "gemm_ms": gemm, "gemm_tflops": flop / (gemm * 1e-3) / 1e12,
           "gemm_frac_fp4": flop / (gemm * 1e-3) / 1e12 / (4 * peaks["bf16"])}
    # context ratio ("Ripensare il Bias di Shrinkage...", Efficienza: fused
    # RHT + quantization about 1.06-1.07x the quantization alone, unfused
    # 1.4-1.6x, on SM90 / SM100 at sizes the pages do not state): NVFP4 of X
    # with the random-sign H16 fused, without a rotation, and as a separate
    # rotation kernel (bf16 out) followed by the quantizer without rotation
    qx, ws = w.qx, w.ws
    Xr = torch.empty_like(w.X)
    NV, RT = fp4.FP4_NVFP4, fp4.FP4_RTNE
    fused = _median_ms(lambda: fp4.quantize(w.X, NV, RT, fp4.FP4_ROT_RH16, axis=1, seed=5, out=qx, workspace=ws),
                       flush, reps)
    none = _median_ms(lambda: fp4.quantize(w.X, NV, RT, fp4.FP4_ROT_NONE, axis=1, out=qx, workspace=ws),
                      flush, reps)

    def unfused():
        fp4.rotate(w.X, fp4.FP4_ROT_RH16, seed=5, out=Xr)
        fp4.quantize(Xr, NV, RT, fp4.FP4_ROT_NONE, axis=1, out=qx, workspace=ws)

    unf = _median_ms(unfused, flush, reps)
    rot_only = _median_ms(lambda: fp4.rotate(w.X, fp4.FP4_ROT_RH16, seed=5, out=Xr), flush, reps)
    out["context_ratio"] = {
        "tensor": "X bf16 %dx%d, NVFP4, RTNE, internal tensor amax (one launch)" % (M, K),
        "fused_rh16_ms": fused, "no_rotation_ms": none, "unfused_rotate_then_quantize_ms": unf,
        "rotate_kernel_alone_ms": rot_only,
        "fused_over_none": fused / none, "unfused_over_none": unf / none,
        "pages": "fused ~1.06-1.07x, unfused ~1.4-1.6x of standalone quantization (SM90/SM100; sizes not stated)"}
    # the two passes of the NVFP4 + H16 quantization of X on their own, each
    # against its own bytes: the rotated amax (fp4_amax, one read) and the
    # quantization given that amax (one read, codes and scales written), beside
    # the one-launch call's two reads
    amax = torch.zeros(1, dtype=torch.float32, device=device)
    H16 = fp4.FP4_ROT_H16

    def amax_only():
        amax.zero_()
        fp4.fp4_amax(w.X, fp4.FP4_IN_BF16, M, K, K, H16, 1, 0, amax)

    t_amax = _median_ms(amax_only, flush, reps)
    t_given = _median_ms(lambda: fp4.quantize(w.X, NV, RT, H16, axis=1, tensor_amax=amax, out=qx), flush, reps)
    t_fused = _median_ms(lambda: fp4.quantize(w.X, NV, RT, H16, axis=1, out=qx, workspace=ws), flush, reps)
    read_b = M * K * 2.0
    one = qbytes(M * K, 2, NV)
    two = qbytes(M * K, 2, NV, reads=2)
    hbm = peaks["hbm"]
    out["quantize_passes"] = {
        "tensor": "X bf16 %dx%d, NVFP4 + H16, RTNE" % (M, K),
        "amax_only": {"ms": t_amax, "gbs": read_b / (t_amax * 1e6), "frac_hbm": read_b / (t_amax * 1e6) / hbm,
                      "bytes": "1 read (the memset of the amax word included in the time)"},
        "quantize_given_amax": {"ms": t_given, "gbs": one / (t_given * 1e6), "frac_hbm": one / (t_given * 1e6) / hbm,
                                "bytes": "1 read, codes and scales written"},
        "one_launch": {"ms": t_fused, "gbs": two / (t_fused * 1e6), "frac_hbm": two / (t_fused * 1e6) / hbm,
                       "bytes": "2 reads (the second mostly from L2), codes and scales written"}}
    del w, Xr
    torch.cuda.empty_cache()
    return out


def run_gpu(args, rank, world, device, host):
    """The timed layer steps, the per-call split and the end-to-end steps;
    `host` holds the layer's inputs in host memory (layer_host_data)."""
    from fp4_block_scaled_h16_b200 import fp4
    peaks = measured_peaks()
    layer = LayerStep(fp4, device, seed=rank, host=host)
    flush = L2Flush(device)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK

    graph = None
    if args.graph:
        # the step as one CUDA graph (its kernels and workspace memsets),
        # captured on a side stream after the eager warm-up
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            layer.step()
            torch.cuda.synchronize()
            with torch.cuda.graph(graph, stream=side):
                layer.step()
        torch.cuda.current_stream(device).wait_stream(side)
        torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clocks:
        step_ms = time_steps(graph.replay if graph is not None else layer.step, flush, args.steps)
    barrier()
    total_ms = sum(step_ms)
    status = fp4.fp4_last_error()

    table, fam = per_call_split(layer, flush, max(3, min(args.steps, 10)), peaks)

    # the same step with each of the 24 operands quantized by its own call
    # (fp4_quantize along one axis; each bf16 tensor is then read for each axis)
    layer.set_both_axes(False)
    sep_reps = max(3, min(args.steps, 10))
    layer.step()
    torch.cuda.synchronize()
    sep_ms = statistics.median(time_steps(layer.step, flush, sep_reps))
    _, sep_fam = per_call_split(layer, flush, sep_reps, peaks)
    layer.set_both_axes(True)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    separate = {"ms_per_step": round(sep_ms, 4), "value": round(layer.flop / (sep_ms * 1e-3) / 1e12, 2),
                "families_ms": {k: round(v["ms"], 4) for k, v in sep_fam.items()},
                "how": "24 fp4_quantize calls (one axis each, with its tensor amax) + the 12 GEMMs, median of %d "
                       "event-timed steps, L2 flushed before each" % sep_reps}

    # end to end through the public API: every step copies its inputs (X, W and
    # dY of the four linears) from pinned host memory and its results (the 12
    # GEMM outputs) back.  Two sets of device buffers on three streams
    # (host->device, compute, device->host) let step i+1's inputs and step
    # i-1's results cross PCIe while step i computes.
    e2e_steps = 0 if args.no_e2e else 4
    if e2e_steps == 0:
        return finish_line(args, rank, world, device, layer, fam, table, total_ms, None, 0, 0, clocks, status, peaks,
                           separate)
    hin = [{k: v.pin_memory() for k, v in h.items()} for h in host]
    hout = [[[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in lin["outs"]] for lin in layer.linears]
            for _ in range(2)]
    second = LayerStep(fp4, device, host=hin)
    slots = [layer, second]
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "run", "out")}
    for k in ev:
        for e in ev[k]:
            e.record()
    torch.cuda.synchronize()
    flush()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for st in (s_run, s_out):
        st.wait_stream(s_in)
    for i in range(e2e_steps):
        k = i % 2
        f = slots[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["run"][k])          # step i-2 is done reading this slot
            for lin, h in zip(f.linears, hin):
                for name, t in lin["t"].items():
                    t.copy_(h[name], non_blocking=True)
            ev["in"][k].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev["in"][k])
            s_run.wait_event(ev["out"][k])         # step i-2's results have left this slot
            f.step()
            ev["run"][k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][k])
            for lin, h in zip(f.linears, hout[k]):
                for o, ho in zip(lin["outs"], h):
                    ho.copy_(o, non_blocking=True)
            ev["out"][k].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = sum(v.numel() * v.element_size() for h in hin for v in h.values())
    d2h = sum(o.numel() * o.element_size() for lin in layer.linears for o in lin["outs"])
    del slots, second, hout
    torch.cuda.empty_cache()

    return finish_line(args, rank, world, device, layer, fam, table, total_ms, e2e_ms, h2d, d2h, clocks, status, peaks,
                       separate)


def finish_line(args, rank, world, device, layer, fam, table, total_ms, e2e_ms, h2d, d2h, clocks, status, peaks,
                separate=None):
    """Max over ranks of the timings, then rank 0's JSON line."""
    from fp4_block_scaled_h16_b200 import fp4
    t = torch.tensor([total_ms, e2e_ms if e2e_ms is not None else 0.0], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    total_max, e2e_max = float(t[0]), float(t[1])
    if rank != 0:
        return None, layer

    ms_per_step = total_max / args.steps
    value = world * args.steps * layer.flop / (total_max * 1e-3) / 1e12
    fp4_peak = peaks["bf16"] * 4.0
    # the dominant kernel family of the step, by time
    dom = max(fam, key=lambda k: fam[k]["ms"])
    f = fam[dom]
    if dom == "gemm":
        roof = {"bound": "tensor", "kernel": "gemm_pair_kernel (NVFP4, 256x256 tiles on CTA pairs, 12 launches per step)",
                "achieved": round(f["tflops"], 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                "frac": round(f["tflops"] / fp4_peak, 4), "traffic": GEMM_TRAFFIC_BYTES_PER_LAUNCH,
                "traffic_is": "ncu DRAM read + write bytes per launch, averaged over the step's 12 GEMMs "
                              "(algorithmic average 241.7 MB)",
                "achieved_is": "GEMM FLOP of the step / summed mean event time of its 12 GEMM launches",
                "peak_is": "%s bf16 burst %.1f TFLOP/s x 4 (nominal fp4 / bf16 ratio)" % (peaks["src"], peaks["bf16"])}
    else:
        roof = {"bound": "hbm", "kernel": {"quant_rows": "quant_rows_kernel, 12 calls per step",
                                           "quant_cols": "quant_cols_kernel (amax + quantize), 12 calls per step",
                                           "quant_both": "quant_cols_kernel, both axes (amax + quantize of the rows "
                                                         "and the columns), 12 calls per step"}[dom],
                "achieved": round(f["gbs"], 1), "peak": round(peaks["hbm"], 1), "unit": "GB/s",
                "frac": round(f["gbs"] / peaks["hbm"], 4),
                "traffic": QUANT_BOTH_TRAFFIC_BYTES_PER_LAUNCH if dom == "quant_both" else None,
                "traffic_is": ("ncu DRAM read + write bytes per launch, averaged over the step's 12 both-axes "
                               "launches (algorithmic average 336.8 MB: the second read of a tensor that fits in "
                               "L2 comes from L2)" if dom == "quant_both" else None),
                "bound_by": ("instruction issue: 59 thread instructions per element at 51% issue for a call with "
                             "SR columns, 7.8% of DRAM throughput (ncu)" if dom == "quant_both" else None),
                "achieved_is": "algorithmic bytes (input read twice: amax pass + quantize; codes and "
                               "scales written) / summed mean event time",
                "peak_is": "%s HBM copy bandwidth" % peaks["src"]}
    roof["families"] = {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                        for k, v in fam.items()}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 scales) -> f32 accumulate; quantizer f32",
        "data": "synthetic (seeded: activations N(0,1) with 8 outlier channels x64 or SwiGLU N(0,1)*silu(N(0,1)), "
                "W N(0,0.02), dY Laplace(0,1e-3); bf16)",
        "config": {"workload": WORKLOAD, "tokens": T,
                   "linears": {n: [d_in, d_out] for n, d_in, d_out, _ in workloads.LAYER_LINEARS},
                   "format": "NVFP4", "rotation": "H16 on all three GEMMs",
                   "rounding": "RTNE; SR on the Wgrad operands", "out": "bf16 (Fprop, Dgrad), f32 (Wgrad)",
                   "gemm_flop_per_step": layer.flop,
                   "value_is": "GEMM FLOP of the step / whole step time (the 24 NVFP4 operands from 12 "
                               "both-axes quantize calls, each axis with its own tensor amax, + 12 GEMMs)",
                   "l2": "flushed before every step (256 MiB write, then 256 MiB read, outside the timed "
                         "events); the step's 1.6 GB of inputs exceed L2",
                   "launch": "the step replayed as one CUDA graph" if args.graph else "eager launches",
                   "parallelism": "independent layer per GPU" if world > 1 else "single GPU"},
        "roofline": roof,
        "components": {"per_call": table, "separate_axes": separate},
        "e2e": ({"value": round(world * layer.flop / (e2e_max * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                 "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_max, 3),
                 "how": "fp4.quantize / fp4.gemm on the layer's inputs copied from pinned host memory every step, "
                        "the 12 GEMM outputs copied back; two buffer sets on 3 streams overlap the copies of "
                        "neighbouring steps with each other and with compute"}
                if e2e_ms is not None else None),
        "gpu_launches": layer.launches * args.steps,
        "clocks": clocks.summary(),
        "device_status": fp4.fp4_status_string(status),
    }
    return line, layer


# ------------------------------------------------------------------------ other workloads

CONFIG_NAMES = ("fprop", "ufp4", "mxnorm", "outctl", "tiny", "wgrad", "dgrad_db")
# c(2, B) for Gaussian rows, E[max of B |N(0,1)|^2]^(1/2) (B = 32: MXFP4, 16:
# NVFP4); the kernel's cost does not depend on the value
MXNORM_C2 = {0: 2.3894571, 1: 2.1329500}


def layer_gemm_shapes(layer):
    """(M, N, K) of the layer's 12 GEMMs."""
    out = []
    for lin in layer.linears:
        for _, ra, rb, _ in GEMMS:
            out.append((lin["qs"][ra]["lines"], lin["qs"][rb]["lines"], lin["qs"][ra]["K"]))
    return out


def measure_configs(fp4, device, peaks, layer=None, reps=10, only=CONFIG_NAMES):
    """Per-kernel timings of the other workloads: quantize GB/s and GEMM TFLOP/s
    with their fractions of the measured HBM and derived FP4 peaks."""
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
        two = fmt != 0 and not db
        gb = qbytes(x.numel(), x.element_size(), fmt, db, reads=2 if two else 1)
        return q, {"ms": ms, "gbs": gb / (ms * 1e6), "frac_hbm": gb / (ms * 1e6) / peaks["hbm"],
                   "bytes": "2 reads (amax pass + quantize)" if two else "1 read"}

    def gemm_entry(qa, qb, out_dtype):
        M, N, K = qa["lines"], qb["lines"], qa["K"]
        C = torch.empty((M, N), dtype=torch.bfloat16 if out_dtype else torch.float32, device=device)
        ms = _median_ms(lambda: fp4.gemm(qa, qb, out_dtype, out=C), flush, reps)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        return {"ms": ms, "tflops": tf, "frac_fp4": tf / fp4_peak, "shape": [M, N, K]}

    NV, MX, UF = fp4.FP4_NVFP4, fp4.FP4_MXFP4, fp4.FP4_UFP4
    BF, F32 = fp4.FP4_OUT_BF16, fp4.FP4_OUT_F32

    if "fprop" in only:
        out["nvfp4_fprop_qkv_8192x6144x4096"] = fprop_component(fp4, device, flush, peaks, reps)

    if "ufp4" in only and layer is not None:
        # the UFP4 recipe (levels k * s, k in [-7, 7]) on the layer's operands:
        # the 24 quantize calls, then the 12 GEMMs.  A UFP4 GEMM runs as an
        # NVFP4 GEMM over the operands' E2M1 parts, 4x the tensor-core work:
        # its ceiling is a quarter of the FP4 peak
        uf, ug = {}, {}
        tot_ms = tot_b = g_ms = g_flop = 0.0
        ws = torch.empty(max(fp4.fp4_gemm_workspace_size(UF, False, *g) for g in layer_gemm_shapes(layer)),
                         dtype=torch.uint8, device=device)
        for lin in layer.linears:
            qs = []
            for role, c in enumerate(lin["calls"]):
                x = lin["t"][c["x"]]
                q, e = quant_entry(x, fmt=UF, rounding=c["rounding"], rotation=fp4.FP4_ROT_H16, axis=c["axis"],
                                   seed=0, tensor_id=c["tensor_id"])
                qs.append(q)
                uf.setdefault(lin["name"], {})[c["name"]] = e
                tot_ms += e["ms"]
                tot_b += e["gbs"] * e["ms"] * 1e6
            for gname, ra, rb, bf16 in GEMMS:
                M, N, K = qs[ra]["lines"], qs[rb]["lines"], qs[ra]["K"]
                C = lin["outs"][[g[0] for g in GEMMS].index(gname)]
                od = BF if bf16 else F32
                ms = _median_ms(lambda: fp4.gemm(qs[ra], qs[rb], od, out=C, workspace=ws), flush, reps)
                tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
                ug.setdefault(lin["name"], {})[gname] = {"ms": ms, "tflops": tf, "frac_fp4_over_4": tf / (fp4_peak / 4),
                                                         "shape": [M, N, K]}
                g_ms += ms
                g_flop += 2.0 * M * N * K
            del qs
        out["ufp4_layer"] = {"quantize": uf, "quantize_total_ms": tot_ms, "quantize_gbs": tot_b / (tot_ms * 1e6),
                             "quantize_frac_hbm": tot_b / (tot_ms * 1e6) / peaks["hbm"],
                             "gemm": ug, "gemm_total_ms": g_ms, "gemm_tflops": g_flop / (g_ms * 1e-3) / 1e12,
                             "gemm_frac_fp4_over_4": g_flop / (g_ms * 1e-3) / 1e12 / (fp4_peak / 4)}
        del ws
        # the same 24 UFP4 operands from 12 both-axes calls
        both_ms = 0.0
        wsb = torch.empty(256, dtype=torch.uint8, device=device)
        for lin in layer.linears:
            for b in lin["both"]:
                x = lin["t"][b["x"]]
                cr, cc = lin["calls"][b["rows"]], lin["calls"][b["cols"]]
                R, C = x.shape
                qr, qc = fp4.alloc_qtensor(R, C, UF, False, device), fp4.alloc_qtensor(C, R, UF, False, device)
                both_ms += _median_ms(lambda: fp4.quantize_both_axes(
                    x, UF, fp4.FP4_ROT_H16, seed=0, rounding_rows=cr["rounding"], tensor_id_rows=cr["tensor_id"],
                    rounding_cols=cc["rounding"], tensor_id_cols=cc["tensor_id"], out_rows=qr, out_cols=qc,
                    workspace=wsb), flush, reps)
                del qr, qc
        out["ufp4_layer"]["quantize_both_axes_total_ms"] = both_ms

    if "mxnorm" in only and layer is not None:
        # MXNorm fused with the cast ("MXNorm: Reusing MXFP block scales...":
        # up to 2.4x over RMSNorm + a separate cast on GB200) on the layer's
        # QKV input, against the cast alone (no rotation) of the same tensor
        x = layer.linears[0]["t"]["X"]
        R, C = x.shape
        ent = {}
        for fmt, name in ((MX, "mxfp4"), (NV, "nvfp4")):
            q = fp4.alloc_qtensor(R, C, fmt, device=device)
            rho = torch.empty(R, dtype=torch.float32, device=device)
            ws = torch.empty(256, dtype=torch.uint8, device=device)
            ms = _median_ms(lambda: fp4.mxnorm_quantize(x, fmt, 2, MXNORM_C2[fmt], out=q, rho=rho, workspace=ws),
                            flush, reps)
            cast = _median_ms(lambda: fp4.quantize(x, fmt, fp4.FP4_RTNE, fp4.FP4_ROT_NONE, axis=1, out=q, workspace=ws),
                              flush, reps)
            reads = 1 if fmt == MX else 2
            gb = qbytes(x.numel(), 2, fmt, reads=reads) + 4 * R
            ent[name] = {"ms": ms, "gbs": gb / (ms * 1e6), "frac_hbm": gb / (ms * 1e6) / peaks["hbm"],
                         "bytes": "%d read%s of x, codes, scales and rho written" % (reads, "s" if reads > 1 else ""),
                         "cast_alone_ms": cast, "mxnorm_over_cast": ms / cast}
        out["mxnorm_p2_qkv_input_8192x4096"] = ent

    if "outctl" in only:
        # OutControl ("TetraJet-v2" 2.C) on the QKV Fprop: calibration on X,
        # the top 10% channels in FP8 (E4M3), the rest NVFP4; split X and W,
        # then the split GEMM (two TMEM accumulators)
        d = workloads.nvfp4_fprop_qkv(seed=0)
        X, W = d["X"].to(device), d["W"].to(device)
        M, K = X.shape
        N = W.shape[0]
        ch = fp4.outctl_channels(fp4.channel_amax(X), 0.10)
        qx, qw = fp4.outctl_quantize(X, ch), fp4.outctl_quantize(W, ch)
        K8 = qx["fp8"]["K"]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        sq_x = _median_ms(lambda: fp4.outctl_quantize(X, ch, out=qx), flush, reps)
        sq_w = _median_ms(lambda: fp4.outctl_quantize(W, ch, out=qw), flush, reps)
        g = _median_ms(lambda: fp4.gemm_outctl(qx, qw, BF, out=C), flush, reps)
        flop_useful, flop_run = 2.0 * M * N * K, 2.0 * M * N * (K + K8)
        out["outcontrol_fprop_qkv_8192x6144x4096"] = {
            "channels_fp8": int(ch.numel()), "K8": int(K8),
            "split_X_ms": sq_x, "split_W_ms": sq_w,
            "split_X_gbs": (qbytes(M * K, 2, NV, reads=2) + M * K8 + 2 * M * ch.numel()) / (sq_x * 1e6),
            "gemm_ms": g, "gemm_tflops_useful": flop_useful / (g * 1e-3) / 1e12,
            "gemm_tflops_run": flop_run / (g * 1e-3) / 1e12,
            "gemm_frac_fp4_run": flop_run / (g * 1e-3) / 1e12 / fp4_peak,
            "note": "FP8 MMAs run at half the FP4 rate; 'run' counts the FP4 and FP8 MACs the kernel issues"}
        del X, W, qx, qw, C

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
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------------ oracle (CPU) arm

ORACLE_SLAB = 128


def oracle_layer_sample(host):
    """The oracle, as it stands, on a fixed sample of the layer step, and the
    step time extrapolated from it.

    Per linear: for each of the six NVFP4 + H16 operands, the rotated amax of
    its first 128 lines and the quantization of those lines given that amax
    (each extrapolated by lines / 128); for each GEMM, the dequantization of
    the two 128-line slabs and the oracle GEMM of the slabs (float64 product
    and bound), the dequantization extrapolated by (M + N) / 256 and the
    product by M N / 128^2.  Returns the extrapolated quantize and GEMM times
    (s), the wall time spent, and the work they stand for."""
    import oracle
    t_amax = t_q = t_dq = t_mm = 0.0
    quant_bytes = flop = 0.0
    wall0 = time.perf_counter()
    for index, d in enumerate(host):
        qs = []
        for role, (tn, axis, sr) in enumerate(OPERANDS):
            x = d[tn]
            R, C = x.shape
            L = R if axis == 1 else C
            slab = x[:ORACLE_SLAB] if axis == 1 else np.ascontiguousarray(x[:, :ORACLE_SLAB])
            t0 = time.perf_counter()
            a = oracle.tensor_amax(slab, axis, oracle.ROT_H16)
            t1 = time.perf_counter()
            q = oracle.quantize(x, oracle.NVFP4, rounding=oracle.SR if sr else oracle.RTNE, rotation=oracle.ROT_H16,
                                axis=axis, seed=0, tensor_id=workloads.layer_tensor_id(index, role), amax=a,
                                lines=np.arange(ORACLE_SLAB))
            t2 = time.perf_counter()
            t_amax += (t1 - t0) * L / ORACLE_SLAB
            t_q += (t2 - t1) * L / ORACLE_SLAB
            quant_bytes += qbytes(R * C, 2, 1, reads=2)
            qs.append((q, L))
        for _, ra, rb, _ in GEMMS:
            (qa, M), (qb, N) = qs[ra], qs[rb]
            K = qa["K"]
            t0 = time.perf_counter()
            oracle.dequantize(qa)
            oracle.dequantize(qb)
            t1 = time.perf_counter()
            oracle.gemm(qa, qb)
            t2 = time.perf_counter()
            dq = t1 - t0
            t_dq += dq * (M + N) / (2 * ORACLE_SLAB)
            t_mm += max(t2 - t1 - dq, 0.0) * (M * N) / (ORACLE_SLAB * ORACLE_SLAB)
            flop += 2.0 * M * N * K
    wall = time.perf_counter() - wall0
    return dict(t_quant=t_amax + t_q, t_gemm=t_dq + t_mm, wall=wall, quant_bytes=quant_bytes, flop=flop,
                t_amax=t_amax, t_q=t_q, t_dq=t_dq, t_mm=t_mm)


SAMPLE_DESC = ("per linear of the layer: the rotated amax and the NVFP4 + H16 quantization of the first %d lines "
               "of each of the 6 operands, and the oracle GEMM (exact dequantization, float64 product and bound) "
               "of %d x %d line slabs of each of the 3 GEMMs; extrapolated to the full layer step "
               "(quantize by lines, dequantization by M + N, product by M N)" % (ORACLE_SLAB, ORACLE_SLAB,
                                                                                 ORACLE_SLAB))


def oracle_baseline_entry(res, ms_per_sample=None):
    import oracle
    t_full = res["t_quant"] + res["t_gemm"]
    e = {"value": res["flop"] / t_full / 1e12, "unit": "TFLOP/s", "cores": oracle.default_threads(),
         "kind": "oracle", "sample": SAMPLE_DESC, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
         "extrapolated_step_s": t_full,
         "quantize_gbs": res["quant_bytes"] / res["t_quant"] / 1e9,
         "gemm_gflops": res["flop"] / res["t_gemm"] / 1e9,
         "quantize_bytes_are": "2 reads of the bf16 input (amax pass + quantize) + codes and scales written"}
    if ms_per_sample is not None:
        e["sample_wall_ms"] = ms_per_sample
    return e


def cpu_baseline(host, reps=3):
    """The oracle sample `reps` times; the median extrapolated step."""
    runs = [oracle_layer_sample(host) for _ in range(reps)]
    runs.sort(key=lambda r: r["t_quant"] + r["t_gemm"])
    res = runs[len(runs) // 2]
    return oracle_baseline_entry(res, statistics.median(r["wall"] for r in runs) * 1e3)


def layer_host_data(seed=0):
    return [workloads.layer_linear(name, seed=seed) for name, _, _, _ in workloads.LAYER_LINEARS]


def host_bits(host):
    return [{k: workloads.bf16_bits(v) for k, v in d.items()} for d in host]


def run_reference(args):
    """The oracle, as it stands, timed on the host cores: each step is the fixed
    sample of the layer step (oracle_layer_sample); `value` is the step's GEMM
    FLOP over the step time extrapolated from the sample, `ms_per_step` the
    measured wall time of one sampled step."""
    bits = host_bits(layer_host_data(seed=0))
    runs = []
    for i in range(args.warmup + args.steps):
        r = oracle_layer_sample(bits)
        if i >= args.warmup:
            runs.append(r)
    wall_ms = statistics.mean(r["wall"] for r in runs) * 1e3
    runs.sort(key=lambda r: r["t_quant"] + r["t_gemm"])
    res = runs[len(runs) // 2]
    base = oracle_baseline_entry(res, wall_ms)
    value = base["value"]
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall_ms, 3),
        "ms_per_step_is": "measured wall time of one sampled oracle step (not the full layer step)",
        "extrapolated_full_step_ms": round(base["extrapolated_step_s"] * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 quantizer, f64 GEMM (CPU oracle)", "data": "synthetic (same seeded workload)",
        "config": {"workload": WORKLOAD, "tokens": T,
                   "linears": {n: [d_in, d_out] for n, d_in, d_out, _ in workloads.LAYER_LINEARS},
                   "format": "NVFP4", "rotation": "H16 on all three GEMMs",
                   "rounding": "RTNE; SR on the Wgrad operands", "out": "f64"},
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fp4", "reference"], default="fp4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config kernel table")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (host copies); for profiling the device step")
    ap.add_argument("--graph", action="store_true",
                    help="time the step replayed as one CUDA graph")
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
    host = layer_host_data(seed=rank)
    line, layer = run_gpu(args, rank, world, device, host=host)
    if rank == 0:
        if world == 1 and not args.no_configs:
            from fp4_block_scaled_h16_b200 import fp4 as _fp4
            only = tuple(c for c in args.configs.split(",") if c)
            unknown = [c for c in only if c not in CONFIG_NAMES]
            if unknown:
                raise SystemExit("unknown --configs entries: %s" % ", ".join(unknown))
            line["components"].update(measure_configs(_fp4, device, measured_peaks(), layer=layer, only=only))
        del layer
        torch.cuda.empty_cache()
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(host_bits(host))
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
