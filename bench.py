#!/usr/bin/env python
"""Benchmark of the quantized linear-layer hot path on B200.

One step = one pass of the whole hot path over the decode sweep (for every
(M, N, K) of the workload: dynamic activation quantization, then the
quantized GEMM), replayed as one CUDA graph with inputs resident in HBM.
Weights rotate over enough copies that every call streams them from HBM
(the working set of a step is far larger than the 126 MB L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qgd|reference] [--quick]

Prints, on rank 0, the detail sections (per-call tables, larger-M rows, CPU
baseline) as lines starting with 'detail ', then the result as one compact
JSON line, always the last line of stdout.  Under torchrun each rank runs an independent
replica on its own GPU (the path has no exchange step); the reported value
is the bytes all ranks moved divided by the slowest rank's time.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from quantized_gemm_decode_b200 import synth, workloads  # noqa: E402
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, MXFP8, NVFP4, W8A8_INT8  # noqa: E402

METRIC = "achieved HBM GB/s & TFLOP/s (fraction of roofline) per format, M=1..32"
L2_BYTES = 126 * 1024 * 1024
ROTATION_BYTES = 3 * L2_BYTES  # distinct weight bytes cycled through per shape for per-call timing
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def path_bytes(fmt: str, M: int, N: int, K: int) -> int:
    """Algorithmic bytes of quantize+GEMM: bf16 X in, weight codes and scales,
    bf16 Y out (the intermediate activation codes are not counted)."""
    if fmt == NVFP4:  # half a byte per weight value, an E4M3 byte per 16, an fp32 per row
        return N * K // 2 + N * (K // 16) + 4 * N + 2 * M * K + 2 * M * N
    wscale = 4 * (N // 128) * (K // 128) if fmt == BLOCK_FP8 else (N * (K // 32) if fmt == MXFP8 else 4 * N)
    return N * K + 2 * M * K + wscale + 2 * M * N


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: a barrier and a max over timings)
# ---------------------------------------------------------------------------
class Dist:
    """Replica plumbing: one process per GPU, a barrier around the timed
    region and max/sum reductions of scalars.  NCCL on GPUs; gloo (CPU
    tensors) for the multi-process tests."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    def init(self):
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            kw = {"timeout": datetime.timedelta(seconds=120)}
            if self.backend == "nccl":
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, **kw)
            self.pg = dist

    def _tensor(self, v: float) -> torch.Tensor:
        dev = "cuda" if self.backend == "nccl" else "cpu"
        return torch.tensor([v], dtype=torch.float64, device=dev)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = self._tensor(v)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, v: float) -> float:
        if not self.pg:
            return v
        t = self._tensor(v)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def aggregate_throughput(bytes_per_rank_step: float, ms_per_step_this_rank: float, dist: Dist) -> tuple:
    """Whole-job GB/s of replicas: every rank's bytes over the slowest rank's
    time.  Returns (GB/s, max ms per step)."""
    ms = dist.max(ms_per_step_this_rank)
    total_bytes = dist.sum(bytes_per_rank_step)
    return total_bytes / (ms * 1e-3) / 1e9, ms


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.proc = None
        self.lines = []
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            self.uuid = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# the decode sweep, resident on the device
# ---------------------------------------------------------------------------
class DecodeSet:
    def __init__(self, wl: workloads.Workload, device: torch.device, keep_host: bool = False,
                 per_call_rotation: bool = True):
        import quantized_gemm_decode_b200 as qgd

        self.qgd = qgd
        self.wl, self.fmt, self.device = wl, wl.fmt, device
        self.fmt_id = {FP8_DYNAMIC: 0, W8A8_INT8: 1, BLOCK_FP8: 2, MXFP8: 3, NVFP4: 4}[wl.fmt]
        self.block_scaled = wl.fmt in (MXFP8, NVFP4)  # no fused quantizer
        self.ms = list(wl.ms)
        self.host_w = {}
        self.weights = {}  # (N, K) -> list of (wq, sw) copies
        for (N, K) in wl.shapes:
            w = synth.weights(N, K, wl.seed)
            if keep_host:
                self.host_w[(N, K)] = w
            wd = w.to(device)
            if self.fmt == BLOCK_FP8:
                wt = qgd.quant_weight_block128(wd)
            elif self.fmt == MXFP8:
                wt = qgd.quant_mx(wd)
            elif self.fmt == NVFP4:
                wt = qgd.quant_nv(wd)  # (codes, block scales, row scales)
            else:
                wt = qgd.quant_weight_per_channel(wd, qgd.QTYPE_INT8 if self.fmt == W8A8_INT8 else qgd.QTYPE_E4M3)
            del wd
            ncopies = len(self.ms)
            if per_call_rotation:
                ncopies = max(ncopies, math.ceil(ROTATION_BYTES / (N * K // (2 if self.fmt == NVFP4 else 1))))
            copies = [wt] + [tuple(t.clone() for t in wt) for _ in range(ncopies - 1)]
            self.weights[(N, K)] = copies
        self.calls = []  # per (M, N, K): dict of buffers
        ws_need = 0
        for mi, M in enumerate(self.ms):
            for (N, K) in wl.shapes:
                x = synth.activations(M, K, wl.seed, outliers=wl.outliers)
                xd = x.to(device)
                qdt = torch.int8 if self.fmt == W8A8_INT8 else torch.float8_e4m3fn
                gx = None
                if self.fmt == NVFP4:
                    xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
                    sx = torch.empty((M, K // 16), dtype=torch.uint8, device=device)
                    gx = torch.empty((M,), dtype=torch.float32, device=device)
                elif self.fmt == MXFP8:
                    xq = torch.empty((M, K), dtype=qdt, device=device)
                    sx = torch.empty((M, K // 32), dtype=torch.uint8, device=device)
                else:
                    xq = torch.empty((M, K), dtype=qdt, device=device)
                    sx = torch.empty((M, K // 128) if self.fmt == BLOCK_FP8 else (M,), dtype=torch.float32,
                                     device=device)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                self.calls.append(dict(M=M, N=N, K=K, mi=mi, x=xd, x_host=x, xq=xq, sx=sx, gx=gx, y=y))
                ws_need = max(ws_need, qgd.qgd_workspace_size(self.fmt_id, M, N, K),
                              0 if self.fmt == MXFP8 else qgd.qgd_layer_workspace_size(self.fmt_id, M, N, K))
        self.ws = qgd.Workspace(ws_need, device)
        torch.cuda.synchronize(device)

    # ---- one call --------------------------------------------------------
    def quant(self, c):
        qgd = self.qgd
        if self.fmt == BLOCK_FP8:
            qgd.quant_act_group128(c["x"], xq=c["xq"], sx=c["sx"])
        elif self.fmt == MXFP8:
            qgd.quant_mx(c["x"], xq=c["xq"], sx=c["sx"])
        elif self.fmt == NVFP4:
            qgd.quant_nv(c["x"], q=c["xq"], s=c["sx"], g=c["gx"])
        else:
            qgd.quant_act_per_token(c["x"], qgd.QTYPE_INT8 if self.fmt == W8A8_INT8 else qgd.QTYPE_E4M3,
                                    xq=c["xq"], sx=c["sx"])

    def gemm(self, c, copy_idx=None):
        qgd = self.qgd
        copies = self.weights[(c["N"], c["K"])]
        wt = copies[(c["mi"] if copy_idx is None else copy_idx) % len(copies)]
        if self.fmt == NVFP4:
            qgd.qlinear_nvfp4(c["xq"], c["sx"], c["gx"], *wt, y=c["y"], ws=self.ws)
            return
        fn = {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
              BLOCK_FP8: qgd.qlinear_block_fp8, MXFP8: qgd.qlinear_mxfp8}[self.fmt]
        fn(c["xq"], c["sx"], *wt, y=c["y"], ws=self.ws)

    def layer(self, c, copy_idx=None):
        """The layer call from bf16 activations (quantizer fused into the GEMM
        where the layer plan says so).  (MXFP8 has no layer call: its
        quantizer kernel, then its GEMM.)"""
        if self.fmt == MXFP8:
            self.quant(c)
            self.gemm(c, copy_idx)
            return
        copies = self.weights[(c["N"], c["K"])]
        wt = copies[(c["mi"] if copy_idx is None else copy_idx) % len(copies)]
        if self.fmt == NVFP4:
            self.qgd.qlinear_nvfp4_bf16(c["x"], *wt, y=c["y"], ws=self.ws)
            return
        self.qgd.qlinear_bf16(self.fmt_id, c["x"], *wt, y=c["y"], ws=self.ws)

    def step(self, gemm_only=False):
        for c in self.calls:
            if gemm_only:
                self.gemm(c)
            else:
                self.layer(c)

    def capture(self, fn) -> torch.cuda.CUDAGraph:
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize(self.device)
        return g

    def launches_per_step(self, gemm_only=False) -> int:
        """Kernels of one step: per call the GEMM, a second reduction kernel
        for two-pass Split-K, and (layer calls) the quantizer unless fused."""
        n = 0
        for c in self.calls:
            get = self.qgd.qgd_get_plan if (gemm_only or self.block_scaled) else self.qgd.qgd_get_layer_plan
            p = get(self.fmt_id, c["M"], c["N"], c["K"])
            n += (0 if gemm_only or p["fused"] else 1) + 1 + (1 if p["split_k"] > 1 and p["reduce"] == 1 else 0)
        return n

    def gemm_kernels(self):
        """The step's GEMM kernels alone: for each call the GEMM on the
        quantized activations, or -- where the layer plan fuses the quantizer
        -- the fused kernel on the bf16 activations (the same kernel the step
        runs).  Returns the algorithmic bytes those launches must move."""
        b = 0
        for c in self.calls:
            if not self.block_scaled and self.qgd.qgd_get_layer_plan(self.fmt_id, c["M"], c["N"], c["K"])["fused"]:
                self.layer(c)
                b += path_bytes(self.fmt, c["M"], c["N"], c["K"])
            else:
                self.gemm(c)
                b += workloads.algorithmic_bytes(self.fmt, c["M"], c["N"], c["K"])
        return b

    def fused_calls(self) -> int:
        if self.block_scaled:
            return 0
        return sum(self.qgd.qgd_get_layer_plan(self.fmt_id, c["M"], c["N"], c["K"])["fused"] for c in self.calls)

    def bytes_per_step(self):
        gemm = sum(workloads.algorithmic_bytes(self.fmt, c["M"], c["N"], c["K"]) for c in self.calls)
        path = sum(path_bytes(self.fmt, c["M"], c["N"], c["K"]) for c in self.calls)
        flops = sum(workloads.flops(c["M"], c["N"], c["K"]) for c in self.calls)
        return gemm, path, flops


def time_graph(g: torch.cuda.CUDAGraph, steps: int, warmup: int, dist: Dist | None = None) -> float:
    """Mean milliseconds per replay, CUDA events on the replaying stream."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        g.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def replay_times(g: torch.cuda.CUDAGraph, reps: int, warmup: int = 3) -> list:
    """Milliseconds of each of `reps` replays (CUDA events around each)."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record()
    for i in range(reps):
        g.replay()
        ev[i + 1].record()
    torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]


def per_call_table(ds: DecodeSet, peak_gbs: float, reps: int = 20):
    """Time of each call, cycling through all weight copies of its shape (at
    least 3x L2 of distinct weights), one graph per call: the GEMM alone (mean,
    median and p90 over replays) and the whole layer call (quantize + GEMM)."""
    rows = []
    for c in ds.calls:
        ncop = len(ds.weights[(c["N"], c["K"])])

        def body(c=c, ncop=ncop):
            for j in range(ncop):
                ds.gemm(c, copy_idx=j)

        def layer(c=c, ncop=ncop):
            for j in range(ncop):
                ds.layer(c, copy_idx=j)

        g = ds.capture(body)
        times = replay_times(g, reps)
        ms = statistics.mean(times) / ncop
        med = statistics.median(times) / ncop
        p90 = sorted(times)[int(0.9 * (len(times) - 1))] / ncop
        del g
        g = ds.capture(layer)
        ms_layer = statistics.mean(replay_times(g, reps)) / ncop
        del g
        b = workloads.algorithmic_bytes(ds.fmt, c["M"], c["N"], c["K"])
        f = workloads.flops(c["M"], c["N"], c["K"])
        p = ds.qgd.qgd_get_plan(ds.fmt_id, c["M"], c["N"], c["K"])
        fused = ds.qgd.qgd_get_layer_plan(ds.fmt_id, c["M"], c["N"], c["K"])["fused"]
        pb = path_bytes(ds.fmt, c["M"], c["N"], c["K"])
        rows.append({"M": c["M"], "N": c["N"], "K": c["K"], "us": round(ms * 1e3, 3), "median_us": round(med * 1e3, 3),
                     "p90_us": round(p90 * 1e3, 3),
                     "gbs": round(b / (ms * 1e-3) / 1e9, 1), "frac": round(b / (ms * 1e-3) / 1e9 / peak_gbs, 4),
                     "tflops": round(f / (ms * 1e-3) / 1e12, 2),
                     "layer_us": round(ms_layer * 1e3, 3),
                     "layer_gbs": round(pb / (ms_layer * 1e-3) / 1e9, 1),
                     "plan": (f"{('std', 'swap', 'pair')[p['variant']]}/"
                              f"{'pers' + str(p['occupancy']) if p['schedule'] == 1 else 's' + str(p['split_k'])}"
                              f"/r{p['reduce']}/st{p['stages']}/k{p['k_slices']}"),
                     "layer_fused": fused})
    return rows


def quant_bytes(fmt: str, M: int, K: int) -> int:
    """Algorithmic bytes of the activation quantizer: bf16 X in, codes and scales out."""
    if fmt == NVFP4:  # half a byte per code, an E4M3 byte per 16, an fp32 per row
        return 2 * M * K + M * K // 2 + M * (K // 16) + 4 * M
    scales = 4 * M * (K // 128) if fmt == BLOCK_FP8 else (M * (K // 32) if fmt == MXFP8 else 4 * M)
    return 2 * M * K + M * K + scales


def quantizer_summary(ds: DecodeSet, reps: int = 20):
    """The activation quantizer on its own: every call's quantizer of the
    sweep in one graph."""
    g = ds.capture(lambda: [ds.quant(c) for c in ds.calls])
    ms = statistics.mean(replay_times(g, reps))
    del g
    b = sum(quant_bytes(ds.fmt, c["M"], c["K"]) for c in ds.calls)
    return {"us_per_call": round(ms * 1e3 / len(ds.calls), 3), "bytes_per_step": b,
            "gbs": round(b / (ms * 1e-3) / 1e9, 1)}


def tensor_probe(reps: int = 3, iters: int = 8192) -> dict:
    """Dense e4m3 / int8 tensor rate of this GPU from the library's tcgen05
    peak probe (best of `reps` launches)."""
    import quantized_gemm_decode_b200 as qgd

    out = {}
    for name, qt in (("e4m3_tflops", qgd.QTYPE_E4M3), ("int8_tops", qgd.QTYPE_INT8)):
        qgd.qgd_mma_peak_probe(qt, 64)
        best = 0.0
        for _ in range(reps):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record()
            f = qgd.qgd_mma_peak_probe(qt, iters)
            t1.record()
            torch.cuda.synchronize()
            best = max(best, f / (t0.elapsed_time(t1) * 1e-3) / 1e12)
        out[name] = round(best, 1)
    # the accumulator ring: a group the issuer waits on (a slot's previous
    # group, before reusing the slot) costs about as long as an N = 256 group
    ring = {}
    for n, slots, wait in ((256, 2, 1), (128, 4, 1), (128, 4, 0)):
        qgd.qgd_mma_ring_probe(n, slots, bool(wait), 64)
        best = 0.0
        for _ in range(reps):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record()
            f = qgd.qgd_mma_ring_probe(n, slots, bool(wait), iters)
            t1.record()
            torch.cuda.synchronize()
            best = max(best, f / (t0.elapsed_time(t1) * 1e-3) / 1e12)
        ring[f"n{n}_slots{slots}_{'wait' if wait else 'nowait'}_tflops"] = round(best, 1)
    out["ring"] = ring
    assert qgd.qgd_device_error() == 0
    out["how"] = (f"qgd_mma_peak_probe: one CTA per SM, {iters} x 4 back-to-back tcgen05.mma (128x256x32) "
                  f"from shared memory, best of {reps}; ring: qgd_mma_ring_probe")
    return out


def format_summary(ds: DecodeSet, steps: int, warmup: int, peak_gbs: float):
    g = ds.capture(ds.step)
    ms = time_graph(g, steps, warmup)
    del g
    gemm_b, path_b, flops = ds.bytes_per_step()
    return {"workload": ds.wl.name, "ms_per_step": round(ms, 5),
            "gbs": round(path_b / (ms * 1e-3) / 1e9, 1), "frac": round(path_b / (ms * 1e-3) / 1e9 / peak_gbs, 4),
            "tflops": round(flops / (ms * 1e-3) / 1e12, 3)}


SPEC_TENSOR_TFLOPS = 4500.0  # dense e4m3 / int8 data-sheet figure


def large_m_summary(fmt: str, device, peaks_: dict, reps: int = 5, probe: dict | None = None):
    """Larger-M config: one GEMM per (M, N, K), timed like the decode calls --
    a graph of calls that cycle through at least 3x L2 of weight copies
    (activations stay resident), mean over `reps` replays.
    frac: against 2x the measured bf16 peak (the nominal e4m3:bf16 ratio);
    frac_probe: against the tcgen05 probe's rate for this operand type;
    frac_spec: against the 4.5 PFLOP/s data-sheet figure."""
    import quantized_gemm_decode_b200 as qgd

    wl = [w for w in workloads.LARGE + workloads.LARGE_BS if w.fmt == fmt][0]
    fmt_id = {FP8_DYNAMIC: 0, W8A8_INT8: 1, BLOCK_FP8: 2, MXFP8: 3, NVFP4: 4}[fmt]
    peak_tc = 2.0 * peaks_["bf16_tflops"]  # e4m3 / int8 dense rate = 2x bf16 (nominal ratio)
    if fmt == NVFP4:
        peak_tc *= 2.0  # e2m1: twice the e4m3 rate (nominal ratio)
    rows = []
    for (N, K) in wl.shapes:
        w = synth.weights(N, K, wl.seed).to(device)
        if fmt == BLOCK_FP8:
            wops = qgd.quant_weight_block128(w)
        elif fmt == MXFP8:
            wops = qgd.quant_mx(w)
        elif fmt == NVFP4:
            q_, s_, g_ = qgd.quant_nv(w)
            wops = (q_, s_, g_)
        else:
            wops = qgd.quant_weight_per_channel(w, qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3)
        del w
        wbytes = workloads.algorithmic_bytes(fmt, 0, N, K)
        ncop = max(2, math.ceil(ROTATION_BYTES / max(wbytes, 1)))
        copies = [wops] + [tuple(t.clone() for t in wops) for _ in range(ncop - 1)]
        for M in wl.ms:
            x = synth.activations(M, K, wl.seed, outliers=wl.outliers).to(device)
            if fmt == BLOCK_FP8:
                xops = qgd.quant_act_group128(x)
            elif fmt == MXFP8:
                xops = qgd.quant_mx(x)
            elif fmt == NVFP4:
                xops = qgd.quant_nv(x)
            else:
                xops = qgd.quant_act_per_token(x, qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            ws = qgd.Workspace(qgd.qgd_workspace_size(fmt_id, M, N, K), device)

            def call(j):
                wo = copies[j]
                if fmt == NVFP4:
                    qgd.qlinear_nvfp4(xops[0], xops[1], xops[2], wo[0], wo[1], wo[2], y=y, ws=ws)
                elif fmt == MXFP8:
                    qgd.qlinear_mxfp8(xops[0], xops[1], wo[0], wo[1], y=y, ws=ws)
                else:
                    {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
                     BLOCK_FP8: qgd.qlinear_block_fp8}[fmt](xops[0], xops[1], wo[0], wo[1], y=y, ws=ws)

            def body():
                for j in range(ncop):
                    call(j)

            s_ = torch.cuda.Stream(device)
            s_.wait_stream(torch.cuda.current_stream(device))
            with torch.cuda.stream(s_):
                body()
            torch.cuda.current_stream(device).wait_stream(s_)
            torch.cuda.synchronize(device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body()
            ms = statistics.mean(replay_times(g, reps)) / ncop
            del g
            b = workloads.algorithmic_bytes(fmt, M, N, K)
            f = workloads.flops(M, N, K)
            t_roof = max(b / (peaks_["hbm_gbs"] * 1e9), f / (peak_tc * 1e12))
            bound = "tensor" if f / (peak_tc * 1e12) > b / (peaks_["hbm_gbs"] * 1e9) else "hbm"
            p = qgd.qgd_get_plan(fmt_id, M, N, K)
            row = {"M": M, "N": N, "K": K, "us": round(ms * 1e3, 2), "tflops": round(f / (ms * 1e-3) / 1e12, 1),
                   "gbs": round(b / (ms * 1e-3) / 1e9, 1), "bound": bound,
                   "frac": round(t_roof / (ms * 1e-3), 4),
                   "frac_spec": round(max(b / (peaks_["hbm_gbs"] * 1e9), f / (SPEC_TENSOR_TFLOPS * 1e12))
                                      / (ms * 1e-3), 4),
                   "plan": (f"{('std', 'swap', 'pair')[p['variant']]}/"
                            f"{'pers' + str(p['occupancy']) if p['schedule'] == 1 else 's' + str(p['split_k'])}"
                            f"/r{p['reduce']}/st{p['stages']}/k{p['k_slices']}")}
            if probe:
                pk = probe["int8_tops"] if fmt == W8A8_INT8 else probe["e4m3_tflops"] * (2.0 if fmt == NVFP4 else 1.0)
                row["frac_probe"] = round(max(b / (peaks_["hbm_gbs"] * 1e9), f / (pk * 1e12)) / (ms * 1e-3), 4)
            rows.append(row)
            del x, xops, y, ws
        del copies, wops
        torch.cuda.empty_cache()
    return rows


def splitk_modes_table(device, ms=(1, 8, 32), reps: int = 10) -> list:
    """The Split-K reductions side by side: for each FP8_Dynamic decode shape
    and token count, the GEMM alone (a graph of calls over >= 3x L2 of weight
    copies) at one split -- the shipped plan's if it splits, else 8, rounded
    down to a power of two so that every reduction takes it -- under each
    reduction: atomic (zeroed accumulator + atomic adds, the pages' scheme
    with fp32 partials), last arriving CTA, a second kernel, and the
    thread-block cluster.  Same tile, ring and K slices for all four."""
    import quantized_gemm_decode_b200 as qgd
    from quantized_gemm_decode_b200.tune import Problem

    names = {qgd.REDUCE_ATOMIC: "atomic", qgd.REDUCE_LAST_CTA: "last_cta", qgd.REDUCE_TWO_PASS: "two_pass",
             qgd.REDUCE_CLUSTER: "cluster"}
    rows = []
    for (N, K) in workloads.FP8_DECODE.shapes:
        for M in ms:
            p = Problem(FP8_DYNAMIC, M, N, K, 1001, device)
            base = qgd.qgd_get_plan(0, M, N, K)
            split = base["split_k"] if (base["variant"] == 1 and base["schedule"] == 0 and base["split_k"] > 1) else 8
            split = 1 << (split.bit_length() - 1)
            row = {"M": M, "N": N, "K": K, "split_k": split}
            for red, name in names.items():
                qgd.qgd_set_override(0, qgd.VARIANT_SWAP_AB, split, red, 2, 0, qgd.SCHEDULE_GRID, 1, 2)
                pl = qgd.qgd_get_plan(0, M, N, K)
                if pl["reduce"] != red:
                    row[name] = None
                    continue
                row[name] = round(p.time_plan(reps=reps, with_quant=False), 2)
            qgd.qgd_set_override(0)
            rows.append(row)
            del p
            torch.cuda.empty_cache()
    return rows


def chain_table(device, reps: int = 20) -> list:
    """The dependent decode-layer chain of one 8B-class layer (qkv -> o ->
    gate_up -> down, FP8_Dynamic, each layer quantizing a column slice of an
    earlier layer's output): one graph per token count, two weight copies
    replayed alternately so every chain streams its 193 MB of weights from
    HBM.  Microseconds per chain and the whole path's GB/s."""
    from quantized_gemm_decode_b200.linear import LAYER_8B, DecodeChain, QuantizedLinear

    shapes = workloads.SHAPES_8B
    chains = []
    for c in range(2):
        layers = []
        for i, (N, K) in enumerate(shapes):
            w = synth.weights(N, K, 2001 + 10 * i + c).to(device)
            layers.append(QuantizedLinear(w, FP8_DYNAMIC))
            del w
        chains.append(DecodeChain(layers, LAYER_8B))
    rows = []
    for M in workloads.DECODE_M:
        x = synth.activations(M, shapes[0][1], 2001, outliers=True).to(device)
        for ch in chains:
            ch.input_buffer(M).copy_(x)
            ch.capture(M)
        for _ in range(3):
            for ch in chains:
                ch.run(M)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(reps):
            for ch in chains:
                ch.run(M)
        t1.record()
        torch.cuda.synchronize()
        us = t0.elapsed_time(t1) * 1e3 / (2 * reps)
        b = sum(path_bytes(FP8_DYNAMIC, M, N, K) for (N, K) in shapes)
        rows.append({"M": M, "us_per_chain": round(us, 2), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                     "bytes_per_chain": b})
    del chains
    torch.cuda.empty_cache()
    return rows


def tp_table(device, ms=(1, 32), gs=(1, 8), reps: int = 10) -> list:
    """Column-parallel layer calls on one GPU (FP8_Dynamic, 8B-class shapes):
    the share of one of G ranks -- an N/G-row weight shard -- as a plain
    layer call, and as the column-parallel call whose epilogue stores every
    element to all G full outputs (here G buffers of this GPU standing in for
    the peers' memory) and raises the flags.  At G = 1 also the call followed
    by its wait kernel.  Each a graph of calls over >= 3x L2 of weight
    copies; microseconds per call."""
    import quantized_gemm_decode_b200 as qgd
    from quantized_gemm_decode_b200.linear import quantize_weight

    F = qgd.FMT_FP8_DYNAMIC
    rows = []

    def per_call_us(fn, copies):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for c in range(copies):
                fn(c)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in range(copies):
                fn(c)
        us = time_graph(g, reps, 3) * 1e3 / copies
        del g
        return round(us, 2)

    for (N, K) in workloads.SHAPES_8B:
        for G in gs:
            n = N // G
            copies = max(3, -(-3 * L2_BYTES // (n * K)))
            wq, sw, _ = quantize_weight(synth.weights(n, K, 3001).to(device), FP8_DYNAMIC)
            wqs = [wq.clone() for _ in range(copies)]
            for M in ms:
                x = synth.activations(M, K, 3001, outliers=True).to(device)
                y = torch.empty((M, n), dtype=torch.bfloat16, device=device)
                outs = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(G)]
                flags = [torch.zeros(G + 1, dtype=torch.int32, device=device) for _ in range(G)]
                ws = qgd.Workspace(max(qgd.qgd_tp_workspace_size(F, M, n, K), qgd.qgd_layer_workspace_size(F, M, n, K)),
                                   device)

                def plain(c):
                    qgd.qlinear_bf16(F, x, wqs[c], sw, y=y, ws=ws)

                def tp(c):
                    qgd.qlinear_tp_bf16(F, x, wqs[c], sw, None, ranks=G, rank=0, col0=0, ldy=N, ys=outs,
                                        flags=flags, ws=ws)

                def tp_wait(c):
                    tp(c)
                    qgd.qgd_tp_wait(flags[0], G)

                row = {"M": M, "N": N, "K": K, "ranks": G, "shard_n": n, "layer_us": per_call_us(plain, copies),
                       "tp_us": per_call_us(tp, copies)}
                if G == 1:
                    row["tp_wait_us"] = per_call_us(tp_wait, copies)
                rows.append(row)
            del wqs, wq
            torch.cuda.empty_cache()
    if qgd.qgd_device_error() != 0:
        raise RuntimeError(f"device error {qgd.qgd_device_error()} during the column-parallel table")
    return rows


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
ORACLE_ROWS = 512  # weight rows per oracle slice (the oracle's encoder is deliberately slow)


def oracle_sample(wl: workloads.Workload, budget_s: float, host_w: dict | None = None, start: int = 0,
                  max_calls: int | None = None, cache: dict | None = None):
    """Run the oracle (dynamic X quantization + GEMM, fp64/exact int) on
    bounded slices of the workload's calls: all M tokens against the first
    ORACLE_ROWS weight rows of each shape.  The weight slices are quantized
    once (weights are static; not timed).  Returns (bytes, seconds, note)."""
    import oracle

    calls = wl.calls()
    tot_b, tot_s, done = 0, 0.0, []
    host_w = host_w if host_w is not None else {}
    cache = cache if cache is not None else {}
    i = 0
    while tot_s < budget_s and (max_calls is None or i < max_calls):
        M, N, K = calls[(start + i) % len(calls)]
        i += 1
        n_sub = min(N, ORACLE_ROWS)
        if (N, K) not in cache:
            w = host_w.get((N, K))
            if w is None:
                w = synth.weights(N, K, wl.seed)
            wsub = w[:n_sub].contiguous()
            if wl.fmt == BLOCK_FP8:
                cache[(N, K)] = oracle.quant_blocks(wsub, 128)
            else:
                cache[(N, K)] = oracle.quant_rows(wsub, oracle.INT8 if wl.fmt == W8A8_INT8 else oracle.E4M3)
        wq, sw = cache[(N, K)]
        x = synth.activations(M, K, wl.seed, outliers=wl.outliers)
        t0 = time.perf_counter()
        if wl.fmt == BLOCK_FP8:
            xq, sx = oracle.quant_groups(x, 128)
            oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
        else:
            qt = oracle.INT8 if wl.fmt == W8A8_INT8 else oracle.E4M3
            xq, sx = oracle.quant_rows(x, qt)
            oracle.gemm_rowscaled(xq, sx, wq, sw, qt)
        dt = time.perf_counter() - t0
        tot_s += dt
        tot_b += path_bytes(wl.fmt, M, n_sub, K)
        done.append(f"{M}x{n_sub}x{K}")
    note = (f"{len(done)} slices (M tokens x {ORACLE_ROWS} weight rows x K) of the sweep: "
            f"{', '.join(done[:8])}{' ...' if len(done) > 8 else ''}")
    return tot_b, tot_s, note


def oracle_large_m_sample(fmt: str = FP8_DYNAMIC, M: int = 8192, N: int = 24576, K: int = 4096,
                          rows: int = 16, cols: int = ORACLE_ROWS, seed: int = 1004):
    """The oracle on a sample of one larger-M GEMM: `rows` tokens x `cols`
    weight rows (quantize the sampled activation rows, then the product).
    Returns the sample's seconds; the full call's time is extrapolated by the
    ratio of output elements (every output costs the same K-long dot)."""
    import oracle

    w = synth.weights(cols, K, seed)
    x = synth.activations(rows, K, seed, outliers=(fmt != W8A8_INT8))
    if fmt == BLOCK_FP8:
        wq, sw = oracle.quant_blocks(w, 128)
        t0 = time.perf_counter()
        xq, sx = oracle.quant_groups(x, 128)
        oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
    else:
        qt = oracle.INT8 if fmt == W8A8_INT8 else oracle.E4M3
        wq, sw = oracle.quant_rows(w, qt)
        t0 = time.perf_counter()
        xq, sx = oracle.quant_rows(x, qt)
        oracle.gemm_rowscaled(xq, sx, wq, sw, qt)
    dt = time.perf_counter() - t0
    return dt, dt * (M * N) / (rows * cols)


def cpu_baseline_leg(wl: workloads.Workload, host_w: dict | None, budget_all: float = 10.0,
                     budget_one: float = 5.0) -> dict:
    """The oracle as it stands on this host's cores: the decode sweep sampled
    on all cores and on one thread, and one larger-M call sampled (its full
    time extrapolated, and labelled so)."""
    import oracle

    all_threads = oracle.num_threads()
    b, s, note = oracle_sample(wl, budget_all, host_w)
    oracle.set_num_threads(1)
    try:
        b1, s1, _ = oracle_sample(wl, budget_one, host_w)
        lm1, lm1_full = oracle_large_m_sample()
    finally:
        oracle.set_num_threads(all_threads)
    lm, lm_full = oracle_large_m_sample()
    return {"value": round(b / s / 1e9, 4), "unit": "GB/s", "cores": all_threads, "kind": "oracle",
            "sample": note[:160] + f"; {s:.1f} s of oracle time",
            "cpu_model": oracle.cpu_model(),
            "single_thread": {"value": round(b1 / s1 / 1e9, 4), "unit": "GB/s", "cores": 1, "seconds": round(s1, 1)},
            "large_m": {"call": "fp8_dynamic M=8192 N=24576 K=4096",
                        "sample": f"16 tokens x {ORACLE_ROWS} weight rows",
                        "sample_s": round(lm, 3), "sample_s_1_thread": round(lm1, 3),
                        "full_s_extrapolated": round(lm_full, 1),
                        "full_s_1_thread_extrapolated": round(lm1_full, 1),
                        "label": "full times extrapolated from the sample by output count, not measured"}}


HEADLINE_MAX_BYTES = 3500  # the result line stays far below what a log tail keeps


def headline(out: dict) -> dict:
    """The one-line result: the keys a reader of the run needs, compact.
    Per-call tables and per-shape larger-M rows stay in the detail record."""
    keep = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "tflops", "frac_of_hbm_peak", "frac_of_8tbs", "gpu_launches")
    line = {k: out[k] for k in keep if k in out}
    cfg = out.get("config", {})
    line["config"] = {k: cfg[k] for k in ("workload", "format", "shapes", "ms", "calls_per_step", "fused_calls", "l2",
                                          "parallelism") if k in cfg}
    rf = out.get("roofline")
    if rf:
        line["roofline"] = {k: rf[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "peak_source",
                                               "avg_launch_us", "algorithmic_bytes_per_launch") if k in rf}
    if "e2e" in out:
        line["e2e"] = {k: out["e2e"][k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step",
                                                  "ms_per_step") if k in out["e2e"]}
    if "clocks" in out:
        line["clocks"] = {k: out["clocks"].get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "power_w_max")}
    if "cpu_baseline" in out:
        cb = out["cpu_baseline"]
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "cpu_model",
                                                   "single_thread") if k in cb}
        if "large_m" in cb:
            lm = cb["large_m"]
            line["cpu_baseline"]["large_m_full_s_extrapolated"] = lm.get("full_s_extrapolated")
    if "formats" in out:
        line["formats"] = {f: {k: v[k] for k in ("gbs", "frac", "ms_per_step") if k in v} |
                           ({"quant_us": v["quantizer"]["us_per_call"]} if "quantizer" in v else {})
                           for f, v in out["formats"].items()}
    if "tensor_probe" in out:
        line["tensor_probe"] = {k: out["tensor_probe"][k] for k in ("e4m3_tflops", "int8_tops")
                                if k in out["tensor_probe"]}
    if "large_m" in out:
        summ = {}
        for f, rows in out["large_m"].items():
            big = [r for r in rows if r["M"] == max(x["M"] for x in rows)]
            summ[f] = {"M": big[0]["M"] if big else None,
                       "frac": round(statistics.mean(r["frac"] for r in big), 4) if big else None,
                       "best_tflops": max((r["tflops"] for r in big), default=None)}
            if big and "frac_probe" in big[0]:
                summ[f]["frac_probe"] = round(statistics.mean(r["frac_probe"] for r in big), 4)
        line["large_m"] = summ
    if "detail" in out:
        line["detail"] = out["detail"]
    return line


def emit(out: dict, detail_path: str | None, stream=None) -> str:
    """Print the detail sections (lines starting 'detail '), write them to
    `detail_path` if given, then print the headline as the last line."""
    stream = stream or sys.stdout
    big = {k: out[k] for k in ("per_call", "formats", "large_m", "tensor_probe", "cpu_baseline", "roofline",
                               "e2e", "splitk_modes", "chain", "fused", "tensor_parallel") if k in out}
    for k, v in big.items():
        stream.write(f"detail {k} {json.dumps(v)}\n")
    if detail_path:
        os.makedirs(os.path.dirname(os.path.abspath(detail_path)), exist_ok=True)
        with open(detail_path, "w") as f:
            json.dump(out, f, indent=1)
        out = dict(out, detail=os.path.relpath(detail_path, ROOT))
    line = json.dumps(headline(out))
    stream.write(line + "\n")
    stream.flush()
    return line


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return 0
    import oracle

    oracle.build()
    wl = workloads.FP8_DECODE
    host_w: dict = {}
    cache: dict = {}
    per_step = max(1.0, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(wl, 0.0, host_w, start=i, max_calls=1, cache=cache)
    tot_b, tot_s, notes = 0, 0.0, []
    for i in range(args.steps):
        b, s, note = oracle_sample(wl, per_step, host_w, start=args.warmup + i, cache=cache)
        tot_b += b
        tot_s += s
        notes.append(note)
    value = tot_b / tot_s / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_s / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "shapes": [list(s) for s in wl.shapes], "ms": list(wl.ms)},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": f"each step: oracle on slices of the sweep for ~{per_step:.1f} s; "
                                                         f"{notes[0] if notes else ''}"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def traffic_record():
    """Per-launch DRAM traffic of the decode GEMM from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.txt")
    if not os.path.exists(path):
        return None, None
    rec = {}
    for ln in open(path):
        if ln.strip() and not ln.startswith("#") and "=" in ln:
            k, v = ln.split("=", 1)
            rec[k.strip()] = v.strip()
    h = hashlib.sha256()
    for f in ("gemm.cu", "sm100.cuh"):
        h.update(open(os.path.join(ROOT, "quantized_gemm_decode_b200", "csrc", f), "rb").read())
    if rec.get("kernel_source_sha256") != h.hexdigest():
        return None, rec
    return rec, rec


def run_case(args):
    """One (format, M, N, K) GEMM: `warmup` + `steps` eager calls that cycle
    through >= 3x L2 of weight copies, then a graph-replay timing."""
    import quantized_gemm_decode_b200 as qgd
    from quantized_gemm_decode_b200.tune import Problem

    fmt, M, N, K = args.case.split(":")
    M, N, K = int(M), int(N), int(K)
    qgd.lib()
    p = Problem(fmt, M, N, K, 1001, torch.device("cuda"))
    p.ws.ensure(qgd.qgd_workspace_size(p.fid, M, N, K))
    for i in range(args.warmup + args.steps):
        p.run(i)
    torch.cuda.synchronize()
    us = p.time_plan(with_quant=False)
    b = workloads.algorithmic_bytes(fmt, M, N, K)
    pk = peaks()
    print(json.dumps({"case": args.case, "plan": qgd.qgd_get_plan(p.fid, M, N, K), "us": round(us, 3),
                      "gbs": round(b / (us * 1e-6) / 1e9, 1), "frac": round(b / (us * 1e-6) / 1e9 / pk["hbm_gbs"], 4),
                      "algorithmic_bytes": b}), flush=True)
    return 0


# ---------------------------------------------------------------------------
# markdown rendering of a detail record (python bench.py --report DETAIL.json)
# ---------------------------------------------------------------------------
def render_report(d: dict) -> str:
    """Markdown tables of a full run's detail record: the headline, each
    format's decode sweep, the FP8 per-call table, the larger-M results, the
    Split-K reductions, the dependent chain and the CPU baseline."""
    out = []
    rf, e2e, clk = d.get("roofline", {}), d.get("e2e", {}), d.get("clocks", {})
    out.append("| quantity | value |\n|---|---:|")
    out.append(f"| {d['config']['workload']}: whole path (quantize + GEMM per call, one graph per step) | "
               f"{d['value']:.0f} GB/s, {d['ms_per_step'] * 1e3:.0f} us per step |")
    out.append(f"| of measured HBM copy peak ({rf.get('peak')} GB/s) / of 8 TB/s | "
               f"{d.get('frac_of_hbm_peak', 0):.3f} / {d.get('frac_of_8tbs', 0):.3f} |")
    out.append(f"| GEMM kernels alone (roofline.achieved, {rf.get('avg_launch_us')} us per launch) | "
               f"{rf.get('achieved')} GB/s = {rf.get('frac')} of measured |")
    out.append(f"| end to end (pinned host X in, Y out, inside the graph) | {e2e.get('value')} GB/s |")
    out.append(f"| SM clock under load (max) / throttle reasons | {clk.get('sm_mhz')} ({clk.get('sm_max_mhz')}) MHz / "
               f"{', '.join(clk.get('reasons') or []) or 'none'} |")
    if "formats" in d:
        out.append("\n| format | workload | step | whole path | of measured HBM | quantizer alone |\n"
                   "|---|---|---:|---:|---:|---:|")
        for f, v in d["formats"].items():
            q = v.get("quantizer", {})
            out.append(f"| {f} | {v.get('workload', '')} | {v['ms_per_step'] * 1e3:.0f} us | {v['gbs']:.0f} GB/s | "
                       f"{v['frac']:.3f} | {q.get('us_per_call', '')} us/call |")
    if "per_call" in d:
        out.append("\nFP8_Dynamic per call (GEMM alone: mean / p90; layer call = quantizer + GEMM):\n")
        out.append("| M | N x K | GEMM us | p90 | GB/s | of HBM | layer us | plan |\n|---:|---|---:|---:|---:|---:|---:|---|")
        for r in d["per_call"]:
            out.append(f"| {r['M']} | {r['N']} x {r['K']} | {r['us']} | {r['p90_us']} | {r['gbs']} | {r['frac']} | "
                       f"{r['layer_us']} | {r['plan']} |")
    if "tensor_probe" in d:
        tp = d["tensor_probe"]
        ring = tp.get("ring", {})
        out.append(f"\nTensor probe (tcgen05 from shared memory, one CTA per SM): {tp.get('e4m3_tflops')} TFLOP/s e4m3, "
                   f"{tp.get('int8_tops')} TOPS int8" +
                   ("; accumulator ring: " + ", ".join(f"{k.replace('_tflops', '')} {v}" for k, v in ring.items())
                    if ring else "") + ".")
    if "large_m" in d:
        out.append("\nLarger M (one GEMM per call; frac against 2 x bf16, frac_probe against the tcgen05 probe):\n")
        out.append("| format | M | mean frac | mean frac_probe | best TFLOP/s |\n|---|---:|---:|---:|---:|")
        for f, rows in d["large_m"].items():
            for M in sorted({r["M"] for r in rows}):
                rr = [r for r in rows if r["M"] == M]
                fp = [r["frac_probe"] for r in rr if "frac_probe" in r]
                out.append(f"| {f} | {M} | {statistics.mean(r['frac'] for r in rr):.3f} | "
                           f"{(statistics.mean(fp) if fp else float('nan')):.3f} | {max(r['tflops'] for r in rr)} |")
    if "splitk_modes" in d:
        out.append("\nSplit-K reductions at one split (GEMM alone, us per call):\n")
        out.append("| M | N x K | split | atomic | last CTA | two-pass | cluster |\n|---:|---|---:|---:|---:|---:|---:|")
        for r in d["splitk_modes"]:
            out.append(f"| {r['M']} | {r['N']} x {r['K']} | {r['split_k']} | {r.get('atomic')} | {r.get('last_cta')} | "
                       f"{r.get('two_pass')} | {r.get('cluster')} |")
    if "chain" in d:
        out.append("\nDependent decode-layer chain (qkv -> o -> gate_up -> down, 8B-class, FP8_Dynamic):\n")
        out.append("| M | us per chain | whole-path GB/s |\n|---:|---:|---:|")
        for r in d["chain"]:
            out.append(f"| {r['M']} | {r['us_per_chain']} | {r['gbs']} |")
    if "tensor_parallel" in d:
        out.append("\nColumn-parallel calls on one GPU (FP8_Dynamic; one rank's N/G shard; us per call):\n")
        out.append("| M | N x K | ranks G | shard rows | layer call | column-parallel call (G outputs) | + wait |\n"
                   "|---:|---|---:|---:|---:|---:|---:|")
        for r in d["tensor_parallel"]:
            out.append(f"| {r['M']} | {r['N']} x {r['K']} | {r['ranks']} | {r['shard_n']} | {r['layer_us']} | "
                       f"{r['tp_us']} | {r.get('tp_wait_us', '')} |")
    if "cpu_baseline" in d:
        cb = d["cpu_baseline"]
        st = cb.get("single_thread", {})
        lm = cb.get("large_m", {})
        out.append(f"\nCPU baseline (the oracle, {cb.get('cpu_model', '')}): {cb['value']} GB/s on {cb['cores']} threads, "
                   f"{st.get('value')} GB/s on one; {lm.get('call', '')}: {lm.get('full_s_extrapolated')} s on all threads "
                   f"({lm.get('label', '')}).")
    return "\n".join(out) + "\n"


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("qgd", "reference"), default="qgd")
    ap.add_argument("--quick", action="store_true", help="headline workload only (no per-call table, "
                                                         "other formats, large M or CPU baseline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out", default=None, help="also write the JSON line to this file")
    ap.add_argument("--detail-out", default=None, metavar="PATH",
                    help="write the full record (per-call tables, larger-M rows, CPU baseline) to this JSON file")
    ap.add_argument("--report", default=None, metavar="DETAIL.json",
                    help="print a detail record (from --detail-out) as markdown tables and exit")
    ap.add_argument("--case", default=None, metavar="FMT:M:N:K",
                    help="time one GEMM shape (eager launches, for profilers) instead of the workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.report:
        with open(args.report) as f:
            sys.stdout.write(render_report(json.load(f)))
        return 0
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    if args.case:
        return run_case(args)

    torch.cuda.set_device(dist.local)
    device = torch.device("cuda", dist.local)
    dist.init()
    import quantized_gemm_decode_b200 as qgd

    qgd.lib()
    pk = peaks()
    wl = workloads.FP8_DECODE
    ds = DecodeSet(wl, device, keep_host=(dist.rank == 0 and not args.quick))
    gemm_b, path_b, flops = ds.bytes_per_step()

    # ---- headline: the whole hot path, one graph per step ----------------
    g_step = ds.capture(ds.step)
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    # keep the GPU busy while the sampler starts, so samples cover load
    t_end = time.time() + 0.4
    while time.time() < t_end:
        for _ in range(20):
            g_step.replay()
        torch.cuda.synchronize()
    ms_step_local = time_graph(g_step, args.steps, 0, dist)
    clk = clocks.stop()
    value, ms_step = aggregate_throughput(path_b, ms_step_local, dist)

    # ---- the dominant kernel (the GEMM, fused or not), same calls ---------
    kern_b = [0]
    g_gemm = ds.capture(lambda: kern_b.__setitem__(0, ds.gemm_kernels()))
    ms_gemm = dist.max(time_graph(g_gemm, max(args.steps, 50), args.warmup, dist))
    del g_gemm
    gemm_b = kern_b[0]

    # ---- e2e: the public layer API with pinned host buffers ---------------
    # every step copies its activations in from pinned host memory and its
    # results back out, inside the captured decode step
    from quantized_gemm_decode_b200.linear import DecodeStep, QuantizedLinear

    calls, xh, yh = [], [], []
    for c in ds.calls:
        wq, sw = ds.weights[(c["N"], c["K"])][c["mi"]]
        calls.append((QuantizedLinear(None, wl.fmt, wq=wq, sw=sw), c["M"]))
        xh.append(c["x_host"].pin_memory())
        yh.append(torch.empty((c["M"], c["N"]), dtype=torch.bfloat16).pin_memory())
    step = DecodeStep(calls, xh, yh)
    for _ in range(args.warmup):
        step.replay()
    torch.cuda.synchronize()
    dist.barrier()
    e2e_steps = max(20, min(args.steps, 200))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(e2e_steps):
        step.replay()
    t1.record()
    torch.cuda.synchronize()
    ms_e2e = dist.max(t0.elapsed_time(t1) / e2e_steps)
    h2d = sum(x.numel() * x.element_size() for x in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh)
    # the last step's results reached the host: check one against the device copy
    assert torch.equal(yh[-1].view(torch.int16), step.y_dev[-1].cpu().view(torch.int16))
    del step, calls

    world = dist.world
    gemm_gbs = gemm_b / (ms_gemm * 1e-3) / 1e9
    launches = ds.launches_per_step() * args.steps

    extra = {}
    if not args.quick:
        extra["per_call"] = per_call_table(ds, pk["hbm_gbs"])
    traffic, _rec = traffic_record()

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": wl.name, "format": wl.fmt, "shapes": [list(s) for s in wl.shapes], "ms": list(wl.ms),
                   "calls_per_step": len(ds.calls), "fused_calls": ds.fused_calls(),
                   "graph": "one CUDA graph per step (one layer call per (M, N, K): quantize + GEMM, "
                            "fused into one kernel where the tuned plan says so)",
                   "l2": f"inputs larger than L2: each call reads its own weight copy; "
                         f"{sum(len(v) for v in ds.weights.values())} copies, "
                         f"{path_b * 1e-9:.3f} GB streamed per step vs 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "tflops": round(flops * world / (ms_step * 1e-3) / 1e12, 3),
        "frac_of_hbm_peak": round(value / world / pk["hbm_gbs"], 4),
        "frac_of_8tbs": round(value / world / 8000.0, 4),
        "roofline": {"bound": "hbm",
                     "kernel": f"GEMM (swapab/standard, all calls of the sweep; {ds.fused_calls()} of {len(ds.calls)} "
                               f"with the activation quantizer fused in, counted with bf16 activations in)",
                     "achieved": round(gemm_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gemm_gbs / pk["hbm_gbs"], 4), "peak_source": pk["source"],
                     # DRAM bytes per launch: the captured case's DRAM/algorithmic ratio
                     # times this workload's algorithmic bytes per launch
                     "traffic": (round(float(traffic["dram_over_algorithmic"]) * gemm_b / len(ds.calls))
                                 if traffic else None),
                     "traffic_case": (traffic.get("case") if traffic else None),
                     "avg_launch_us": round(ms_gemm * 1e3 / len(ds.calls), 3),
                     "algorithmic_bytes_per_launch": round(gemm_b / len(ds.calls))},
        "e2e": {"value": round(path_b * world / (ms_e2e * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 4),
                "how": "linear.DecodeStep: one graph per step; pinned host X -> device on a copy stream "
                       "(the compute stream joins them once per 4 layers), quantize + GEMM per layer, "
                       "Y -> pinned host on a second copy stream"},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if not args.quick:
        fmts = {}
        del g_step
        fmts[FP8_DYNAMIC] = {"workload": wl.name, "ms_per_step": round(ms_step, 5), "gbs": round(value / world, 1),
                             "frac": round(value / world / pk["hbm_gbs"], 4),
                             "quantizer": quantizer_summary(ds)}
        keep = ds
        for wl2 in (workloads.INT8_DECODE, workloads.BLOCK_DECODE, workloads.MX_DECODE, workloads.NV_DECODE):
            ds2 = DecodeSet(wl2, device, per_call_rotation=True)
            fmts[wl2.fmt] = format_summary(ds2, args.steps, args.warmup, pk["hbm_gbs"])
            fmts[wl2.fmt]["quantizer"] = quantizer_summary(ds2)
            fmts[wl2.fmt]["per_call"] = per_call_table(ds2, pk["hbm_gbs"])
            del ds2
            torch.cuda.empty_cache()
        out["formats"] = fmts
        probe = tensor_probe()
        out["tensor_probe"] = probe
        out["large_m"] = {f: large_m_summary(f, device, pk, probe=probe)
                          for f in (FP8_DYNAMIC, W8A8_INT8, BLOCK_FP8, MXFP8, NVFP4)}
        out["splitk_modes"] = splitk_modes_table(device)
        out["chain"] = chain_table(device)
        out["tensor_parallel"] = tp_table(device)
        out.update(extra)
        ds = keep
    if dist.rank == 0 and dist.world == 1 and not args.quick and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_leg(wl, ds.host_w)
    if dist.rank == 0:
        line = emit(out, args.detail_out)
        if args.out:
            with open(args.out, "w") as f:
                f.write(line + "\n")
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
