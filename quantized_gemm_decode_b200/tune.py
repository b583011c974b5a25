"""Measure every legal plan per (format, N, K, M-bucket) on this GPU and write
the fastest to a dispatch table.

The method tunes its GEMM per layer shape and per token count (1, 2, 4, 8,
16, 24, 32) with the algorithm choice -- Standard, Split-K with split_k a
power of two up to 256, Swap-AB -- inside the search space, and it measures
candidates under CUDA-graph replay ("Building a High-Performance and
Portable vLLM Linear Backend with Helion", sections "Put algorithm selection
inside the search space", "Hybrid dispatch addresses runtime overhead" and
"Autoajuste de los kernels").  Here the space is small and discrete, so it is
searched exhaustively: variant x tile x split_k x reduction x schedule x
occupancy x K slices per stage at the deepest pipeline (and, for the
thread-block-cluster reduction and for CTA-pair tiles, other split counts,
which can fill the SMs more evenly than a power of two), then the pipeline
depth of the best few.  Each candidate is first checked against the
split-free result (bit-exact int32 accumulators for W8A8_INT8, a relative
bound for the fp32-accumulating formats), then timed as a graph of layer
calls (activation quantizer + GEMM, as the layer runs) that cycle through at
least 3x L2 of distinct weight copies.

    python -m quantized_gemm_decode_b200.tune [--formats fp8_dynamic,...] [--out tables/b200.tsv]
        [--large-m] [--resume [--recheck PCT]]

Tuning time is reported separately on stderr.  With --resume, keys already in
the output file are kept and skipped; with --recheck PCT as well, each kept
entry's plan is first timed again, and an entry now more than PCT percent
slower than the time recorded beside it (a plan measured on older kernels) is
tuned afresh.
"""
from __future__ import annotations

import argparse
import math
import os
import sys
import time

import torch

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth, workloads
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, MXFP8, NVFP4, W8A8_INT8

L2_BYTES = 126 * 1024 * 1024
FMT_ID = {FP8_DYNAMIC: 0, W8A8_INT8: 1, BLOCK_FP8: 2, MXFP8: 3, NVFP4: 4}
VAR_NAME = {0: "standard", 1: "swap_ab", 2: "standard_pair"}
RED_NAME = {0: "last_cta", 1: "two_pass", 2: "atomic", 3: "cluster"}
SCHED_NAME = {0: "grid", 1: "persistent"}


def parse_table_line(ln: str):
    """(key, plan, recorded us) of one dispatch-table line -- key (fmt, N, K,
    M bucket), plan (variant, split_k, reduce, stages, tile_n, schedule,
    occupancy, k_slices, fused) as the override calls take them, the time the
    tuner wrote beside it (None if absent) -- or None for a comment line."""
    body, _, note = ln.partition("#")
    f = body.split()
    if not f:
        return None
    if len(f) not in (11, 12, 13):
        raise ValueError(f"not a dispatch-table line: {ln!r}")
    var = {v: k for k, v in VAR_NAME.items()}[f[4]]
    red = {v: k for k, v in RED_NAME.items()}[f[6]]
    sch = {v: k for k, v in SCHED_NAME.items()}[f[9]]
    kps = int(f[11]) if len(f) > 11 else 0
    fz = int(f[12]) if len(f) > 12 else 0
    plan = (var, int(f[5]), red, int(f[7]), int(f[8]), sch, int(f[10]), kps, fz)
    us = None
    words = note.split()
    if len(words) >= 2 and words[1].rstrip(",") == "us":
        try:
            us = float(words[0])
        except ValueError:
            us = None
    return (f[0], int(f[1]), int(f[2]), int(f[3])), plan, us


def format_table_line(key, plan, us: float, gbs: float) -> str:
    """One dispatch-table line: key (fmt, N, K, M bucket), plan as
    parse_table_line returns it, and the measured time and bandwidth."""
    fmt, N, K, M = key
    var, s, r, st, t, sch, occ, kps, fz = plan
    return (f"{fmt} {N} {K} {M} {VAR_NAME[var]} {s} {RED_NAME[r]} {st} {t} {SCHED_NAME[sch]} {occ} {kps} {fz}"
            f"   # {us:.2f} us, {gbs:.0f} GB/s")


def is_stale(recorded_us, measured_us: float, pct: float) -> bool:
    """A table entry is stale when its plan now takes more than pct percent
    longer than the time recorded for it (no recorded time: stale)."""
    return recorded_us is None or measured_us > recorded_us * (1.0 + pct / 100.0)


def _quant_w(fmt, w):
    """The weight operand tuple the GEMM takes: (wq, sw), or NVFP4's (wq, sw, gw)."""
    if fmt == BLOCK_FP8:
        return qgd.quant_weight_block128(w)
    if fmt == MXFP8:
        return qgd.quant_mx(w)
    if fmt == NVFP4:
        return qgd.quant_nv(w)
    return qgd.quant_weight_per_channel(w, qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3)


def _quant_x(fmt, x):
    """The activation operand tuple: (xq, sx), or NVFP4's (xq, sx, gx)."""
    if fmt == BLOCK_FP8:
        return qgd.quant_act_group128(x)
    if fmt == MXFP8:
        return qgd.quant_mx(x)
    if fmt == NVFP4:
        return qgd.quant_nv(x)
    return qgd.quant_act_per_token(x, qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3)


SMEM_PER_SM = 233472  # bytes of shared memory per SM on sm_100 (228 KB)


def swap_mpad(M: int) -> int:
    """Token columns of the Swap-AB MMA: the next of 16, 32, 64, 128."""
    return 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128


FUSED_BYTES = 128 * 4 * 4 + 36 * 32 * 4  # the fused kernel's row maxima and group-scale ring


def two_per_sm_stages(M: int, kps: int, cluster: bool, fused: bool = False) -> int:
    """Deepest Swap-AB ring (at least 2 stages) that still lets two CTAs share an SM; 0 (the
    deepest ring, one CTA per SM) when no such ring exists."""
    mpad = swap_mpad(M)
    per_stage = kps * (128 * 128 + mpad * 128)
    fixed = (1024 + 1024 + ((128 + 8) * mpad * 4 if cluster else 0) + 1024  # alignment, control, receive buffer, reserve
             + (FUSED_BYTES if fused else 0))
    st = min(16, (SMEM_PER_SM // 2 - fixed) // per_stage)
    return st if st >= 2 else 0


def candidates(fmt: str, M: int, N: int, K: int, num_sms: int = 148, fused: bool = True):
    """(variant, split_k, reduce, tile_n, schedule, occupancy, k_slices, stages, fused) tuples legal
    for the shape; stages 0 = the deepest ring.  A Swap-AB grid with more CTAs than SMs, and the
    persistent schedule sized for two CTAs per SM, are tried at the ring depth that fits two CTAs per
    SM; a Swap-AB grid of at most one CTA per SM is tried at the deepest ring and at that shallower
    one (which leaves room for the next layer's CTAs to start streaming beside it).  At decode token
    counts every Swap-AB candidate is also tried with the activation quantizer fused in."""
    if fmt in (MXFP8, NVFP4):
        # the Swap-AB kernel only, no two-pass reduction, no fused quantizer
        return [c + (0,) for c in _candidates(fmt, M, N, K, num_sms, False) if c[0] == 1 and c[2] != 1]
    if fused and M <= 32:
        # the fused quantizer has no two-pass reduction (it would need the scales in memory)
        base = _candidates(fmt, M, N, K, num_sms, False)
        return [c + (0,) for c in base] + [c + (1,) for c in _candidates(fmt, M, N, K, num_sms, True)
                                           if c[0] == 1 and c[2] != 1]
    return [c + (0,) for c in _candidates(fmt, M, N, K, num_sms, False)]


def _candidates(fmt: str, M: int, N: int, K: int, num_sms: int, fz: bool):
    nkt = ((K // 2 if fmt == NVFP4 else K) + 127) // 128  # 128-byte K slices (NVFP4: two values per byte)
    n_tiles = (N + 127) // 128
    splits = [s for s in (1, 2, 4, 8, 16, 32, 64, 128, 256) if s <= nkt]
    out = []

    def swap_grid(s, r, kps):
        st2 = two_per_sm_stages(M, kps, r == 3, fz)
        if n_tiles * s > num_sms:
            out.append((1, s, r, 128, 0, 0, kps, st2))
        else:
            out.append((1, s, r, 128, 0, 0, kps, 0))
            if st2:
                out.append((1, s, r, 128, 0, 0, kps, st2))

    # Swap-AB: decode token counts, and up to 128 tokens for the per-token formats (the two-pass
    # reduction covers at most 32)
    swap_ok = M <= 32 or (M <= 128 and fmt != BLOCK_FP8)
    reduces = (0, 1, 2) if M <= 32 else (0, 2)
    if swap_ok:
        for kps in ((1, 2) if nkt >= 2 else (1,)):
            for r in reduces:
                # Swap-AB, persistent: one CTA per SM at the deepest ring, or two at a ring that fits
                out.append((1, 1, r, 128, 1, 1, kps, 0))
                st2 = two_per_sm_stages(M, kps, False, fz)
                if st2:
                    out.append((1, 1, r, 128, 1, 2, kps, st2))
        for s in splits:
            for r in ((0,) if s == 1 else reduces):
                swap_grid(s, r, 1)
            if nkt >= 2 and s <= (nkt + 1) // 2:
                swap_grid(s, 0, 2)  # two K slices per stage
        # the splits of a tile as one thread-block cluster (DSMEM reduction): any count 2..8
        for s in range(2, 9):
            if s <= nkt:
                swap_grid(s, 3, 1)
                if nkt >= 2 and s <= (nkt + 1) // 2:
                    swap_grid(s, 3, 2)
    tiles = (128, 256)
    # Standard: one K block per stage, and two (half the hand-offs and MMA commits) where the
    # tensor pipe is the bound
    kps_std = (1, 2) if (M > 32 and nkt >= 2) else (1,)
    for t in tiles:
        for kps in kps_std:
            nku = (nkt + kps - 1) // kps
            for s in splits:
                if (M <= 32 and s > 16) or s > nku:
                    continue  # Standard at decode sizes wastes 3/4 of each tile; prune deep splits
                for r in ((0,) if s == 1 else (0, 1, 2)):
                    out.append((0, s, r, t, 0, 0, kps, 0))
            for s in (1, 2):
                if s <= nku:
                    for r in ((0,) if s == 1 else (0, 1)):
                        out.append((0, s, r, t, 1, 0, kps, 0))  # Standard, persistent
            # the splits of a tile as one thread-block cluster (DSMEM reduction), per-token formats
            if fmt in (FP8_DYNAMIC, W8A8_INT8) and M > 32:
                for s in range(2, 9):
                    if s <= nku:
                        out.append((0, s, 3, t, 0, 0, kps, 0))
    # Standard pair tiles (256 x 256 on two SMs): the per-token formats past 128 tokens;
    # Split-K (two-pass) when the pair tiles are fewer than the SM pairs
    if fmt in (FP8_DYNAMIC, W8A8_INT8) and M > 128:
        pair_tiles = -(-M // 256) * -(-N // 256)
        for kps in kps_std:
            nku = -(-nkt // kps)
            for sched in (0, 1):
                out.append((2, 1, 0, 256, sched, 0, kps, 0))
            for s in range(2, 7):
                if s <= nku and pair_tiles < num_sms // 2:
                    out.append((2, s, 1, 256, 0, 0, kps, 0))
    return out


class Problem:
    def __init__(self, fmt, M, N, K, seed, device):
        self.fmt, self.M, self.N, self.K = fmt, M, N, K
        self.fid = FMT_ID[fmt]
        w = synth.weights(N, K, seed).to(device)
        wt = _quant_w(fmt, w)
        del w
        wbytes = N * K // 2 if fmt == NVFP4 else N * K
        ncopies = max(2, math.ceil(3 * L2_BYTES / wbytes))
        self.copies = [wt] + [tuple(t.clone() for t in wt) for _ in range(ncopies - 1)]
        x = synth.activations(M, K, seed, outliers=(fmt != W8A8_INT8)).to(device)
        self.x = x
        self.xt = _quant_x(fmt, x)
        self.xq, self.sx = self.xt[0], self.xt[1]
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.ws = qgd.Workspace(0, device)
        self.fn = {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
                   BLOCK_FP8: qgd.qlinear_block_fp8, MXFP8: qgd.qlinear_mxfp8, NVFP4: qgd.qlinear_nvfp4}[fmt]

    def run(self, j=0):
        return self.fn(*self.xt, *self.copies[j % len(self.copies)], y=self.y, ws=self.ws)

    def layer_call(self, j=0):
        """What the layer runs per call: the layer call from bf16 activations
        (quantizer kernel + GEMM, or one fused kernel, as the layer plan says)."""
        wt = self.copies[j % len(self.copies)]
        if self.fmt == MXFP8:  # the quantizer kernel, then the GEMM
            qgd.quant_mx(self.x, xq=self.xq, sx=self.sx)
            return self.run(j)
        if self.fmt == NVFP4:
            return qgd.qlinear_nvfp4_bf16(self.x, *wt, y=self.y, ws=self.ws)
        return qgd.qlinear_bf16(self.fid, self.x, *wt, y=self.y, ws=self.ws)

    def acc32(self):
        return qgd.qgd_w8a8_int8_acc32(self.xq, self.copies[0][0], ws=self.ws)

    def time_plan(self, reps=10, with_quant=True) -> float:
        """Microseconds per call of a graph of n calls (layer calls, or the
        GEMM alone), each on its own weight copy."""
        n = len(self.copies)
        call = self.layer_call if with_quant else self.run
        self.ws.ensure(max(qgd.qgd_workspace_size(self.fid, self.M, self.N, self.K),
                           qgd.qgd_layer_workspace_size(self.fid, self.M, self.N, self.K)))
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for j in range(n):
                call(j)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(n):
                call(j)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(reps):
            g.replay()
        t1.record()
        torch.cuda.synchronize()
        del g
        return t0.elapsed_time(t1) / (reps * n) * 1e3  # microseconds per call


def tune_problem(p: Problem, log=None, tp: bool = False):
    """Time every candidate, then the ring depth of the three fastest.
    Returns the best (us, variant, split_k, reduce, stages, tile_n, schedule,
    occupancy, k_slices, fused) and the first pass's results.  tp: only the
    plans a column-parallel call runs (Swap-AB, reduced inside the GEMM)."""
    fid = p.fid
    qgd.qgd_set_fused_override(fid, 0)
    qgd.qgd_set_override(fid, qgd.VARIANT_SWAP_AB if p.M <= 32 else qgd.VARIANT_STANDARD, 1, 0, 0, 0,
                         qgd.SCHEDULE_GRID, 0, 1)
    p.ws.ensure(qgd.qgd_workspace_size(fid, p.M, p.N, p.K))
    ref = p.run().float().clone()
    ref_acc = p.acc32().clone() if p.fmt == W8A8_INT8 else None
    scale = ref.abs().max().item() + 1e-30
    results = []
    num_sms = torch.cuda.get_device_properties(p.y.device).multi_processor_count

    def ensure_ws():
        p.ws.ensure(max(qgd.qgd_workspace_size(fid, p.M, p.N, p.K),
                        qgd.qgd_layer_workspace_size(fid, p.M, p.N, p.K)))

    def timed(var, s, r, st, t, sch, occ, kps, fz):
        qgd.qgd_set_override(fid, var, s, r, st, t, sch, occ, kps)
        qgd.qgd_set_fused_override(fid, fz)
        ensure_ws()
        us = p.time_plan()
        pl = qgd.qgd_get_layer_plan(fid, p.M, p.N, p.K)
        return (us, var, pl["split_k"], r, pl["stages"], t, sch, pl["occupancy"], pl["k_slices"], pl["fused"])

    cands = candidates(p.fmt, p.M, p.N, p.K, num_sms)
    if tp:
        cands = [c for c in cands if c[0] == 1 and c[2] != 1]
    for var, s, r, t, sch, occ, kps, st0, fz in cands:
        qgd.qgd_set_override(fid, var, s, r, st0, t, sch, occ, kps)
        qgd.qgd_set_fused_override(fid, fz)
        ensure_ws()
        y = p.layer_call().float()
        ok = (y - ref).abs().max().item() <= 2e-2 * scale
        if ok and ref_acc is not None:
            # exact int32 sums: every plan, fused or not, gives the same bits
            ok = torch.equal(y, ref) and torch.equal(p.acc32(), ref_acc)
        if not ok:
            if log:
                log(f"  reject {VAR_NAME[var]} s={s} r={RED_NAME[r]} t={t} {SCHED_NAME[sch]} occ={occ} "
                    f"kps={kps} fused={fz}: differs from the split-free result")
            continue
        results.append(timed(var, s, r, st0, t, sch, occ, kps, fz))
    results.sort()
    refined = list(results[:3])
    for us0, var, s, r, smax, t, sch, occ, kps, fz in results[:3]:
        for st in (2, 3, 4, 5, 6, 8, 10):  # shallower rings
            if st < smax:
                refined.append(timed(var, s, r, st, t, sch, occ, kps, fz))
    refined.sort()
    qgd.qgd_set_override(fid)
    qgd.qgd_set_fused_override(fid)
    return refined[0], results


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--formats", default="fp8_dynamic,w8a8_int8,block_fp8,mxfp8,nvfp4")
    ap.add_argument("--out", default=qgd.DEFAULT_TABLE)
    ap.add_argument("--large-m", action="store_true", help="also tune the larger-M buckets")
    ap.add_argument("--resume", action="store_true")
    ap.add_argument("--recheck", type=float, default=None, metavar="PCT",
                    help="with --resume: time each kept entry's plan again and re-tune it when it is more "
                         "than PCT percent slower than recorded")
    ap.add_argument("--only-m", default=None, help="comma-separated M values to tune")
    ap.add_argument("--tp8", action="store_true",
                    help="also tune the 8-way column-parallel shards of the 8B-class shapes (FP8_Dynamic)")
    args = ap.parse_args(argv)

    os.environ["QGD_NO_TABLE"] = "1"
    qgd.lib()
    qgd.qgd_clear_dispatch_table()
    device = torch.device("cuda")
    fmts = args.formats.split(",")
    wls = [w for w in (workloads.FP8_DECODE, workloads.INT8_DECODE, workloads.BLOCK_DECODE, workloads.MX_DECODE,
                       workloads.NV_DECODE) if w.fmt in fmts]
    if args.large_m:
        wls += [w for w in workloads.LARGE + workloads.LARGE_BS if w.fmt in fmts]
    if args.tp8:
        wls.append(workloads.FP8_TP8)
    done = {}
    if args.recheck is not None and not args.resume:
        ap.error("--recheck needs --resume (it re-times the entries of an existing table)")
    if args.resume and os.path.exists(args.out):
        for ln in open(args.out):
            parsed = parse_table_line(ln)
            if parsed is not None:
                done[parsed[0]] = ln.rstrip("\n")
    only_m = set(int(m) for m in args.only_m.split(",")) if args.only_m else None
    t_start = time.time()
    lines = dict(done)

    def log(msg):
        print(msg, file=sys.stderr, flush=True)

    def flush():
        tmp = args.out + ".tmp"
        with open(tmp, "w") as f:
            f.write("# Dispatch table for B200 (sm_100a), measured by quantized_gemm_decode_b200.tune\n")
            f.write("# fmt N K M_bucket variant split_k reduce stages tile_n schedule occupancy k_slices fused"
                    "   # us per layer call (quantize + GEMM)\n")
            for k in sorted(lines):
                f.write(lines[k] + "\n")
        os.replace(tmp, args.out)

    for wl in wls:
        for (N, K) in wl.shapes:
            for M in wl.ms:
                if only_m and M not in only_m:
                    continue
                key = (wl.fmt, N, K, M)
                p = None
                if key in done:
                    if args.recheck is None:
                        continue
                    _, plan, rec_us = parse_table_line(done[key])
                    p = Problem(wl.fmt, M, N, K, wl.seed, device)
                    qgd.qgd_set_override(p.fid, *plan[:8])
                    qgd.qgd_set_fused_override(p.fid, plan[8])
                    p.ws.ensure(max(qgd.qgd_workspace_size(p.fid, M, N, K),
                                    qgd.qgd_layer_workspace_size(p.fid, M, N, K)))
                    now_us = p.time_plan()
                    qgd.qgd_set_override(p.fid)
                    qgd.qgd_set_fused_override(p.fid)
                    if not is_stale(rec_us, now_us, args.recheck):
                        log(f"{wl.fmt} N={N} K={K} M={M}: kept ({now_us:.2f} us now, {rec_us} us recorded)")
                        del p
                        torch.cuda.empty_cache()
                        continue
                    log(f"{wl.fmt} N={N} K={K} M={M}: stale ({now_us:.2f} us now, {rec_us} us recorded), re-tuning")
                t0 = time.time()
                if p is None:
                    p = Problem(wl.fmt, M, N, K, wl.seed, device)
                best, allres = tune_problem(p, log, tp=(wl is workloads.FP8_TP8))
                us, var, s, r, st, t, sch, occ, kps, fz = best
                gbs = workloads.algorithmic_bytes(wl.fmt, M, N, K) / (us * 1e-6) / 1e9
                lines[key] = format_table_line(key, (var, s, r, st, t, sch, occ, kps, fz), us, gbs)
                log(f"{wl.fmt} N={N} K={K} M={M}: {VAR_NAME[var]} s={s} {RED_NAME[r]} st={st} t={t} "
                    f"{SCHED_NAME[sch]} occ={occ} kps={kps} fused={fz} {us:.2f} us {gbs:.0f} GB/s "
                    f"({len(allres)} candidates, {time.time() - t0:.1f} s)")
                del p
                torch.cuda.empty_cache()
                flush()
    flush()
    log(f"tuning wall time: {time.time() - t_start:.1f} s")


if __name__ == "__main__":
    main()
