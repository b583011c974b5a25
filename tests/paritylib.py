"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare at the stated bars.

Bars:
  * quantized bytes and scales: bit-exact;
  * W8A8_INT8 int32 accumulators: bit-exact;
  * W8A8_INT8 bf16 output: within one bf16 ulp of the oracle's fp32 result;
  * FP8 outputs (FP8_Dynamic, Block_FP8):
        |y - y_ref| <= 1e-2 |y_ref| + 2e-3 * (sum_k |x^_k||w^_k|) / sqrt(K)
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, W8A8_INT8

FMT_ID = {FP8_DYNAMIC: qgd.FMT_FP8_DYNAMIC, W8A8_INT8: qgd.FMT_W8A8_INT8, BLOCK_FP8: qgd.FMT_BLOCK_FP8}


def as_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.abs(v.astype(np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), 0.0)


def check_fp8_tolerance(y: np.ndarray, yref: np.ndarray, bound: np.ndarray, K: int, what: str = "") -> float:
    tol = 1e-2 * np.abs(yref) + 2e-3 * bound / math.sqrt(K)
    err = np.abs(y - yref)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"y={y[i]!r} ref={yref[i]!r} tol={tol[i]!r}")
    return float((err / np.maximum(tol, 1e-30)).max())


def check_within_one_ulp(y: np.ndarray, yref: np.ndarray, what: str = "") -> None:
    ref32 = yref.astype(np.float32).astype(np.float64)
    err = np.abs(y - ref32)
    ulp = bf16_ulp(ref32)
    bad = err > ulp
    if bad.any():
        i = np.unravel_index(np.argmax(err - ulp), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} beyond 1 bf16 ulp; worst at {i}: "
                             f"y={y[i]!r} ref32={ref32[i]!r} ulp={ulp[i]!r}")


class Case:
    """One (format, M, N, K) problem: inputs, GPU-quantized operands and the
    oracle's own quantization of the same inputs."""

    def __init__(self, fmt: str, M: int, N: int, K: int, seed: int = 0, outliers: bool = True,
                 x: torch.Tensor | None = None, w: torch.Tensor | None = None):
        self.fmt, self.M, self.N, self.K = fmt, M, N, K
        self.x = x if x is not None else synth.activations(M, K, seed, outliers=outliers)
        self.w = w if w is not None else synth.weights(N, K, seed)
        dev = torch.device("cuda")
        self.xd = self.x.to(dev)
        self.wd = self.w.to(dev)
        if fmt == BLOCK_FP8:
            self.xq, self.sx = qgd.quant_act_group128(self.xd)
            self.wq, self.sw = qgd.quant_weight_block128(self.wd)
        else:
            qt = qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3
            self.xq, self.sx = qgd.quant_act_per_token(self.xd, qt)
            self.wq, self.sw = qgd.quant_weight_per_channel(self.wd, qt)
        torch.cuda.synchronize()

    # ---- oracle side -------------------------------------------------
    def oracle_quant(self, rows: np.ndarray | None = None):
        """Oracle quantization of X and of W (all rows, or the given row band
        start indices for block scaling / row indices for per-channel)."""
        if self.fmt == BLOCK_FP8:
            xq, sx = oracle.quant_groups(self.x, 128)
            wq, sw = oracle.quant_blocks(self.w if rows is None else self.w[rows], 128)
        else:
            qt = oracle.INT8 if self.fmt == W8A8_INT8 else oracle.E4M3
            xq, sx = oracle.quant_rows(self.x, qt)
            wq, sw = oracle.quant_rows(self.w if rows is None else self.w[rows], qt)
        return xq, sx, wq, sw

    def oracle_gemm(self, xq, sx, wq, sw, want_acc=False):
        if self.fmt == BLOCK_FP8:
            return oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
        qt = oracle.INT8 if self.fmt == W8A8_INT8 else oracle.E4M3
        return oracle.gemm_rowscaled(xq, sx, wq, sw, qt, want_acc=want_acc)

    # ---- CUDA side ---------------------------------------------------
    def run(self, ws=None) -> torch.Tensor:
        fn = {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
              BLOCK_FP8: qgd.qlinear_block_fp8}[self.fmt]
        y = fn(self.xq, self.sx, self.wq, self.sw, ws=ws)
        torch.cuda.synchronize()
        return y

    def check_output(self, y: torch.Tensor, yref: np.ndarray, bound: np.ndarray, what: str = "") -> None:
        yy = bf16_to_f64(y)
        if self.fmt == W8A8_INT8:
            check_within_one_ulp(yy, yref, what)
        else:
            check_fp8_tolerance(yy, yref, bound, self.K, what)
