"""Parity at the full workload sizes, in the launch configuration the
benchmark times (the shipped dispatch table, no overrides).

For every (N, K) of the three decode sweeps, at a few token counts, the GPU
computes the whole Y; the oracle computes a sample of it -- all M tokens
against 128-row bands of weight rows: the first and the last, and two
interior bands where the plan's work partition puts CTA boundaries inside a
tile (so tiles summed from several CTAs' partials are compared at full size),
whole bands so Block_FP8's 128 x 128 weight scales are the oracle's own --
from the same seeded inputs,
quantizing them itself.  The larger-M set is sampled in both tokens and
weight rows.  Bars as everywhere: bit-exact codes and scales, one bf16 ulp
for W8A8_INT8, the FP8 tolerance otherwise.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth, workloads
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, MXFP8, W8A8_INT8
from paritylib import as_u8, bf16_to_f64, check_fp8_tolerance, check_within_one_ulp

pytestmark = pytest.mark.gpu

DECODE = (workloads.FP8_DECODE, workloads.INT8_DECODE, workloads.BLOCK_DECODE, workloads.MX_DECODE)
FMT_ID = {FP8_DYNAMIC: 0, W8A8_INT8: 1, BLOCK_FP8: 2, MXFP8: 3}
CASES = [(wl, n, k, m) for wl in DECODE for (n, k) in wl.shapes for m in (1, 17, 32)]


@pytest.fixture(scope="module", autouse=True)
def shipped_table():
    qgd.lib()
    for f in range(4):
        qgd.qgd_set_override(f)
    if qgd.DEFAULT_TABLE:
        qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
    yield


_weights = {}


def _weights_for(wl, N, K):
    key = (wl.fmt, N, K)
    if key not in _weights:
        _weights.clear()  # one shape at a time: the largest is 262 M elements
        w = synth.weights(N, K, wl.seed)
        wd = w.cuda()
        if wl.fmt == BLOCK_FP8:
            wq, sw = qgd.quant_weight_block128(wd)
        elif wl.fmt == MXFP8:
            wq, sw = qgd.quant_mx(wd)
        else:
            wq, sw = qgd.quant_weight_per_channel(wd, qgd.QTYPE_INT8 if wl.fmt == W8A8_INT8 else qgd.QTYPE_E4M3)
        del wd
        _weights[key] = (w, wq, sw)
    return _weights[key]


def _quant_x(fmt, x):
    if fmt == BLOCK_FP8:
        return qgd.quant_act_group128(x)
    if fmt == MXFP8:
        return qgd.quant_mx(x)
    return qgd.quant_act_per_token(x, qgd.QTYPE_INT8 if fmt == W8A8_INT8 else qgd.QTYPE_E4M3)


def _gemm(fmt, xq, sx, wq, sw):
    fn = {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
          BLOCK_FP8: qgd.qlinear_block_fp8, MXFP8: qgd.qlinear_mxfp8}[fmt]
    return fn(xq, sx, wq, sw)


_oracle_w = {}


def _oracle_sample(fmt, x_rows, w_rows, wkey):
    """Oracle on sampled tokens x sampled weight rows; the weight rows'
    quantization is cached per (shape, rows)."""
    if wkey not in _oracle_w:
        _oracle_w.clear()
        if fmt == BLOCK_FP8:
            _oracle_w[wkey] = oracle.quant_blocks(w_rows, 128)
        elif fmt == MXFP8:
            _oracle_w[wkey] = oracle.quant_mx(w_rows)
        else:
            _oracle_w[wkey] = oracle.quant_rows(w_rows, oracle.INT8 if fmt == W8A8_INT8 else oracle.E4M3)
    wq, sw = _oracle_w[wkey]
    if fmt == BLOCK_FP8:
        xq, sx = oracle.quant_groups(x_rows, 128)
        y, bound = oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
    elif fmt == MXFP8:
        xq, sx = oracle.quant_mx(x_rows)
        y, bound = oracle.gemm_mx(xq, sx, wq, sw)
    else:
        qt = oracle.INT8 if fmt == W8A8_INT8 else oracle.E4M3
        xq, sx = oracle.quant_rows(x_rows, qt)
        y, bound = oracle.gemm_rowscaled(xq, sx, wq, sw, qt)
    return xq, wq, y, bound


def _check(fmt, y_gpu, y_ref, bound, K, what):
    if fmt == W8A8_INT8:
        check_within_one_ulp(y_gpu, y_ref, what)
    else:
        check_fp8_tolerance(y_gpu, y_ref, bound, K, what)


def _interior_bands(plan: dict, M: int, N: int, K: int) -> list:
    """Two interior 128-row weight bands that several CTAs contribute to.
    Persistent Swap-AB deals the (tile, K unit) units out in equal contiguous
    ranges, CTA c taking [c*U/G, (c+1)*U/G): the first two ranges that start
    inside a tile give the bands.  Other plans split every tile alike; the
    bands are then one third and two thirds of the way along N."""
    n_tiles = N // 128
    if plan["variant"] == qgd.VARIANT_SWAP_AB and plan["schedule"] == qgd.SCHEDULE_PERSISTENT:
        nkt = (K + 127) // 128
        nku = (nkt + plan["k_slices"] - 1) // plan["k_slices"]
        U = n_tiles * nku
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        G = min(U, sms * plan["occupancy"])
        found = []
        for c in range(1, G):
            start = c * U // G
            if start % nku and start // nku not in found and 0 < start // nku < n_tiles - 1:
                found.append(start // nku)
            if len(found) == 2:
                return found
        if found:
            return found
    return sorted({max(1, n_tiles // 3), max(1, (2 * n_tiles) // 3)} - {0, n_tiles - 1}) or [0]


@pytest.mark.parametrize("wl,N,K,M", CASES, ids=[f"{wl.fmt}-{n}x{k}-M{m}" for wl, n, k, m in CASES])
def test_decode_full_size_sampled(wl, N, K, M):
    w, wq, sw = _weights_for(wl, N, K)
    x = synth.activations(M, K, wl.seed, outliers=wl.outliers)
    xq, sx = _quant_x(wl.fmt, x.cuda())
    y = bf16_to_f64(_gemm(wl.fmt, xq, sx, wq, sw))
    torch.cuda.synchronize()
    plan = qgd.qgd_get_plan(FMT_ID[wl.fmt], M, N, K)
    bands = sorted(set([0, N // 128 - 1] + _interior_bands(plan, M, N, K)))
    rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in bands])
    oxq, owq, y_ref, bound = _oracle_sample(wl.fmt, x, w[torch.from_numpy(rows)],
                                            (wl.fmt, N, K, "decode", tuple(bands)))
    np.testing.assert_array_equal(as_u8(xq), oxq.view(np.uint8))
    np.testing.assert_array_equal(as_u8(wq[torch.from_numpy(rows).cuda()]), owq.view(np.uint8))
    _check(wl.fmt, y[:, rows], y_ref, bound, K, f"{wl.fmt} M={M} N={N} K={K} bands={bands} plan={plan}")


LARGE = [(wl, n, k, m) for wl in workloads.LARGE for (n, k) in wl.shapes[:2] for m in (64, 512, 2048)]


@pytest.mark.parametrize("wl,N,K,M", LARGE, ids=[f"{wl.fmt}-{n}x{k}-M{m}" for wl, n, k, m in LARGE])
def test_large_m_full_size_sampled(wl, N, K, M):
    w, wq, sw = _weights_for(wl, N, K)
    x = synth.activations(M, K, wl.seed, outliers=wl.outliers)
    xq, sx = _quant_x(wl.fmt, x.cuda())
    y = bf16_to_f64(_gemm(wl.fmt, xq, sx, wq, sw))
    torch.cuda.synchronize()
    toks = np.unique(np.concatenate([np.arange(0, M, max(1, M // 12)), [M - 1]]))
    bands = [0, N // 256, N // 128 - 1]
    rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in bands])
    _, _, y_ref, bound = _oracle_sample(wl.fmt, x[torch.from_numpy(toks)], w[torch.from_numpy(rows)],
                                        (wl.fmt, N, K, "large"))
    _check(wl.fmt, y[np.ix_(toks, rows)], y_ref, bound, K, f"{wl.fmt} M={M} N={N} K={K}")
