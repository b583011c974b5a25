"""Parity of the NVFP4 path (E2M1 values, an E4M3 scale per 16 along K that
the tensor core applies, an fp32 scale per row that the epilogue applies)
with the oracle: packed codes, block scales and row scales bit-exact, GEMM
outputs within the FP8 tolerance, over the Swap-AB plan shapes the library
runs (grid with and without Split-K, the Split-K reductions, persistent
schedules, one or two K slices per stage) and token counts up to 64.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from paritylib import bf16_to_f64, check_fp8_tolerance

pytestmark = pytest.mark.gpu

F = qgd.FMT_NVFP4
SW, GRID, PERS = qgd.VARIANT_SWAP_AB, qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
LAST, ATOM, CLUS = qgd.REDUCE_LAST_CTA, qgd.REDUCE_ATOMIC, qgd.REDUCE_CLUSTER


@pytest.fixture(autouse=True)
def _clean():
    qgd.lib()
    qgd.qgd_set_override(F)
    yield
    qgd.qgd_set_override(F)


def _quant_check(x, gpu_x=None):
    q, s, g = qgd.quant_nv(x.cuda() if gpu_x is None else gpu_x)
    torch.cuda.synchronize()
    oq, os_, og = oracle.quant_nv(x)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)
    np.testing.assert_array_equal(g.cpu().numpy().view(np.uint32), og.view(np.uint32))
    return q, s, g, oq, os_, og


def test_quantizer_bit_exact_with_edge_rows_and_blocks():
    x = synth.activations(9, 1024, 3, outliers=True)
    x[1] = 0.0                                   # all-zero row: the amax floor, scale bytes 0, codes +0
    x[2, :16] = 0.0                              # an all-zero block in a live row
    x[2, 16] = -0.0
    x[3, 32:64] = torch.linspace(-6, 6, 32).to(torch.bfloat16)
    x[4, 64:96] = 3.0e38                         # near the bf16 maximum
    x[5] = torch.randn(1024) * 1e-20             # small values throughout
    x[6, :] = -0.0                               # negative zeros keep their sign
    x[6, 500] = 1.0
    _quant_check(x)


def test_quantizer_ties_and_saturation():
    # block maxima that make x / d land on E2M1 midpoints and past 6
    x = torch.zeros(4, 256)
    x[0, :16] = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5,
                              -5.0, -6.0])
    x[1, :16] = torch.linspace(-7, 7, 16)
    x[2] = torch.randn(256) * 100
    x[3, ::16] = 1.0
    _quant_check(x.to(torch.bfloat16))


@pytest.mark.parametrize("R,K", [(1, 256), (5, 4096), (64, 12288), (33, 640)])
def test_quantizer_bit_exact_shapes(R, K):
    _quant_check(synth.activations(R, K, R + K, outliers=True))


def test_quantizer_reads_a_column_slice():
    wide = synth.activations(5, 3072, 4, outliers=True)
    _quant_check(wide[:, :2048].contiguous(), gpu_x=wide.cuda()[:, :2048])


PLANS = [
    (SW, 1, LAST, 0, 0, GRID, 1, 1),
    (SW, 1, LAST, 0, 0, GRID, 1, 2),
    (SW, 4, LAST, 2, 0, GRID, 1, 2),
    (SW, 4, CLUS, 2, 0, GRID, 1, 1),
    (SW, 3, CLUS, 2, 0, GRID, 1, 2),
    (SW, 8, ATOM, 2, 0, GRID, 1, 1),
    (SW, 1, LAST, 2, 0, PERS, 1, 2),
    (SW, 1, LAST, 3, 0, PERS, 2, 1),
    (SW, 1, LAST, 0, 0, PERS, 1, 1),
]
SHAPES = [(1, 1024, 1024), (5, 768, 2048), (16, 1024, 4096), (32, 512, 2304), (64, 512, 2048), (65, 640, 1024),
          (100, 512, 2048), (128, 1024, 2304)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"M{m}-N{n}-K{k}" for m, n, k in SHAPES])
@pytest.mark.parametrize("plan", PLANS, ids=[f"s{p[1]}-r{p[2]}-sch{p[5]}-occ{p[6]}-k{p[7]}" for p in PLANS])
def test_nv_gemm_matches_oracle(shape, plan):
    M, N, K = shape
    x = synth.activations(M, K, M + N, outliers=True)
    w = synth.weights(N, K, M + N)
    xq, sx, gx, oxq, osx, ogx = _quant_check(x)
    wq, sw, gw, owq, osw, ogw = _quant_check(w)
    qgd.qgd_set_override(F, *plan)
    y = qgd.qlinear_nvfp4(xq, sx, gx, wq, sw, gw, ws=qgd.Workspace(qgd.qgd_workspace_size(F, M, N, K)))
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 0
    yref, bound = oracle.gemm_nv(oxq, osx, ogx, owq, osw, ogw)
    p = qgd.qgd_get_plan(F, M, N, K)
    check_fp8_tolerance(bf16_to_f64(y), yref, bound, K, f"NVFP4 M={M} N={N} K={K} plan={p}")


@pytest.mark.parametrize("M", [1, 7, 32, 64, 97, 128])
def test_nv_layer_call_from_bf16(M):
    # quantizer into the workspace, then the GEMM: the same output
    N, K = 1024, 2048
    x = synth.activations(M, K, 40 + M, outliers=True)
    w = synth.weights(N, K, 40 + M)
    wq, sw, gw, owq, osw, ogw = _quant_check(w)
    y = qgd.qlinear_nvfp4_bf16(x.cuda(), wq, sw, gw)
    torch.cuda.synchronize()
    oxq, osx, ogx = oracle.quant_nv(x)
    yref, bound = oracle.gemm_nv(oxq, osx, ogx, owq, osw, ogw)
    check_fp8_tolerance(bf16_to_f64(y), yref, bound, K, f"NVFP4 layer call M={M}")
    xq, sx, gx = qgd.quant_nv(x.cuda())
    y2 = qgd.qlinear_nvfp4(xq, sx, gx, wq, sw, gw)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_nv_rejects_what_it_does_not_cover():
    L = qgd.lib()
    import ctypes
    P = ctypes.c_void_p
    # K not a multiple of 256, more than 128 tokens: refused before any launch
    assert L.qlinear_nvfp4(P(16), P(16), P(16), P(16), P(16), P(16), P(16), 4, 512, 1152, None, 0, None) == -2
    assert L.qlinear_nvfp4(P(16), P(16), P(16), P(16), P(16), P(16), P(16), 129, 512, 1024, None, 0, None) == -2
    assert L.quant_nvfp4(P(16), 4, 1000, 1000, P(16), P(16), P(16), None) == -2
