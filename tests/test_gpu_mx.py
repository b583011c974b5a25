"""Parity of the MXFP8 path (OCP Microscaling v1.0 blocks of 32 along K with
E8M0 scales, e4m3 values; the tensor core applies the block scales) with the
oracle: quantizer codes and scale bytes bit-exact, GEMM outputs within the
FP8 tolerance, over every Swap-AB plan shape the library runs (grid with and
without Split-K, the Split-K reductions, persistent schedules, one or two K
slices per stage) and token counts up to 128.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from paritylib import as_u8, bf16_to_f64, check_fp8_tolerance

pytestmark = pytest.mark.gpu

F = qgd.FMT_MXFP8
SW, GRID, PERS = qgd.VARIANT_SWAP_AB, qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
LAST, ATOM, CLUS = qgd.REDUCE_LAST_CTA, qgd.REDUCE_ATOMIC, qgd.REDUCE_CLUSTER


@pytest.fixture(autouse=True)
def _clean():
    qgd.lib()
    qgd.qgd_set_override(F)
    yield
    qgd.qgd_set_override(F)


def _quant_check(x):
    xq, sx = qgd.quant_mx(x.cuda())
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_mx(x)
    np.testing.assert_array_equal(as_u8(xq), oq)
    np.testing.assert_array_equal(sx.cpu().numpy(), os_)
    return xq, sx, oq, os_


def test_quantizer_bit_exact_with_edge_blocks():
    x = synth.activations(9, 1024, 3, outliers=True)
    x[1] = 0.0                                  # all-zero blocks: scale byte 0
    x[2, :32] = 2.0 ** -130                     # tiny block: exponent clamps at -127
    x[3, 32:64] = torch.linspace(-448, 448, 32).to(torch.bfloat16)
    x[4, 64:96] = 3.0e38                        # near the bf16 maximum
    x[5] = torch.randn(1024) * 1e-20            # small values throughout
    _quant_check(x)


def test_quantizer_reads_a_column_slice():
    wide = synth.activations(5, 3072, 4, outliers=True)
    xq_v, sx_v = qgd.quant_mx(wide.cuda()[:, :2048])
    oq, os_ = oracle.quant_mx(wide[:, :2048].contiguous())
    np.testing.assert_array_equal(as_u8(xq_v), oq)
    np.testing.assert_array_equal(sx_v.cpu().numpy(), os_)


PLANS = [
    (SW, 1, LAST, 0, 0, GRID, 1, 1),
    (SW, 1, LAST, 0, 0, GRID, 1, 2),
    (SW, 4, LAST, 2, 0, GRID, 1, 2),
    (SW, 4, CLUS, 2, 0, GRID, 1, 1),
    (SW, 3, CLUS, 2, 0, GRID, 1, 2),
    (SW, 7, CLUS, 2, 0, GRID, 1, 1),
    (SW, 8, ATOM, 2, 0, GRID, 1, 1),
    (SW, 1, LAST, 2, 0, PERS, 1, 2),
    (SW, 1, LAST, 3, 0, PERS, 2, 1),
]
SHAPES = [(1, 1024, 1024), (5, 768, 2048), (16, 1024, 4096), (32, 512, 1152), (64, 512, 2048), (65, 640, 1024),
          (100, 512, 2048), (128, 1024, 1152)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"M{m}-N{n}-K{k}" for m, n, k in SHAPES])
@pytest.mark.parametrize("plan", PLANS, ids=[f"s{p[1]}-r{p[2]}-sch{p[5]}-occ{p[6]}-k{p[7]}" for p in PLANS])
def test_mx_gemm_matches_oracle(shape, plan):
    M, N, K = shape
    x = synth.activations(M, K, M + N, outliers=True)
    w = synth.weights(N, K, M + N)
    xq, sx, oxq, osx = _quant_check(x)
    wq, sw, owq, osw = _quant_check(w)
    qgd.qgd_set_override(F, *plan)
    y = qgd.qlinear_mxfp8(xq, sx, wq, sw, ws=qgd.Workspace(qgd.qgd_workspace_size(F, M, N, K)))
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 0
    yref, bound = oracle.gemm_mx(oxq, osx, owq, osw)
    p = qgd.qgd_get_plan(F, M, N, K)
    check_fp8_tolerance(bf16_to_f64(y), yref, bound, K, f"MXFP8 M={M} N={N} K={K} plan={p}")


@pytest.mark.parametrize("M", [1, 7, 32, 97, 128])
def test_mx_layer_call_from_bf16(M):
    # quantizer into the workspace, then the GEMM: the same codes and output
    N, K = 1024, 2048
    x = synth.activations(M, K, 40 + M, outliers=True)
    w = synth.weights(N, K, 40 + M)
    wq, sw, owq, osw = _quant_check(w)
    y = qgd.qlinear_bf16(F, x.cuda(), wq, sw)
    torch.cuda.synchronize()
    oxq, osx = oracle.quant_mx(x)
    yref, bound = oracle.gemm_mx(oxq, osx, owq, osw)
    check_fp8_tolerance(bf16_to_f64(y), yref, bound, K, f"MXFP8 layer call M={M}")
    xq, sx = qgd.quant_mx(x.cuda())
    y2 = qgd.qlinear_mxfp8(xq, sx, wq, sw)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_mx_rejects_what_it_does_not_cover():
    L = qgd.lib()
    import ctypes
    P = ctypes.c_void_p
    # K not a multiple of 128, more than 128 tokens: refused before any launch
    assert L.qlinear_mxfp8(P(16), P(16), P(16), P(16), P(16), 4, 512, 1056, None, 0, None) == -2
    assert L.qlinear_mxfp8(P(16), P(16), P(16), P(16), P(16), 129, 512, 1024, None, 0, None) == -2
    assert L.quant_act_mx(P(16), 4, 1000, 1000, P(16), P(16), None) == -2


@pytest.mark.parametrize("fmt", [qgd.FMT_MXFP8, qgd.FMT_NVFP4])
def test_block_scaled_128_token_plans_take_the_whole_sm(fmt):
    # 65..128 tokens: 512 tensor-memory columns, and a ring of at least four K
    # slices, which keeps one CTA per SM whatever the override asks
    for kps, stages in ((1, 2), (2, 2), (1, 0), (2, 0)):
        qgd.qgd_set_override(fmt, SW, 1, LAST, stages, 0, GRID, 1, kps)
        p = qgd.qgd_get_plan(fmt, 100, 4096, 4096)
        assert p["stages"] * p["k_slices"] >= 4, p
    qgd.qgd_set_override(fmt)
