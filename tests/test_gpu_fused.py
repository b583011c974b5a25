"""Parity of the layer calls from bf16 activations (qlinear_*_bf16), with the
activation quantizer fused into the Swap-AB GEMM and without.

For each format and a spread of plans (grid schedule with and without
Split-K, the cluster reduction, persistent schedules whose CTAs cover
several tiles, one or two K slices per stage), the fused kernel's own
activation codes and scales -- written out through the capture hook -- are
compared bit for bit with the oracle's quantization of the same bf16
input, and Y with the oracle at the usual bars.  The fused and unfused
layer calls under the same plan quantize identically and accumulate in the
same order, so their outputs must agree bit for bit as well.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, W8A8_INT8
from paritylib import FMT_ID, Case, as_u8

pytestmark = pytest.mark.gpu

SW, GRID, PERS = qgd.VARIANT_SWAP_AB, qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
LAST, TWO, ATOM, CLUS = qgd.REDUCE_LAST_CTA, qgd.REDUCE_TWO_PASS, qgd.REDUCE_ATOMIC, qgd.REDUCE_CLUSTER


@pytest.fixture(autouse=True)
def _clean():
    qgd.lib()
    for f in range(3):
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f)
    qgd.qgd_test_capture_fused(None, None)
    yield
    qgd.qgd_test_capture_fused(None, None)
    for f in range(3):
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f)


def _layer(case, x=None):
    return qgd.qlinear_bf16(FMT_ID[case.fmt], case.xd if x is None else x, case.wq, case.sw)


def _run_fused_and_check(case, plan, x=None):
    fid = FMT_ID[case.fmt]
    qgd.qgd_set_override(fid, *plan)
    qgd.qgd_set_fused_override(fid, 1)
    lp = qgd.qgd_get_layer_plan(fid, case.M, case.N, case.K)
    assert lp["fused"] == 1 and lp["variant"] == SW, lp
    xq = torch.full((case.M, case.K), 0x5A, dtype=torch.uint8, device="cuda")
    nsx = (case.M, case.K // 128) if case.fmt == BLOCK_FP8 else (case.M,)
    sx = torch.full(nsx, float("nan"), dtype=torch.float32, device="cuda")
    qgd.qgd_test_capture_fused(xq, sx)
    y = _layer(case, x)
    torch.cuda.synchronize()
    qgd.qgd_test_capture_fused(None, None)
    assert qgd.qgd_device_error() == 0
    oxq, osx, owq, osw = case.oracle_quant()
    np.testing.assert_array_equal(xq.cpu().numpy(), oxq.view(np.uint8), err_msg=f"fused codes, plan {lp}")
    np.testing.assert_array_equal(sx.cpu().numpy(), osx, err_msg=f"fused scales, plan {lp}")
    yref, bound = case.oracle_gemm(oxq, osx, owq, osw)
    case.check_output(y, yref, bound, f"fused {case.fmt} M={case.M} N={case.N} K={case.K} plan={lp}")
    # the same plan unfused: quantizer kernel + GEMM.  Same bits, except that
    # atomic fp32 Split-K adds the partials in a varying order
    qgd.qgd_set_fused_override(fid, 0)
    y2 = _layer(case, x)
    torch.cuda.synchronize()
    if lp["reduce"] == ATOM and lp["split_k"] > 1 and case.fmt != W8A8_INT8:
        case.check_output(y2, yref, bound, f"unfused, plan {lp}")
    else:
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"fused and unfused differ, plan {lp}"
    return y


# (variant, split_k, reduce, stages, tile_n, schedule, occupancy, k_slices)
PLANS = [
    (SW, 1, LAST, 0, 0, GRID, 1, 1),
    (SW, 1, LAST, 0, 0, GRID, 1, 2),
    (SW, 4, LAST, 2, 0, GRID, 1, 2),
    (SW, 4, CLUS, 2, 0, GRID, 1, 1),
    (SW, 8, ATOM, 2, 0, GRID, 1, 1),
    (SW, 1, LAST, 2, 0, PERS, 1, 2),
    (SW, 1, LAST, 3, 0, PERS, 2, 1),
]
SHAPES = [(1, 1024, 1024), (3, 768, 2048), (16, 1024, 4096), (32, 512, 1152), (5, 512, 1040)]


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8, BLOCK_FP8])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"M{m}-N{n}-K{k}" for m, n, k in SHAPES])
@pytest.mark.parametrize("plan", PLANS, ids=[f"s{p[1]}-r{p[2]}-sch{p[5]}-occ{p[6]}-k{p[7]}" for p in PLANS])
def test_fused_layer_call_matches_oracle(fmt, shape, plan):
    M, N, K = shape
    if fmt == BLOCK_FP8 and K % 128:
        pytest.skip("Block_FP8 needs K % 128 == 0")
    case = Case(fmt, M, N, K, seed=7 * M + N + K + FMT_ID[fmt], outliers=(fmt != W8A8_INT8))
    _run_fused_and_check(case, plan)


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("M", [48, 64, 100, 128])
def test_fused_wide_token_counts(fmt, M):
    # 64- and 128-token MMAs (per-token formats only), read 32 tokens at a time
    case = Case(fmt, M, 512, 2048, seed=M, outliers=(fmt != W8A8_INT8))
    _run_fused_and_check(case, (SW, 2, LAST, 0, 0, GRID, 1, 2))


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, BLOCK_FP8])
def test_fused_persistent_ctas_spanning_three_tiles(fmt):
    # 304 tiles x 2 K units over the SMs: every CTA's range crosses tile
    # boundaries, so the quantizer runs ahead across segments
    case = Case(fmt, 8, 38912, 256, seed=5)
    _run_fused_and_check(case, (SW, 1, LAST, 2, 0, PERS, 1, 1))


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8, BLOCK_FP8])
def test_fused_reads_a_column_slice(fmt):
    M, N, K = 5, 1024, 2048
    wide = synth.activations(M, 3072, 9, outliers=True)
    x = wide[:, :K].contiguous()
    case = Case(fmt, M, N, K, seed=9, x=x)
    xv = wide.cuda()[:, :K]  # rows 3072 elements apart
    assert xv.stride(0) == 3072
    _run_fused_and_check(case, (SW, 2, LAST, 0, 0, GRID, 1, 1), x=xv)


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, BLOCK_FP8])
def test_fused_zero_rows_and_ties(fmt):
    M, N, K = 6, 512, 1024
    x = synth.activations(M, K, 11, outliers=False)
    x[2] = 0.0                      # all-zero row: every code 0, scale from the floor
    x[4, :128] = 0.0                # an all-zero 1x128 group
    x[5] = torch.linspace(-3, 3, K).to(torch.bfloat16)
    case = Case(fmt, M, N, K, seed=11, x=x)
    _run_fused_and_check(case, (SW, 1, LAST, 0, 0, GRID, 1, 2))


def test_layer_workspace_covers_the_unfused_path():
    case = Case(FP8_DYNAMIC, 8, 1024, 4096, seed=3)
    fid = FMT_ID[FP8_DYNAMIC]
    qgd.qgd_set_override(fid, SW, 4, LAST, 2, 0, GRID, 1, 2)
    qgd.qgd_set_fused_override(fid, 0)
    need = qgd.qgd_layer_workspace_size(fid, 8, 1024, 4096)
    assert need >= qgd.qgd_workspace_size(fid, 8, 1024, 4096) + 8 * 4096
    with pytest.raises(qgd.QGDError) as e:
        qgd.qlinear_bf16(fid, case.xd, case.wq, case.sw,
                         ws=torch.zeros(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == -3
    y = qgd.qlinear_bf16(fid, case.xd, case.wq, case.sw, ws=qgd.Workspace(need))
    torch.cuda.synchronize()
    yref, bound = case.oracle_gemm(*case.oracle_quant())
    case.check_output(y, yref, bound, "unfused layer call")


def test_layer_calls_leave_the_counter_header_zero():
    # an unfused layer call whose GEMM needs no workspace still keeps its
    # activation codes out of the counter header, so a Split-K call sharing
    # the workspace afterwards starts from zeroed counters
    fid = FMT_ID[FP8_DYNAMIC]
    ws = qgd.Workspace(8 << 20)
    a = Case(FP8_DYNAMIC, 16, 1024, 4096, seed=31)
    qgd.qgd_set_override(fid, SW, 1, LAST, 0, 0, GRID, 1, 1)
    qgd.qgd_set_fused_override(fid, 0)
    qgd.qlinear_bf16(fid, a.xd, a.wq, a.sw, ws=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws.buf[:65536]).item() == 0
    qgd.qgd_set_override(fid, SW, 4, LAST, 2, 0, GRID, 1, 2)
    y = qgd.qlinear_fp8_dynamic(a.xq, a.sx, a.wq, a.sw, ws=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws.buf[:65536]).item() == 0
    yref, bound = a.oracle_gemm(*a.oracle_quant())
    a.check_output(y, yref, bound, "split call after a layer call on the same workspace")
