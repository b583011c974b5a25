"""GPU parity of the quantized GEMMs against the oracle, per algorithm variant.

Every variant (Swap-AB / Standard, split_k, reduction mode) is forced through
qgd_set_override and compared with the oracle on the same seeded inputs:
INT8 accumulators bit-exact, INT8 bf16 output within one ulp of the oracle's
fp32 value, FP8 outputs within the stated tolerance.
"""
import numpy as np
import pytest
import torch

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, W8A8_INT8
from paritylib import FMT_ID, Case, as_u8, bf16_to_f64, check_fp8_tolerance, check_within_one_ulp

pytestmark = pytest.mark.gpu

ALL_FMTS = [FP8_DYNAMIC, W8A8_INT8, BLOCK_FP8]


@pytest.fixture(autouse=True)
def _no_override():
    qgd.lib()
    for f in range(3):
        qgd.qgd_set_override(f)
    yield
    for f in range(3):
        qgd.qgd_set_override(f)
    qgd.qgd_set_pdl(-1)


def _oracle(case: Case, want_acc=False):
    xq, sx, wq, sw = case.oracle_quant()
    # the GPU and the oracle quantize independently; bytes must agree first
    np.testing.assert_array_equal(as_u8(case.xq), xq.view(np.uint8))
    np.testing.assert_array_equal(as_u8(case.wq), wq.view(np.uint8))
    return case.oracle_gemm(xq, sx, wq, sw, want_acc=want_acc)


def test_tiny_fp8_dynamic_default_plan():
    # FP8_Dynamic, X 4x1024 ~N(0,1), W 512x1024 ~N(0,0.02), seed 0
    case = Case(FP8_DYNAMIC, 4, 512, 1024, seed=0, outliers=False)
    yref, bound = _oracle(case)
    case.check_output(case.run(), yref, bound, "tiny default")


GRID, PERSISTENT = qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
VARIANTS = (
    [(qgd.VARIANT_SWAP_AB, s, r, 0, GRID) for s in (1, 2, 4, 8) for r in (0, 1, 2)]
    + [(qgd.VARIANT_SWAP_AB, 1, r, 0, PERSISTENT) for r in (0, 1, 2)]
    + [(qgd.VARIANT_STANDARD, s, r, t, GRID) for t in (128, 256) for s in (1, 2, 8) for r in (0, 1, 2)]
    + [(qgd.VARIANT_STANDARD, s, r, t, PERSISTENT) for t in (128, 256) for s in (1, 2) for r in (0, 1, 2)]
)


def _vid(v):
    sched = "pers" if v[4] == PERSISTENT else f"s{v[1]}"
    return f"{'swap' if v[0] == qgd.VARIANT_SWAP_AB else 'std'}-{sched}-r{v[2]}-t{v[3]}"


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("variant", VARIANTS, ids=_vid)
def test_every_variant_tiny(fmt, variant):
    var, split, red, tile, sched = variant
    case = Case(fmt, 4, 512, 1024, seed=1, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], var, split, red, 0, tile, sched)
    plan = qgd.qgd_get_plan(FMT_ID[fmt], 4, 512, 1024)
    assert plan["variant"] == var and plan["split_k"] == split and plan["source"] == 2
    assert plan["schedule"] == sched
    case.check_output(case.run(), yref, bound, f"{fmt} {_vid(variant)}")


@pytest.mark.parametrize("variant", VARIANTS, ids=_vid)
def test_int8_acc32_bit_exact_every_variant(variant):
    var, split, red, tile, sched = variant
    case = Case(W8A8_INT8, 5, 640, 2048, seed=2, outliers=True)
    _, _, acc = _oracle(case, want_acc=True)
    qgd.qgd_set_override(qgd.FMT_W8A8_INT8, var, split, red, 0, tile, sched)
    got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("M", [1, 2, 3, 8, 15, 16, 17, 24, 31, 32])
def test_decode_m_range(fmt, M):
    case = Case(fmt, M, 768, 2048, seed=M, outliers=True)
    yref, bound = _oracle(case)[:2]
    case.check_output(case.run(), yref, bound, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("M,N,K", [(33, 512, 1024), (100, 384, 2048), (130, 640, 1024), (257, 256, 512)])
def test_large_m_standard(fmt, M, N, K):
    case = Case(fmt, M, N, K, seed=M + N, outliers=True)
    yref, bound = _oracle(case)[:2]
    assert qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)["variant"] == qgd.VARIANT_STANDARD
    case.check_output(case.run(), yref, bound, f"{fmt} M={M}")


BLOCK_TWO_BLOCK_PLANS = [(1, 0, GRID, 1), (2, 0, GRID, 1), (4, 1, GRID, 2), (2, 2, GRID, 1), (1, 0, PERSISTENT, 2),
                         (1, 0, PERSISTENT, 1), (2, 0, PERSISTENT, 1)]


@pytest.mark.parametrize("M,N,K", [(130, 384, 1024), (257, 640, 2048), (64, 256, 512), (200, 1152, 1536)])
@pytest.mark.parametrize("plan", BLOCK_TWO_BLOCK_PLANS,
                         ids=[f"s{p[0]}-r{p[1]}-sch{p[2]}-k{p[3]}" for p in BLOCK_TWO_BLOCK_PLANS])
def test_block_fp8_two_block_tiles(M, N, K, plan):
    # 128 x 256 tiles: two 128-row weight blocks, each promoted with its own
    # scale by one pair of epilogue warps; N an odd number of blocks leaves the
    # last tile's second block past N
    split, red, sched, kps = plan
    case = Case(BLOCK_FP8, M, N, K, seed=M + N + K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8, qgd.VARIANT_STANDARD, split, red, 0, 256, sched, 0, kps)
    p = qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, M, N, K)
    assert p["tile_n"] == 256 and p["variant"] == qgd.VARIANT_STANDARD and p["k_slices"] == min(kps, K // 128)
    case.check_output(case.run(), yref, bound, f"Block_FP8 256-wide M={M} N={N} K={K} plan={p}")
    assert qgd.qgd_device_error() == 0


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("M,N,K", [(3, 528, 1040), (20, 1040, 272), (40, 272, 1040), (1, 16, 16)])
def test_ragged_tiles(fmt, M, N, K):
    # N not a multiple of the 128/256 tile, K not a multiple of the 128 stage
    case = Case(fmt, M, N, K, seed=N, outliers=True)
    yref, bound = _oracle(case)[:2]
    for var, split, red, sched in ((qgd.VARIANT_SWAP_AB, 1, 0, GRID), (qgd.VARIANT_SWAP_AB, 4, 0, GRID),
                                   (qgd.VARIANT_SWAP_AB, 1, 0, PERSISTENT), (qgd.VARIANT_SWAP_AB, 1, 1, PERSISTENT),
                                   (qgd.VARIANT_STANDARD, 1, 0, GRID), (qgd.VARIANT_STANDARD, 2, 1, GRID)):
        if var == qgd.VARIANT_SWAP_AB and M > 32:
            continue
        qgd.qgd_set_override(FMT_ID[fmt], var, split, red, 0, 0, sched)
        case.check_output(case.run(), yref, bound, f"{fmt} M={M} N={N} K={K} var={var} s={split}")


@pytest.mark.parametrize("fmt", ALL_FMTS)
def test_empty_m(fmt):
    case = Case(fmt, 1, 256, 1024, seed=5)
    xq = case.xq[:0]
    fn = {FP8_DYNAMIC: qgd.qlinear_fp8_dynamic, W8A8_INT8: qgd.qlinear_w8a8_int8,
          BLOCK_FP8: qgd.qlinear_block_fp8}[fmt]
    y = fn(xq, case.sx[:0], case.wq, case.sw)
    assert y.shape == (0, 256)


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("reduce", [qgd.REDUCE_LAST_CTA, qgd.REDUCE_TWO_PASS])
@pytest.mark.parametrize("sched", [GRID, PERSISTENT])
def test_deterministic_split_reductions_repeat_bitwise(fmt, reduce, sched):
    case = Case(fmt, 7, 1024, 4096, seed=9)
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, 8, reduce, 0, 0, sched)
    ys = [case.run().view(torch.int16).cpu() for _ in range(4)]
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_split_k_up_to_256():
    # K = 32768 gives 256 K tiles, so every power of two up to 256 is legal
    case = Case(W8A8_INT8, 2, 256, 32768, seed=4)
    _, _, acc = _oracle(case, want_acc=True)
    for split in (16, 64, 256):
        for red in (0, 1, 2):
            qgd.qgd_set_override(qgd.FMT_W8A8_INT8, qgd.VARIANT_SWAP_AB, split, red, 0, 0, GRID)
            assert qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 2, 256, 32768)["split_k"] == split
            got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc, err_msg=f"s={split} r={red}")


def test_graph_replay_matches_eager():
    case = Case(FP8_DYNAMIC, 8, 1024, 4096, seed=3)
    ws = qgd.Workspace(qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 8, 1024, 4096) + 4096)
    y_eager = case.run(ws=ws).clone()
    y = torch.empty_like(y_eager)
    xq = torch.empty_like(case.xq)
    sx = torch.empty_like(case.sx)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):  # warm up outside capture
            qgd.quant_act_per_token(case.xd, qgd.QTYPE_E4M3, xq=xq, sx=sx)
            qgd.qlinear_fp8_dynamic(xq, sx, case.wq, case.sw, y=y, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        qgd.quant_act_per_token(case.xd, qgd.QTYPE_E4M3, xq=xq, sx=sx)
        qgd.qlinear_fp8_dynamic(xq, sx, case.wq, case.sw, y=y, ws=ws)
    for _ in range(5):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))


def test_workspace_errors_are_reported():
    case = Case(FP8_DYNAMIC, 4, 512, 4096, seed=3)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 4, qgd.REDUCE_LAST_CTA, 0, 0, GRID)
    need = qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 512, 4096)
    assert need > 0
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(qgd.QGDError) as e:
        qgd.qlinear_fp8_dynamic(case.xq, case.sx, case.wq, case.sw, ws=small)
    assert e.value.status == -3
    assert qgd.qgd_device_error() == 0


def test_shared_workspace_across_modes_and_shapes():
    # one workspace serves calls of different shapes and reduction modes in any
    # order: partials never land on the arrival counters
    ws = qgd.Workspace(64 * 1024 + 64 * 4 * 4096 * 4)
    cases = [Case(FP8_DYNAMIC, 4, 512, 1024, seed=1), Case(W8A8_INT8, 3, 1024, 2048, seed=2),
             Case(BLOCK_FP8, 5, 768, 4096, seed=3)]
    refs = [_oracle(c)[:2] for c in cases]
    for rnd in range(2):
        for red in (qgd.REDUCE_TWO_PASS, qgd.REDUCE_LAST_CTA, qgd.REDUCE_ATOMIC, qgd.REDUCE_LAST_CTA):
            for c, (yref, bound) in zip(cases, refs):
                for f in range(3):
                    qgd.qgd_set_override(f, qgd.VARIANT_SWAP_AB, 4 if rnd == 0 else 8, red, 0, 0,
                                         GRID if rnd == 0 else PERSISTENT)
                c.check_output(c.run(ws=ws), yref, bound, f"{c.fmt} red={red} rnd={rnd}")
    assert qgd.qgd_device_error() == 0


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("reduce", [qgd.REDUCE_LAST_CTA, qgd.REDUCE_TWO_PASS, qgd.REDUCE_ATOMIC])
@pytest.mark.parametrize("M,N,K", [(1, 1024, 4096), (13, 384, 8192), (32, 2048, 1024), (5, 128, 25600)])
def test_persistent_schedule_uneven_units(fmt, reduce, M, N, K):
    # unit counts that do not divide by the CTA count: tiles shared by 1..many CTAs
    case = Case(fmt, M, N, K, seed=N + K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, -1, reduce, 0, 0, PERSISTENT)
    case.check_output(case.run(), yref, bound, f"{fmt} M={M} N={N} K={K} r={reduce}")
    if fmt == W8A8_INT8:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("stages", [2, 3, 5])
@pytest.mark.parametrize("occupancy", [1, 2])
def test_persistent_shallow_pipelines_one_or_two_ctas_per_sm(stages, occupancy):
    # shallow rings leave room for two CTAs per SM: sized for one or two
    case = Case(FP8_DYNAMIC, 16, 4096, 4096, seed=stages)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, stages, 0, PERSISTENT, occupancy, 1)
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 16, 4096, 4096)["occupancy"] == occupancy
    case.check_output(case.run(), yref, bound, f"stages={stages} occupancy={occupancy}")


@pytest.mark.parametrize("pdl", ["0", "1"])
def test_chained_layers_with_and_without_programmatic_launch(pdl):
    # quantize -> GEMM -> quantize(Y) -> GEMM on one stream: the second layer
    # reads the first layer's output, so any missing dependency shows
    qgd.qgd_set_pdl(int(pdl))
    x = synth.activations(8, 2048, seed=31, outliers=True).cuda()
    w1 = synth.weights(1024, 2048, seed=32).cuda()
    w2 = synth.weights(512, 1024, seed=33).cuda()
    wq1, sw1 = qgd.quant_weight_per_channel(w1)
    wq2, sw2 = qgd.quant_weight_per_channel(w2)
    ref = None
    for rep in range(3):
        xq, sx = qgd.quant_act_per_token(x)
        h = qgd.qlinear_fp8_dynamic(xq, sx, wq1, sw1)
        hq, hs = qgd.quant_act_per_token(h)
        y = qgd.qlinear_fp8_dynamic(hq, hs, wq2, sw2)
        torch.cuda.synchronize()
        if ref is None:
            # the same chain, one call at a time with a synchronize between
            xq2, sx2 = qgd.quant_act_per_token(x); torch.cuda.synchronize()
            h2 = qgd.qlinear_fp8_dynamic(xq2, sx2, wq1, sw1); torch.cuda.synchronize()
            hq2, hs2 = qgd.quant_act_per_token(h2); torch.cuda.synchronize()
            ref = qgd.qlinear_fp8_dynamic(hq2, hs2, wq2, sw2); torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"rep {rep}"


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("M,N,K,split", [(640, 2048, 1024, 1), (300, 4096, 512, 1), (1000, 768, 2048, 2),
                                         (2048, 1024, 768, 1)])
def test_persistent_standard_many_tiles_per_cta(fmt, M, N, K, split):
    # more tiles than SMs: each CTA walks several tiles through the
    # double-buffered accumulator; checked on sampled rows with the oracle
    case = Case(fmt, M, N, K, seed=M + K, outliers=True)
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD, split, 0, 0, 0, PERSISTENT)
    y = bf16_to_f64(case.run())
    rows = np.unique(np.concatenate([np.arange(0, M, 97), [M - 1]]))
    xsub = case.x[torch.from_numpy(rows)]
    sub = Case.__new__(Case)
    sub.fmt, sub.M, sub.N, sub.K, sub.x, sub.w = fmt, len(rows), N, K, xsub, case.w
    xq, sx, wq, sw = sub.oracle_quant()
    yref, bound = sub.oracle_gemm(xq, sx, wq, sw)[:2]
    if fmt == W8A8_INT8:
        check_within_one_ulp(y[rows], yref, f"{fmt} M={M}")
    else:
        check_fp8_tolerance(y[rows], yref, bound, K, f"{fmt} M={M}")


# Two K blocks per pipeline stage in the Standard kernel: a stage carries two
# 128-wide K blocks of X and W, with one hand-off and one commit; a split
# whose K range is odd ends in a one-block stage.  Block_FP8 still gives every
# K block its own TMEM slot.
STD_TWO_BLOCK_PLANS = [(GRID, 1, 0, 128), (GRID, 2, 1, 256), (GRID, 2, 2, 128), (PERSISTENT, 1, 0, 256),
                       (PERSISTENT, 2, 1, 128), (PERSISTENT, 1, 0, 128)]


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("plan", STD_TWO_BLOCK_PLANS, ids=[f"sch{p[0]}-s{p[1]}-r{p[2]}-t{p[3]}" for p in STD_TWO_BLOCK_PLANS])
@pytest.mark.parametrize("M,N,K", [(40, 384, 1152), (130, 512, 1408), (300, 256, 640), (33, 1280, 256)])
def test_standard_two_blocks_per_stage(fmt, plan, M, N, K):
    sched, split, red, tile = plan
    case = Case(fmt, M, N, K, seed=M + N + K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD, split, red, 0, tile, sched, 0, 2)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    assert p["variant"] == qgd.VARIANT_STANDARD and p["k_slices"] == 2
    y = case.run()
    case.check_output(y, yref, bound, f"{fmt} Standard two blocks M={M} N={N} K={K} plan={p}")
    if fmt == W8A8_INT8 and red != qgd.REDUCE_ATOMIC:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert qgd.qgd_device_error() == 0


# Standard pair tiles (256 tokens x 256 weight rows on two SMs, tcgen05
# cta_group::2): each CTA loads half the token rows and half the weight rows;
# M = 40 leaves the second CTA's token rows all past M (zero-filled copies),
# N = 528 a ragged last weight tile, K = 1152 an odd block count.  With
# Split-K (two-pass) the K blocks split unevenly where the count is odd.
PAIR_PLANS = [(GRID, 1, 256, 1), (GRID, 2, 256, 1), (PERSISTENT, 1, 256, 1), (PERSISTENT, 2, 256, 1),
              (GRID, 1, 256, 2), (GRID, 2, 256, 4), (PERSISTENT, 1, 256, 4), (GRID, 1, 256, 3)]


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("plan", PAIR_PLANS, ids=[f"sch{p[0]}-k{p[1]}-t{p[2]}-s{p[3]}" for p in PAIR_PLANS])
@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (40, 528, 1152), (300, 1024, 128), (520, 784, 2048)])
def test_standard_pair_tiles(fmt, plan, M, N, K):
    sched, kps, tile, split = plan
    case = Case(fmt, M, N, K, seed=M * 3 + N + K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD_PAIR, split, qgd.REDUCE_TWO_PASS, 0, tile, sched, 0,
                         kps)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    kps = kps if K > 128 else 1
    nku = -(-(K // 128) // kps)
    want_split = min(split, nku)
    assert (p["variant"], p["tile_n"], p["split_k"], p["k_slices"]) == (qgd.VARIANT_STANDARD_PAIR, tile, want_split,
                                                                        kps)
    assert p["reduce"] == (qgd.REDUCE_TWO_PASS if want_split > 1 else qgd.REDUCE_LAST_CTA)
    y1 = case.run()
    case.check_output(y1, yref, bound, f"{fmt} pair M={M} N={N} K={K} plan={p}")
    y2 = case.run()
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    if fmt == W8A8_INT8:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert qgd.qgd_device_error() == 0


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("tile", [256])
def test_standard_pair_persistent_many_tiles(fmt, tile):
    # 8 x 20 = 160 pair tiles: every pair walks several through the
    # double-buffered accumulator; sampled rows against the oracle
    M, N, K = 2048, 5120, 512
    case = Case(fmt, M, N, K, seed=77, outliers=True)
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD_PAIR, 1, 0, 0, tile, PERSISTENT, 0, 2)
    y = bf16_to_f64(case.run())
    rows = np.unique(np.concatenate([np.arange(0, M, 61), [127, 128, 255, 256, M - 1]]))
    xsub = case.x[torch.from_numpy(rows)]
    sub = Case.__new__(Case)
    sub.fmt, sub.M, sub.N, sub.K, sub.x, sub.w = fmt, len(rows), N, K, xsub, case.w
    xq, sx, wq, sw = sub.oracle_quant()
    yref, bound = sub.oracle_gemm(xq, sx, wq, sw)[:2]
    if fmt == W8A8_INT8:
        check_within_one_ulp(y[rows], yref, f"{fmt} pair persistent")
    else:
        check_fp8_tolerance(y[rows], yref, bound, K, f"{fmt} pair persistent")
    assert qgd.qgd_device_error() == 0


# Two 128-wide K slices per pipeline stage (Swap-AB): units are pairs of
# slices, and a tile with an odd slice count ends in a one-slice unit.
TWO_SLICE_PLANS = [(GRID, 1, 0, 0), (GRID, 2, 0, 0), (GRID, 4, 1, 0), (GRID, 4, 2, 0),
                   (PERSISTENT, -1, 0, 1), (PERSISTENT, -1, 1, 2), (PERSISTENT, -1, 2, 1), (PERSISTENT, -1, 0, 2)]


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("plan", TWO_SLICE_PLANS,
                         ids=lambda p: f"{'pers' if p[0] == PERSISTENT else 'grid'}-s{p[1]}-r{p[2]}-o{p[3]}")
@pytest.mark.parametrize("M,N,K", [(4, 512, 1024), (13, 384, 896), (32, 1024, 1152), (1, 2048, 4096)])
def test_two_slices_per_stage(fmt, plan, M, N, K):
    sched, split, red, occ = plan
    case = Case(fmt, M, N, K, seed=M * 7 + K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, split, red, 0, 0, sched, occ, 2)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    assert p["k_slices"] == 2 and p["variant"] == qgd.VARIANT_SWAP_AB
    case.check_output(case.run(), yref, bound, f"{fmt} two slices {plan} M={M} N={N} K={K}")
    if fmt == W8A8_INT8:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("sched", [GRID, PERSISTENT])
def test_two_slices_partial_last_slice(fmt, sched):
    # K = 1040: nine slices, the last one 16 wide (zero-filled past K)
    case = Case(fmt, 3, 528, 1040, seed=5, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, 2 if sched == GRID else -1, 0, 0, 0, sched, 0, 2)
    case.check_output(case.run(), yref, bound, f"{fmt} two slices K=1040")


# Split-K inside a thread-block cluster: partial rows travel through
# distributed shared memory to the CTA that owns them.
@pytest.mark.parametrize("fmt", ALL_FMTS)
# Any split count from 2 to 8: with 3, 5, 6 or 7 the 128 weight rows of a tile
# do not divide evenly among the owners (ceil(128 j / S) row boundaries).
@pytest.mark.parametrize("split,kps", [(2, 1), (4, 1), (8, 1), (4, 2), (8, 2), (3, 1), (5, 2), (6, 1), (7, 2)])
@pytest.mark.parametrize("M,N,K", [(1, 1024, 4096), (17, 384, 2048), (32, 2048, 1152), (5, 256, 1024)])
def test_cluster_split_reduction(fmt, split, kps, M, N, K):
    case = Case(fmt, M, N, K, seed=split * 31 + M, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, split, qgd.REDUCE_CLUSTER, 0, 0, GRID, 0, kps)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    nku = -(-(-(-K // 128)) // kps)  # K units of kps slices: the split is at most that
    expect = min(split, nku)
    assert p["reduce"] == qgd.REDUCE_CLUSTER and p["split_k"] == expect
    y1 = case.run()
    case.check_output(y1, yref, bound, f"{fmt} cluster s={split} k={kps} M={M} N={N} K={K}")
    y2 = case.run()  # fixed split order: bitwise repeatable
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    if fmt == W8A8_INT8:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert qgd.qgd_device_error() == 0


def test_cluster_split_reduction_ragged_n_and_graph():
    # N = 528: the last tile has 16 live weight rows; every row still reports
    case = Case(FP8_DYNAMIC, 3, 528, 1040, seed=9, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 8, qgd.REDUCE_CLUSTER, 0, 0, GRID, 0, 1)
    y = torch.empty((3, 528), dtype=torch.bfloat16, device="cuda")
    call = lambda: qgd.qlinear_fp8_dynamic(case.xq, case.sx, case.wq, case.sw, y=y)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    case.check_output(y, yref, bound, "cluster ragged N under graph replay")
    assert qgd.qgd_device_error() == 0


# Swap-AB past the decode range (FP8_Dynamic and W8A8_INT8, up to 128 tokens):
# the MMA's token dimension is 64 or 128 and the epilogue walks each
# accumulator row 32 tokens at a time.
SWAP_WIDE_PLANS = [(GRID, 1, 0, 0, 1), (GRID, 4, 0, 0, 2), (GRID, 4, 2, 0, 1), (GRID, 8, 3, 0, 1),
                   (GRID, 4, 3, 0, 2), (PERSISTENT, -1, 0, 1, 1), (PERSISTENT, -1, 2, 1, 2), (PERSISTENT, -1, 0, 2, 1)]


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("plan", SWAP_WIDE_PLANS,
                         ids=lambda p: f"{'pers' if p[0] == PERSISTENT else 'grid'}-s{p[1]}-r{p[2]}-o{p[3]}-k{p[4]}")
@pytest.mark.parametrize("M,N,K", [(33, 512, 1024), (64, 1024, 2048), (100, 384, 1152), (128, 640, 4096)])
def test_swap_ab_wide_token_counts(fmt, plan, M, N, K):
    sched, split, red, occ, kps = plan
    case = Case(fmt, M, N, K, seed=M + 3 * K, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_SWAP_AB, split, red, 0, 0, sched, occ, kps)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    assert p["variant"] == qgd.VARIANT_SWAP_AB and p["reduce"] == red
    case.check_output(case.run(), yref, bound, f"{fmt} swap wide {plan} M={M} N={N} K={K}")
    if fmt == W8A8_INT8:
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert qgd.qgd_device_error() == 0


STD_CLUSTER_PLANS = [(2, 256, 2), (3, 256, 1), (4, 128, 2), (5, 256, 1), (8, 128, 1), (8, 256, 1), (2, 128, 1)]


@pytest.mark.parametrize("fmt", [FP8_DYNAMIC, W8A8_INT8])
@pytest.mark.parametrize("plan", STD_CLUSTER_PLANS, ids=[f"s{p[0]}-t{p[1]}-k{p[2]}" for p in STD_CLUSTER_PLANS])
@pytest.mark.parametrize("M,N,K", [(130, 528, 2048), (257, 256, 4096), (40, 1040, 1536), (512, 768, 1024)])
def test_standard_cluster_split(fmt, plan, M, N, K):
    # Standard tiles whose K splits form one thread-block cluster: every row's
    # owner adds the splits' partials in split order, so the output equals the
    # last-arriving-CTA reduction's bit for bit
    split, tile, kps = plan
    case = Case(fmt, M, N, K, seed=M + 2 * N + K + split, outliers=True)
    yref, bound = _oracle(case)[:2]
    qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD, split, qgd.REDUCE_CLUSTER, 0, tile, GRID, 0, kps)
    p = qgd.qgd_get_plan(FMT_ID[fmt], M, N, K)
    if p["reduce"] != qgd.REDUCE_CLUSTER:
        pytest.skip(f"plan legalised to {p}")
    assert p["variant"] == qgd.VARIANT_STANDARD and p["tile_n"] == tile
    y1 = case.run()
    case.check_output(y1, yref, bound, f"{fmt} Standard cluster M={M} N={N} K={K} plan={p}")
    assert qgd.qgd_device_error() == 0
    if p["split_k"] & (p["split_k"] - 1) == 0:  # the other reductions take powers of two only
        qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD, p["split_k"], qgd.REDUCE_LAST_CTA, p["stages"], tile,
                             GRID, 0, p["k_slices"])
        y2 = case.run()
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    if fmt == W8A8_INT8:
        qgd.qgd_set_override(FMT_ID[fmt], qgd.VARIANT_STANDARD, split, qgd.REDUCE_CLUSTER, 0, tile, GRID, 0, kps)
        _, _, acc = _oracle(case, want_acc=True)
        got = qgd.qgd_w8a8_int8_acc32(case.xq, case.wq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert qgd.qgd_device_error() == 0
