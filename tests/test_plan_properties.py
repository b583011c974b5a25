"""Property tests of plan legalisation (host only): for random shapes of every
format and random plan overrides, with and without the shipped dispatch table,
the plan the library would run satisfies every rule its kernels rely on."""
import pytest
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

import quantized_gemm_decode_b200 as qgd

FP8, INT8, BLOCK, MX, NV = (qgd.FMT_FP8_DYNAMIC, qgd.FMT_W8A8_INT8, qgd.FMT_BLOCK_FP8, qgd.FMT_MXFP8,
                            qgd.FMT_NVFP4)
SWAP, STD, PAIR = qgd.VARIANT_SWAP_AB, qgd.VARIANT_STANDARD, qgd.VARIANT_STANDARD_PAIR
CLUSTER = qgd.REDUCE_CLUSTER


def mpad(M: int) -> int:
    return 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128


def tmem_cols(M: int, stages: int, kps: int, fmt: int) -> int:
    need = 2 * mpad(M) + stages * kps * (32 if fmt == NV else 8)
    c = 32
    while c < need:
        c *= 2
    return c


@st.composite
def shapes(draw):
    fmt = draw(st.sampled_from([FP8, INT8, BLOCK, MX, NV]))
    m_cap = 128 if fmt in (MX, NV) else 8192
    M = draw(st.integers(1, m_cap))
    n_unit = 128 if fmt == BLOCK else 16
    k_unit = 256 if fmt == NV else (128 if fmt in (BLOCK, MX) else 16)
    N = n_unit * draw(st.integers(1, 65536 // n_unit))
    K = k_unit * draw(st.integers(1, 16384 // k_unit))
    return fmt, M, N, K


overrides = st.tuples(
    st.sampled_from([-1, STD, SWAP, PAIR]),      # variant
    st.sampled_from([-1, 1, 2, 3, 4, 5, 8, 16, 64, 256]),  # split_k
    st.sampled_from([-1, 0, 1, 2, 3]),           # reduce
    st.integers(0, 8),                           # stages (0: deepest)
    st.sampled_from([0, 128, 256]),              # tile_n
    st.sampled_from([-1, 0, 1]),                 # schedule
    st.integers(0, 2),                           # occupancy
    st.integers(0, 2),                           # k_slices
)


@pytest.fixture(scope="module", autouse=True)
def _library():
    qgd.lib()
    yield
    for f in range(5):
        qgd.qgd_set_override(f)
    qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)


@pytest.mark.parametrize("table", [False, True], ids=["built-in", "shipped-table"])
@settings(max_examples=300, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(shape=shapes(), ov=overrides)
def test_every_plan_is_legal(table, shape, ov):
    fmt, M, N, K = shape
    if table:
        qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
    else:
        qgd.qgd_clear_dispatch_table()
    try:
        qgd.qgd_set_override(fmt, *ov)
    except qgd.QGDError:
        assume(False)  # an override the library refuses outright (e.g. split 3 without the cluster)
    try:
        p = qgd.qgd_get_plan(fmt, M, N, K)
        ws = qgd.qgd_workspace_size(fmt, M, N, K)
    finally:
        qgd.qgd_set_override(fmt)
    v, s, r, stages, tile, sched, occ, kps = (p["variant"], p["split_k"], p["reduce"], p["stages"], p["tile_n"],
                                              p["schedule"], p["occupancy"], p["k_slices"])
    nkt = -(-(K // 2 if fmt == NV else K) // 128)
    assert v in (STD, SWAP, PAIR)
    if fmt in (MX, NV):
        assert v == SWAP
    if v == SWAP:
        assert M <= (32 if fmt == BLOCK else 128) and tile == 128
    if v == STD:
        assert tile in (128, 256)
    if v == PAIR:
        assert fmt in (FP8, INT8) and tile == 256
        assert r == (1 if s > 1 else 0)  # Split-K through the two-pass reduction only
    assert kps in (1, 2) and (kps == 1 or nkt >= 2)
    assert stages >= 2 and occ >= 1 and sched in (0, 1)
    assert 1 <= s <= 256 and s <= -(-nkt // kps)
    assert r in (0, 1, 2, 3)
    if r == CLUSTER:
        assert 2 <= s <= 8 and sched == 0
        assert v == SWAP or (v == STD and fmt in (FP8, INT8))
        if v == STD:
            rows = -(-128 // s)
            assert (s - 1) * rows * tile * 4 <= stages * kps * (128 + tile) * 128  # received rows fit the ring
        assert ws == 0
    elif v != PAIR:
        assert s & (s - 1) == 0  # a power of two outside a cluster and pair tiles
    if v == SWAP and M > 32:
        assert r != 1  # the two-pass reduction kernel covers 32 tokens
    if fmt in (MX, NV):
        assert r != 1
        cols = tmem_cols(M, stages, kps, fmt)
        if M <= 64:
            assert cols <= 256
        else:
            assert cols <= 512 and stages * kps >= 4  # a CTA that has its SM to itself
    if v == PAIR and s > 1:
        assert ws == 65536 + ((M * N * 4 * s + 255) // 256) * 256  # one fp32 partial per split
    if s == 1 and r != CLUSTER:
        assert ws == 0 or v == SWAP  # (Swap-AB persistent plans may split tiles between CTAs)
    assert ws >= 0
