"""CPU-only checks of the C ABI: the library loads, exports every function
include/qgd.h declares, and its host-side logic (M buckets, default plans,
dispatch-table parsing, overrides, workspace sizing, argument rejection)
behaves as documented.  No GPU and no kernel launch is needed."""
import ctypes
import os
import re

import pytest

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgd.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    qgd.lib()
    yield
    qgd.qgd_clear_dispatch_table()
    for f in range(3):
        qgd.qgd_set_override(f)


@pytest.fixture(autouse=True)
def clean_state():
    qgd.qgd_clear_dispatch_table()
    for f in range(3):
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f)
    yield


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^QGD_API\s+[\w\s\*]+?\b(\w+)\(", text, flags=re.M)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for required in ("quant_act_per_token", "quant_act_group128", "quant_weight_block128",
                     "qlinear_fp8_dynamic", "qlinear_w8a8_int8", "qlinear_block_fp8",
                     "qgd_load_dispatch_table", "qgd_workspace_size", "qgd_set_override",
                     "qgd_w8a8_int8_acc32", "qgd_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(qgd.LIB_PATH)
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version():
    L = qgd.lib()
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert L.qgd_status_string(st)
    assert qgd.qgd_version().count(".") == 2


@pytest.mark.parametrize("M,b", [(1, 1), (2, 2), (3, 4), (5, 8), (9, 16), (17, 24), (25, 32), (33, 64),
                                 (100, 128), (129, 512), (600, 2048), (3000, 8192), (100000, 8192)])
def test_m_buckets(M, b):
    assert qgd.qgd_m_bucket(M) == b


def test_default_plans():
    # decode: Swap-AB on the persistent schedule (grid-schedule split until
    # the 148 SMs are covered)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 4096)
    assert p["variant"] == qgd.VARIANT_SWAP_AB and p["source"] == 0
    assert p["schedule"] == qgd.SCHEDULE_PERSISTENT
    assert p["split_k"] == 8  # 32 tiles * 8 >= 148
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 32, 24576, 4096)
    assert p["split_k"] == 1  # 192 tiles already cover the SMs
    # large M: Standard, no split
    p = qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 512, 6144, 4096)
    assert p["variant"] == qgd.VARIANT_STANDARD and p["split_k"] == 1 and p["tile_n"] == 256
    assert p["schedule"] == qgd.SCHEDULE_PERSISTENT
    p = qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, 512, 6144, 4096)
    assert p["tile_n"] == 256  # two 128-row weight blocks per tile
    # split never exceeds the number of 128-wide K tiles
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 128, 256)
    assert p["split_k"] == 2


def test_override_and_clamping():
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 256, qgd.REDUCE_ATOMIC, 5, 0, qgd.SCHEDULE_GRID)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)
    assert (p["variant"], p["split_k"], p["reduce"], p["stages"], p["source"]) == (1, 32, 2, 5, 2)
    # Swap-AB cannot take more than 128 tokens: it falls back to Standard
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 4, 0, 0, 0, qgd.SCHEDULE_GRID)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 129, 4096, 4096)
    assert p["variant"] == qgd.VARIANT_STANDARD and p["schedule"] == qgd.SCHEDULE_GRID
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, 1, 3, 0, 0, 0)  # split not a power of two
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, 1, 9, qgd.REDUCE_CLUSTER, 0, 0)  # cluster of 9: too many
    # the cluster reduction takes any split count from 2 to 8, capped at the K units
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 6, qgd.REDUCE_CLUSTER, 0, 0, qgd.SCHEDULE_GRID, 0, 2)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 6144, 4096)
    assert (p["variant"], p["split_k"], p["reduce"], p["schedule"]) == (1, 6, qgd.REDUCE_CLUSTER, qgd.SCHEDULE_GRID)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 6144, 640)  # 5 K slices -> 3 units of two
    assert (p["split_k"], p["reduce"]) == (3, qgd.REDUCE_CLUSTER)
    # another reduction cannot take a split of 6: it is rounded down to a power of two
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 6, qgd.REDUCE_CLUSTER, 0, 0, qgd.SCHEDULE_PERSISTENT)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 6144, 4096)
    assert p["reduce"] != qgd.REDUCE_CLUSTER and p["split_k"] in (1, 2, 4)
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(7, 1, 2, 0, 0, 0)


def test_workspace_size_follows_plan():
    hdr = 64 * 1024  # arrival-counter header
    G = qgd.SCHEDULE_GRID
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 1, 0, 0, 0, G)
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096) == 0
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 8, qgd.REDUCE_LAST_CTA, 0, 0, G)
    # header + 32 tiles x 8 splits x 128 rows x 4 tokens of fp32
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096) == hdr + 32 * 8 * 128 * 4 * 4
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 8, qgd.REDUCE_TWO_PASS, 0, 0, G)
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096) == hdr + 32 * 8 * 128 * 4 * 4
    # 5 tokens: rows of partials are padded to 8 words (two 16-byte vectors)
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 5, 4096, 4096) == hdr + 32 * 8 * 128 * 8 * 4
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 8, qgd.REDUCE_ATOMIC, 0, 0, G)
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096) == hdr + 4 * 4096 * 4
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_STANDARD, 2, qgd.REDUCE_LAST_CTA, 0, 128, G)
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 40, 4096, 4096) == hdr + 2 * 40 * 4096 * 4


def _persistent_geometry(N, K, ctas):
    """Contributors per tile when ctas CTAs share the (tile, K-slice) units."""
    nkt, tiles = (K + 127) // 128, (N + 127) // 128
    U = tiles * nkt
    G = min(U, ctas)
    owner = lambda u: ((u + 1) * G - 1) // U  # noqa: E731
    return max(owner(t * nkt + nkt - 1) - owner(t * nkt) + 1 for t in range(tiles)), tiles


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (32, 6144, 4096), (8, 24576, 4096), (3, 4096, 12288),
                                   (1, 256, 256), (16, 51200, 5120)])
def test_persistent_workspace_matches_unit_partition(M, N, K):
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, qgd.REDUCE_LAST_CTA, 0, 0,
                         qgd.SCHEDULE_PERSISTENT)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, M, N, K)
    assert p["schedule"] == qgd.SCHEDULE_PERSISTENT and p["occupancy"] == 1
    # the deepest pipelines leave room for one CTA per SM (148 SMs)
    maxc, tiles = _persistent_geometry(N, K, 148)
    mstride = (M + 3) // 4 * 4
    want = 0 if maxc == 1 else 64 * 1024 + ((tiles * maxc * 128 * mstride * 4 + 255) // 256) * 256
    assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, M, N, K) == want


def test_too_many_tiles_for_counters_fall_back_to_two_pass():
    # Standard tiles of 128 x 128 over 8192 x 262144 exceed the 16384 counters
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_STANDARD, 2, qgd.REDUCE_LAST_CTA, 0, 128, 0)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 8192, 262144, 4096)
    assert p["reduce"] == qgd.REDUCE_TWO_PASS


def test_table_load_and_lookup(tmp_path):
    t = tmp_path / "t.tsv"
    t.write_text("# fmt N K M_bucket variant split_k reduce stages tile_n schedule occupancy\n"
                 "fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 grid 0\n"
                 "\n"
                 "w8a8_int8 5120 5120 32 swap_ab 4 atomic 3 0 persistent 2  # trailing comment\n")
    qgd.qgd_load_dispatch_table(str(t))
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 3, 4096, 4096)  # bucket 4
    assert (p["variant"], p["split_k"], p["reduce"], p["stages"], p["tile_n"], p["source"]) == (0, 2, 1, 4, 256, 1)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 5, 4096, 4096)  # bucket 8: not in the table
    assert p["source"] == 0
    p = qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 25, 5120, 5120)
    assert (p["variant"], p["split_k"], p["reduce"], p["schedule"], p["occupancy"], p["source"]) == (1, 4, 2, 1, 2, 1)
    qgd.qgd_clear_dispatch_table()
    assert qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 25, 5120, 5120)["source"] == 0


@pytest.mark.parametrize("bad", [
    "fp8_dynamic 4096 4096 4 standard 3 two_pass 4 256 grid 0\n",      # split not a power of two
    "fp8_dynamic 4096 4096 4 swap_ab 9 cluster 2 128 grid 1\n",        # cluster of 9 CTAs
    "fp8_dynamic 4096 4096 5 standard 2 two_pass 4 256 grid 0\n",      # 5 is not a bucket
    "fp9 4096 4096 4 standard 2 two_pass 4 256 grid 0\n",              # unknown format
    "fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 grid\n",        # missing field
    "fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 grid 0 7\n",    # extra field
    "fp8_dynamic 4096 4096 4 diagonal 2 two_pass 4 256 grid 0\n",      # unknown variant
    "fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 stream 0\n",    # unknown schedule
    "fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 grid 3\n",      # occupancy out of range
])
def test_malformed_table_is_rejected_and_keeps_previous(tmp_path, bad):
    good = tmp_path / "good.tsv"
    good.write_text("fp8_dynamic 4096 4096 4 standard 2 two_pass 4 256 grid 0\n")
    qgd.qgd_load_dispatch_table(str(good))
    t = tmp_path / "bad.tsv"
    t.write_text(bad)
    with pytest.raises(qgd.QGDError) as e:
        qgd.qgd_load_dispatch_table(str(t))
    assert e.value.status == -5
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)["source"] == 1


def test_missing_table_file():
    with pytest.raises(qgd.QGDError) as e:
        qgd.qgd_load_dispatch_table("/nonexistent/table.tsv")
    assert e.value.status == -5


def test_shipped_table_parses():
    if os.path.exists(qgd.DEFAULT_TABLE):
        qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)


def test_argument_rejection_before_any_launch():
    L = qgd.lib()
    P = ctypes.c_void_p
    # null pointers / bad shapes are rejected on the host, with no device call
    assert L.qlinear_fp8_dynamic(None, None, None, None, None, 4, 512, 1024, None, 0, None) == -1
    assert L.qlinear_fp8_dynamic(P(16), P(16), P(16), P(16), P(16), 4, 500, 1024, None, 0, None) == -2
    assert L.qlinear_block_fp8(P(16), P(16), P(16), P(16), P(16), 4, 512, 1000, None, 0, None) == -2
    assert L.qlinear_w8a8_int8(P(16), P(16), P(16), P(16), P(16), -1, 512, 1024, None, 0, None) == -1
    assert L.qlinear_fp8_dynamic(P(17), P(16), P(16), P(16), P(16), 4, 512, 1024, None, 0, None) == -1
    assert L.quant_act_per_token(P(16), 4, 12, 0, P(16), P(16), None) == -2
    assert L.quant_act_per_token(P(16), 4, 16, 5, P(16), P(16), None) == -1
    # M == 0 is an empty, successful call
    assert L.qlinear_fp8_dynamic(None, None, None, None, None, 0, 512, 1024, None, 0, None) == 0
    assert b"16" in L.qgd_last_error_message() or L.qgd_last_error_message() is not None


def test_persistent_occupancy_follows_shared_memory():
    # deep rings fit one CTA per SM; shallow ones two, unless one is asked for
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 4, 0, qgd.SCHEDULE_PERSISTENT)
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)["occupancy"] == 2
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 4, 0, qgd.SCHEDULE_PERSISTENT, 1)
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)["occupancy"] == 1
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 10, 0, qgd.SCHEDULE_PERSISTENT, 2)
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)["occupancy"] == 1  # 2 do not fit
    # fewer CTAs share each tile with one CTA per SM: a smaller workspace
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 4, 0, qgd.SCHEDULE_PERSISTENT, 1)
    one = qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 4, 0, qgd.SCHEDULE_PERSISTENT, 2)
    two = qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)
    assert 0 < one < two


def test_mma_peak_probe_rejects_bad_arguments():
    L = qgd.lib()
    flops = ctypes.c_double(0.0)
    assert L.qgd_mma_peak_probe(2, 16, ctypes.byref(flops), None) == -1  # qtype
    assert L.qgd_mma_peak_probe(qgd.QTYPE_E4M3, 0, ctypes.byref(flops), None) == -1
    assert L.qgd_mma_peak_probe(qgd.QTYPE_INT8, 200001, ctypes.byref(flops), None) == -1
    for n, slots, wait, iters in ((64, 1, 1, 16), (256, 4, 1, 16), (128, 3, 0, 16), (128, 1, 2, 16), (128, 1, 1, 0)):
        assert L.qgd_mma_ring_probe(n, slots, wait, iters, ctypes.byref(flops), None) == -1


def test_k_slices_plan_field():
    P = qgd.SCHEDULE_PERSISTENT
    # default: one slice per stage
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 4096)["k_slices"] == 1
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 0, 0, P, 1, 2)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 4096)
    assert p["k_slices"] == 2 and p["occupancy"] == 1
    # deepest ring with two 16 KB weight slices + 2 KB activation slices per stage
    assert p["stages"] == (232448 - 1024 - 1024) // (2 * (16384 + 16 * 128))
    # a single-slice K has one slice per stage
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 128)["k_slices"] == 1
    # the Standard kernel takes two K blocks per stage too: 128 x 256 tiles then fit two stages
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_STANDARD, 1, 0, 0, 256, P, 0, 2)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 64, 4096, 4096)
    assert p["k_slices"] == 2 and p["stages"] == (232448 - 1024 - 1024) // (2 * (16384 + 32768))
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8, qgd.VARIANT_STANDARD, 1, 0, 0, 128, P, 0, 2)
    p = qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, 64, 4096, 4096)
    assert p["k_slices"] == 2 and p["stages"] == 3
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8)
    # grid Split-K counts units of two slices: at most ceil(nkt / 2) splits
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 32, 0, 0, 0, qgd.SCHEDULE_GRID, 0, 2)
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 4096)["split_k"] == 16
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, 1, 1, 0, 0, 0, P, 1, 3)


def test_k_slices_workspace_counts_two_slice_units():
    P = qgd.SCHEDULE_PERSISTENT
    hdr = 64 * 1024
    # partial slots per tile = most CTAs sharing a tile, counted over the
    # schedule's units: 32 tiles x 16 two-slice units, or x 32 one-slice units
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 0, 0, P, 1, 2)
    ws2 = qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, -1, 0, 0, 0, P, 1, 1)
    ws1 = qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)

    def maxc(U, G, per_tile, tiles):
        own = lambda u: ((u + 1) * G - 1) // U
        return max(own(t * per_tile + per_tile - 1) - own(t * per_tile) + 1 for t in range(tiles))

    assert ws2 == hdr + 32 * maxc(512, 148, 16, 32) * 128 * 4 * 4
    assert ws1 == hdr + 32 * maxc(1024, 148, 32, 32) * 128 * 4 * 4


def test_table_k_slices_column(tmp_path):
    t = tmp_path / "t.tsv"
    t.write_text("fp8_dynamic 4096 4096 1 swap_ab 1 last_cta 0 0 persistent 1 2\n"
                 "fp8_dynamic 4096 4096 2 swap_ab 1 last_cta 0 0 persistent 1\n")
    qgd.qgd_load_dispatch_table(str(t))
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 1, 4096, 4096)["k_slices"] == 2
    assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 2, 4096, 4096)["k_slices"] == 1
    bad = tmp_path / "b.tsv"
    bad.write_text("fp8_dynamic 4096 4096 1 swap_ab 1 last_cta 0 0 persistent 1 3\n")
    with pytest.raises(qgd.QGDError):
        qgd.qgd_load_dispatch_table(str(bad))
    bad.write_text("fp8_dynamic 4096 4096 1 swap_ab 1 last_cta 0 0 persistent 1 2 9\n")
    with pytest.raises(qgd.QGDError):
        qgd.qgd_load_dispatch_table(str(bad))


def test_standard_pair_plan_rules():
    P, G = qgd.SCHEDULE_PERSISTENT, qgd.SCHEDULE_GRID
    for fmt in (qgd.FMT_FP8_DYNAMIC, qgd.FMT_W8A8_INT8):
        qgd.qgd_set_override(fmt, qgd.VARIANT_STANDARD_PAIR, 1, qgd.REDUCE_TWO_PASS, 0, 128, P, 0, 2)
        p = qgd.qgd_get_plan(fmt, 4096, 6144, 4096)
        # pair tiles are 256 wide; two K blocks per stage fit three stages
        assert (p["variant"], p["tile_n"], p["split_k"], p["reduce"], p["k_slices"], p["stages"],
                p["occupancy"]) == (qgd.VARIANT_STANDARD_PAIR, 256, 1, qgd.REDUCE_LAST_CTA, 2, 3, 1)
        assert qgd.qgd_workspace_size(fmt, 4096, 6144, 4096) == 0
        # Split-K always takes the two-pass reduction: one fp32 partial per split
        # after the 64 KiB header, any count up to the K units
        for split, red in ((4, qgd.REDUCE_LAST_CTA), (4, qgd.REDUCE_ATOMIC), (3, qgd.REDUCE_CLUSTER),
                           (64, qgd.REDUCE_TWO_PASS)):
            qgd.qgd_set_override(fmt, qgd.VARIANT_STANDARD_PAIR, split, red, 0, 0, G, 0, 2)
            p = qgd.qgd_get_plan(fmt, 512, 1024, 4096)
            want = {4: 4, 3: 3, 64: 16}[split]  # 32 K blocks / 2 per stage = 16 K units
            assert (p["variant"], p["split_k"], p["reduce"]) == (qgd.VARIANT_STANDARD_PAIR, want,
                                                                 qgd.REDUCE_TWO_PASS), (split, red, p)
            assert qgd.qgd_workspace_size(fmt, 512, 1024, 4096) == 65536 + 512 * 1024 * 4 * want
        # more 128 x 256 tiles than arrival counters: pair tiles use none, so no split keeps no workspace
        qgd.qgd_set_override(fmt, qgd.VARIANT_STANDARD_PAIR, 1, 0, 0, 0, P, 0, 2)
        p = qgd.qgd_get_plan(fmt, 8192, 131072, 4096)
        assert (p["variant"], p["split_k"], p["reduce"]) == (qgd.VARIANT_STANDARD_PAIR, 1, qgd.REDUCE_LAST_CTA)
        assert qgd.qgd_workspace_size(fmt, 8192, 131072, 4096) == 0
        qgd.qgd_set_override(fmt, qgd.VARIANT_STANDARD_PAIR, 1, 0, 0, 0, G, 0, 1)
        # one-block stages of 32 KB beside the 32 KB output staging area
        assert qgd.qgd_get_plan(fmt, 512, 6144, 4096)["stages"] == (232448 - 2048 - 32768) // 32768
        qgd.qgd_set_override(fmt)
    # Block_FP8 and MXFP8 have no pair tiles
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8, qgd.VARIANT_STANDARD_PAIR, 1, 0, 0, 0, P)
    assert qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, 4096, 6144, 4096)["variant"] == qgd.VARIANT_STANDARD
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8)
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, 3, 1, 0, 0, 0)


def test_table_standard_pair_name(tmp_path):
    t = tmp_path / "t.tsv"
    t.write_text("fp8_dynamic 6144 4096 8192 standard_pair 1 last_cta 3 256 persistent 1 2\n")
    qgd.qgd_load_dispatch_table(str(t))
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 8192, 6144, 4096)
    assert (p["variant"], p["stages"], p["k_slices"], p["schedule"], p["source"]) == \
        (qgd.VARIANT_STANDARD_PAIR, 3, 2, qgd.SCHEDULE_PERSISTENT, 1)


def test_cluster_reduction_plan_rules():
    G, P = qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
    C = qgd.REDUCE_CLUSTER
    for split in (2, 3, 4, 5, 6, 7, 8):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, split, C, 0, 0, G, 0, 1)
        p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)
        assert p["reduce"] == C and p["split_k"] == split
        # the splits exchange partials through shared memory: no workspace
        assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096) == 0
    # beyond a portable cluster, on the persistent schedule, or with one split
    # the reduction falls back to the last-arriving CTA
    for args in ((qgd.VARIANT_SWAP_AB, 16, C, 0, 0, G), (qgd.VARIANT_SWAP_AB, -1, C, 0, 0, P),
                 (qgd.VARIANT_STANDARD, 4, C, 0, 128, P), (qgd.VARIANT_SWAP_AB, 1, C, 0, 0, G)):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, *args)
        assert qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 4, 4096, 4096)["reduce"] == qgd.REDUCE_LAST_CTA
    # Standard tiles of the per-token formats: the splits' rows meet in the owners' rings
    for fmt in (qgd.FMT_FP8_DYNAMIC, qgd.FMT_W8A8_INT8):
        for split in (2, 3, 5, 8):
            qgd.qgd_set_override(fmt, qgd.VARIANT_STANDARD, split, C, 0, 256, G, 0, 2)
            p = qgd.qgd_get_plan(fmt, 512, 4096, 4096)
            assert (p["variant"], p["reduce"], p["split_k"]) == (qgd.VARIANT_STANDARD, C, split)
            assert qgd.qgd_workspace_size(fmt, 512, 4096, 4096) == 0
        qgd.qgd_set_override(fmt)
    # Block_FP8 promotes into registers: no cluster reduction in its Standard kernel
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8, qgd.VARIANT_STANDARD, 4, C, 0, 256, G, 0, 2)
    assert qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, 512, 4096, 4096)["reduce"] == qgd.REDUCE_LAST_CTA
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8)
    # the received rows must fit the ring: two one-block stages of 128 x 256 hold 96 KB,
    # less than the 7 x 16 rows x 1 KB that eight splits send
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_STANDARD, 8, C, 2, 256, G, 0, 1)
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 512, 4096, 4096)
    assert (p["reduce"], p["split_k"]) == (qgd.REDUCE_LAST_CTA, 8)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, 1, 4, 4, 0, 0, G)


def test_table_cluster_reduce_name(tmp_path):
    t = tmp_path / "t.tsv"
    t.write_text("w8a8_int8 5120 5120 8 swap_ab 4 cluster 0 0 grid 0 2\n"
                 "w8a8_int8 5120 5120 16 swap_ab 5 cluster 0 0 grid 0 2\n")
    qgd.qgd_load_dispatch_table(str(t))
    p = qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 8, 5120, 5120)
    assert (p["reduce"], p["split_k"], p["k_slices"], p["source"]) == (qgd.REDUCE_CLUSTER, 4, 2, 1)
    p = qgd.qgd_get_plan(qgd.FMT_W8A8_INT8, 16, 5120, 5120)
    assert (p["reduce"], p["split_k"], p["k_slices"], p["source"]) == (qgd.REDUCE_CLUSTER, 5, 2, 1)


@pytest.mark.parametrize("fmt,M,N,K", [("fp8_dynamic", 1, 4096, 4096), ("w8a8_int8", 16, 34816, 5120),
                                       ("block_fp8", 32, 5120, 25600), ("fp8_dynamic", 512, 6144, 4096),
                                       ("fp8_dynamic", 64, 24576, 4096), ("w8a8_int8", 128, 4096, 12288),
                                       ("block_fp8", 64, 6144, 4096), ("mxfp8", 16, 4096, 4096),
                                       ("mxfp8", 64, 6144, 4096), ("nvfp4", 1, 4096, 4096),
                                       ("nvfp4", 32, 4096, 12288), ("nvfp4", 64, 6144, 4096),
                                       ("fp8_dynamic", 2048, 6144, 4096), ("w8a8_int8", 512, 4096, 12288)])
def test_tuner_candidates_are_legal_plans(fmt, M, N, K):
    # every plan the tuner times is one the library runs as asked (no silent
    # legalization), and a grid-schedule Swap-AB candidate with more CTAs than
    # SMs fits two CTAs per SM
    from quantized_gemm_decode_b200 import tune

    fid = tune.FMT_ID[fmt]
    cands = tune.candidates(fmt, M, N, K, 148)
    # fused candidates at decode token counts (the block-scaled formats have no fused quantizer)
    assert any(c[8] for c in cands) == (M <= 32 and fmt not in ("mxfp8", "nvfp4"))
    for var, s, r, t, sch, occ, kps, st, fz in cands:
        qgd.qgd_set_override(fid, var, s, r, st, t, sch, occ, kps)
        qgd.qgd_set_fused_override(fid, fz)
        p = qgd.qgd_get_layer_plan(fid, M, N, K)
        assert (p["variant"], p["reduce"], p["schedule"], p["k_slices"], p["fused"]) == (var, r, sch, kps, fz), \
            (var, s, r, sch, kps, fz)
        if sch == qgd.SCHEDULE_PERSISTENT and var == qgd.VARIANT_SWAP_AB:
            assert p["occupancy"] == occ
        if sch == qgd.SCHEDULE_GRID:
            assert p["split_k"] == s
        if st:
            assert p["stages"] == st
            if var == qgd.VARIANT_SWAP_AB and (sch == qgd.SCHEDULE_GRID or occ == 2) and not fz:
                mpad = tune.swap_mpad(M)
                smem = 1024 + st * kps * (16384 + mpad * 128) + 1024 + ((128 + 8) * mpad * 4 if r == 3 else 0)
                assert 2 * (smem + 1024) <= 233472
    qgd.qgd_set_override(fid)
    qgd.qgd_set_fused_override(fid)
    # pair tiles split K (any count) only where they are fewer than the SM pairs
    pair_splits = sorted({c[1] for c in cands if c[0] == qgd.VARIANT_STANDARD_PAIR and c[1] > 1})
    pair_tiles = -(-M // 256) * -(-N // 256)
    assert pair_splits == ([2, 3, 4, 5, 6] if fmt in ("fp8_dynamic", "w8a8_int8") and M > 128 and pair_tiles < 74
                           else [])


def test_fused_plan_field():
    G, P = qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
    fid = qgd.FMT_FP8_DYNAMIC
    # not fused by default; the qlinear_* plan never is
    assert qgd.qgd_get_layer_plan(fid, 4, 4096, 4096)["fused"] == 0
    qgd.qgd_set_fused_override(fid, 1)
    qgd.qgd_set_override(fid, qgd.VARIANT_SWAP_AB, 4, qgd.REDUCE_TWO_PASS, 0, 0, G, 0, 2)
    lp = qgd.qgd_get_layer_plan(fid, 4, 4096, 4096)
    assert lp["fused"] == 1 and lp["source"] == 2
    # the fused kernel has no two-pass reduction: the last CTA adds instead
    assert lp["reduce"] == qgd.REDUCE_LAST_CTA
    assert qgd.qgd_get_plan(fid, 4, 4096, 4096)["fused"] == 0
    # a fused layer call needs only the GEMM's workspace; unfused it also holds codes and scales
    assert qgd.qgd_layer_workspace_size(fid, 4, 4096, 4096) == qgd.qgd_workspace_size(fid, 4, 4096, 4096)
    qgd.qgd_set_fused_override(fid, 0)
    ws0 = qgd.qgd_layer_workspace_size(fid, 4, 4096, 4096)
    assert ws0 >= qgd.qgd_workspace_size(fid, 4, 4096, 4096) + 4 * 4096 + 4 * 4
    # Standard plans are never fused
    qgd.qgd_set_fused_override(fid, 1)
    qgd.qgd_set_override(fid, qgd.VARIANT_STANDARD, 1, 0, 0, 128, P)
    assert qgd.qgd_get_layer_plan(fid, 64, 4096, 4096)["fused"] == 0
    with pytest.raises(qgd.QGDError):
        qgd.qgd_set_fused_override(fid, 2)
    qgd.qgd_set_fused_override(fid)


def test_table_fused_column(tmp_path):
    t = tmp_path / "t.tsv"
    t.write_text("fp8_dynamic 4096 4096 1 swap_ab 8 cluster 2 128 grid 0 2 1\n"
                 "fp8_dynamic 4096 4096 2 swap_ab 8 cluster 2 128 grid 0 2 0\n")
    qgd.qgd_load_dispatch_table(str(t))
    assert qgd.qgd_get_layer_plan(0, 1, 4096, 4096)["fused"] == 1
    assert qgd.qgd_get_layer_plan(0, 2, 4096, 4096)["fused"] == 0
    assert qgd.qgd_get_plan(0, 1, 4096, 4096)["fused"] == 0
    t.write_text("fp8_dynamic 4096 4096 1 swap_ab 8 cluster 2 128 grid 0 2 3\n")
    with pytest.raises(qgd.QGDError):
        qgd.qgd_load_dispatch_table(str(t))



def test_swap_ab_up_to_128_tokens():
    G = qgd.SCHEDULE_GRID
    for M in (33, 64, 100, 128):
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 4, qgd.REDUCE_TWO_PASS, 0, 0, G, 0, 1)
        p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, M, 4096, 4096)
        # Swap-AB covers up to 128 tokens; its two-pass kernel only 32, so the last CTA adds
        assert p["variant"] == qgd.VARIANT_SWAP_AB and p["reduce"] == qgd.REDUCE_LAST_CTA
        # partial rows are padded to 4 tokens
        assert qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, M, 4096, 4096) == 64 * 1024 + 32 * 4 * 128 * (-(-M // 4) * 4) * 4
    p = qgd.qgd_get_plan(qgd.FMT_FP8_DYNAMIC, 129, 4096, 4096)
    assert p["variant"] == qgd.VARIANT_STANDARD
    qgd.qgd_set_override(qgd.FMT_BLOCK_FP8, qgd.VARIANT_SWAP_AB, 4, 0, 0, 0, G, 0, 1)
    assert qgd.qgd_get_plan(qgd.FMT_BLOCK_FP8, 33, 4096, 4096)["variant"] == qgd.VARIANT_STANDARD


def test_shipped_table_covers_every_benchmarked_shape():
    # the shipped table parses, names only legal plans, and has an entry for every
    # (format, N, K, M) the benchmark runs, so no benchmarked call falls back to
    # the built-in default
    from quantized_gemm_decode_b200 import workloads

    qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
    fid = {"fp8_dynamic": 0, "w8a8_int8": 1, "block_fp8": 2}
    for wl in (workloads.FP8_DECODE, workloads.INT8_DECODE, workloads.BLOCK_DECODE, *workloads.LARGE):
        for (N, K) in wl.shapes:
            for M in wl.ms:
                p = qgd.qgd_get_plan(fid[wl.fmt], M, N, K)
                assert p["source"] == 1, (wl.fmt, N, K, M)
                if p["variant"] == qgd.VARIANT_SWAP_AB:
                    assert M <= (32 if wl.fmt == "block_fp8" else 128)
                # the workspace the plan needs is what the size query reports
                assert qgd.qgd_workspace_size(fid[wl.fmt], M, N, K) >= 0


def test_shipped_table_entries_run_as_written():
    # every entry of the shipped table is what a call of its bucket's token
    # count runs, field for field: none is silently legalised into another plan
    for f in range(5):
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f)
    qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
    fid = {"fp8_dynamic": 0, "w8a8_int8": 1, "block_fp8": 2, "mxfp8": 3, "nvfp4": 4}
    var = {"standard": 0, "swap_ab": 1, "standard_pair": 2}
    red = {"last_cta": 0, "two_pass": 1, "atomic": 2, "cluster": 3}
    sch = {"grid": 0, "persistent": 1}
    n = 0
    for ln in open(qgd.DEFAULT_TABLE):
        f = ln.split("#")[0].split()
        if not f:
            continue
        fmt, N, K, M = fid[f[0]], int(f[1]), int(f[2]), int(f[3])
        want = dict(variant=var[f[4]], split_k=int(f[5]), reduce=red[f[6]], stages=int(f[7]), tile_n=int(f[8]),
                    schedule=sch[f[9]], occupancy=int(f[10]), k_slices=int(f[11]))
        p = qgd.qgd_get_plan(fmt, M, N, K)
        got = {k: p[k] for k in want}
        assert got == want and p["source"] == 1, (ln, got)
        assert qgd.qgd_get_layer_plan(fmt, M, N, K)["fused"] == int(f[12]), ln
        n += 1
    assert n > 200


def test_tuner_reads_back_every_shipped_table_line():
    # the tuner's table-line parser (used by --resume / --recheck) gives back the
    # plan each line names, in the override calls' argument order, and its time
    from quantized_gemm_decode_b200 import tune

    qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
    for ln in open(qgd.DEFAULT_TABLE):
        parsed = tune.parse_table_line(ln)
        if parsed is None:
            assert ln.startswith("#") or not ln.strip()
            continue
        (fmt, N, K, M), plan, us = parsed
        assert us is not None and us > 0, ln
        fid = tune.FMT_ID[fmt]
        qgd.qgd_clear_dispatch_table()
        qgd.qgd_set_override(fid, *plan[:8])
        qgd.qgd_set_fused_override(fid, plan[8])
        try:
            p = qgd.qgd_get_layer_plan(fid, M, N, K)
        finally:
            qgd.qgd_set_override(fid)
            qgd.qgd_set_fused_override(fid)
            qgd.qgd_load_dispatch_table(qgd.DEFAULT_TABLE)
        assert (p["variant"], p["split_k"], p["reduce"], p["stages"], p["tile_n"], p["schedule"], p["k_slices"],
                p["fused"]) == (plan[0], plan[1], plan[2], plan[3], plan[4], plan[5], plan[7], plan[8]), ln
        # and the writer gives the line back byte for byte from what was read
        gbs = float(ln.split("#")[1].split(",")[1].split()[0])
        assert tune.format_table_line((fmt, N, K, M), plan, us, gbs) == ln.rstrip("\n")
    assert tune.parse_table_line("   # only a comment") is None
    with pytest.raises(ValueError):
        tune.parse_table_line("fp8_dynamic 4096 4096 1 swap_ab 1")
    # stale: more than PCT percent slower than recorded, or nothing recorded
    assert not tune.is_stale(10.0, 11.4, 15.0) and tune.is_stale(10.0, 11.6, 15.0)
    assert tune.is_stale(None, 1.0, 15.0)


def test_binding_checks_gemm_operands_before_any_launch():
    # CPU tensors: every shape / dtype / size check runs before the device
    # check, so each mistake is reported as what it is, and nothing reaches
    # the library
    import torch

    M, N, K = 4, 256, 512
    f8 = torch.float8_e4m3fn
    xq = torch.zeros((M, K), dtype=f8)
    wq = torch.zeros((N, K), dtype=f8)
    sx = torch.ones(M)
    sw = torch.ones(N)
    y = torch.zeros((M, N), dtype=torch.bfloat16)
    cases = [
        (dict(wq=torch.zeros((N, K - 128), dtype=f8)), "K mismatch"),
        (dict(sx=torch.ones(M - 1)), "sx holds"),
        (dict(sw=torch.ones(N - 16)), "sw holds"),
        (dict(sw=torch.ones(N, dtype=torch.float64)), "sw must be"),
        (dict(y=torch.zeros((M, N - 16), dtype=torch.bfloat16)), "y must be"),
        (dict(y=torch.zeros((M, N), dtype=torch.float32)), "y must be"),
        (dict(xq=torch.zeros((M, K), dtype=torch.int8)), "xq has dtype"),
        ({}, "must be a CUDA tensor"),
    ]
    for change, msg in cases:
        args = dict(xq=xq, sx=sx, wq=wq, sw=sw, y=y) | change
        for fn in (qgd.qlinear_fp8_dynamic, qgd.qlinear_fp8_dynamic_noalloc):
            with pytest.raises(ValueError, match=msg):
                fn(args["xq"], args["sx"], args["wq"], args["sw"], y=args["y"])
    with pytest.raises(ValueError, match="y is None"):
        qgd.qlinear_fp8_dynamic_noalloc(xq, sx, wq, sw, None)
    # Block_FP8 scales: [M, K/128] and [N/128, K/128]
    with pytest.raises(ValueError, match="sw holds"):
        qgd.qlinear_block_fp8(xq, torch.ones(M, K // 128), wq, torch.ones(N // 128, K // 128 - 1), y=y)
    # W8A8_INT8 codes are int8
    with pytest.raises(ValueError, match="xq has dtype"):
        qgd.qlinear_w8a8_int8(xq, sx, wq, sw, y=y)


def test_strided_quantizer_rejects_bad_row_stride():
    L = qgd.lib()
    P = ctypes.c_void_p
    # ldx below K, or not a multiple of 8: refused before any launch
    assert L.quant_act_per_token_strided(P(16), 4, 512, 500, 0, P(16), P(16), None) == -1
    assert L.quant_act_per_token_strided(P(16), 4, 512, 516, 0, P(16), P(16), None) == -1
    assert L.quant_act_group128_strided(P(16), 4, 512, 256, P(16), P(16), None) == -1
    # an empty call with a valid stride is fine
    assert L.quant_act_per_token_strided(P(16), 0, 512, 1024, 0, P(16), P(16), None) == 0


def test_layer_call_rejects_bad_arguments():
    L = qgd.lib()
    P = ctypes.c_void_p
    # row stride below K, misaligned x, null operands: refused before any launch
    assert L.qlinear_fp8_dynamic_bf16(P(16), 512, P(16), P(16), P(16), 4, 512, 1024, None, 0, None) == -1
    assert L.qlinear_fp8_dynamic_bf16(P(17), 1024, P(16), P(16), P(16), 4, 512, 1024, None, 0, None) == -1
    assert L.qlinear_w8a8_int8_bf16(None, 1024, P(16), P(16), P(16), 4, 512, 1024, None, 0, None) == -1
    assert L.qlinear_block_fp8_bf16(P(16), 1000, P(16), P(16), P(16), 4, 512, 1000, None, 0, None) == -2
    # an empty call is fine
    assert L.qlinear_fp8_dynamic_bf16(None, 1024, None, None, None, 0, 512, 1024, None, 0, None) == 0


def test_nvfp4_plan_rules_and_rejects():
    F = qgd.FMT_NVFP4
    # Swap-AB only, no two-pass reduction, the ring capped by tensor memory:
    # 2 x 16 accumulator columns + 32 scale-factor columns per (stage, K slice) <= 256
    qgd.qgd_set_override(F, qgd.VARIANT_STANDARD, 4, qgd.REDUCE_TWO_PASS, 0, 0, qgd.SCHEDULE_GRID, 0, 1)
    p = qgd.qgd_get_plan(F, 8, 4096, 4096)
    assert (p["variant"], p["reduce"]) == (qgd.VARIANT_SWAP_AB, qgd.REDUCE_LAST_CTA)
    assert 2 * 16 + p["stages"] * p["k_slices"] * 32 <= 256
    qgd.qgd_set_override(F, qgd.VARIANT_SWAP_AB, 1, 0, 0, 0, qgd.SCHEDULE_PERSISTENT, 1, 2)
    p = qgd.qgd_get_plan(F, 64, 4096, 4096)
    assert p["k_slices"] == 2 and 2 * 64 + p["stages"] * 2 * 32 <= 256
    # K units count 128-byte slices of packed codes: K = 4096 values is 16 slices
    qgd.qgd_set_override(F, qgd.VARIANT_SWAP_AB, 32, 0, 0, 0, qgd.SCHEDULE_GRID, 0, 1)
    assert qgd.qgd_get_plan(F, 4, 4096, 4096)["split_k"] == 16
    qgd.qgd_set_override(F)
    L = qgd.lib()
    P = ctypes.c_void_p
    assert L.qlinear_nvfp4(P(16), P(16), P(16), P(16), P(16), P(16), P(16), 4, 512, 1152, None, 0, None) == -2
    assert L.qlinear_nvfp4(P(16), P(16), P(16), P(16), P(16), P(16), P(16), 129, 512, 1024, None, 0, None) == -2
    assert L.quant_nvfp4(P(16), 4, 1000, 1000, P(16), P(16), P(16), None) == -2
    assert L.qlinear_nvfp4(P(16), None, P(16), P(16), P(16), P(16), P(16), 4, 512, 1024, None, 0, None) == -1
    # the layer workspace holds the packed codes, the row scales and the block scales
    ws = qgd.qgd_layer_workspace_size(F, 8, 4096, 4096)
    assert ws >= 8 * 2048 + 8 * 4 + 8 * 256


def _tp_desc(ranks=2, rank=0, col0=0, ldy=512, null_y=False):
    d = qgd._Tp()
    d.ranks, d.rank, d.col0, d.ldy = ranks, rank, col0, ldy
    for r in range(min(max(ranks, 0), qgd.MAX_TP_RANKS)):
        d.y[r] = None if null_y and r == ranks - 1 else 4096 * (r + 1)
        d.flags[r] = 8192 * (r + 1)
    return d


def test_column_parallel_call_rules():
    L = qgd.lib()
    P = ctypes.c_void_p
    for name in ("qlinear_tp_bf16", "qgd_tp_wait", "qgd_tp_workspace_size", "qgd_ipc_malloc", "qgd_ipc_open",
                 "qgd_ipc_close", "qgd_ipc_free"):
        assert name in declared_functions()
    assert ctypes.sizeof(qgd._Tp) == 4 * 4 + 2 * 8 * 8  # four ints, two pointer arrays
    # the workspace always holds the 64 KiB counter header (its last word counts finished CTAs)
    for fmt in range(5):
        assert qgd.qgd_tp_workspace_size(fmt, 4, 256, 1024) >= 64 * 1024
        assert qgd.qgd_tp_workspace_size(fmt, 4, 256, 1024) >= qgd.qgd_layer_workspace_size(fmt, 4, 256, 1024)

    def call(desc, fmt=0, M=4, N=256, K=1024, ws=P(1 << 20), wsn=1 << 20):
        return L.qlinear_tp_bf16(fmt, P(16), K, P(16), P(16), None, M, N, K,
                                 ctypes.byref(desc) if desc is not None else None, ws, wsn, None)

    assert call(None) == -1
    assert call(_tp_desc(ranks=0)) == -1
    assert call(_tp_desc(ranks=9)) == -1
    assert call(_tp_desc(rank=2)) == -1
    assert call(_tp_desc(col0=300)) == -1                 # shard past the full output
    assert call(_tp_desc(ldy=260)) == -1                  # not a multiple of 8
    assert call(_tp_desc(null_y=True)) == -1
    assert call(_tp_desc(), fmt=0, M=129) == -2           # beyond the Swap-AB kernel's 128 tokens
    assert call(_tp_desc(), fmt=2, M=33) == -2            # Block_FP8: 32
    assert call(_tp_desc(), fmt=4, M=129, K=1024) == -2   # NVFP4: 128
    assert call(_tp_desc(), ws=None, wsn=0) == -3
    assert call(_tp_desc(), fmt=5) == -1
    assert L.qgd_tp_wait(None, 1, None) == -1
    assert L.qgd_tp_wait(P(16), 0, None) == -1
    assert L.qgd_tp_wait(P(16), 9, None) == -1
    assert L.qgd_tp_wait(P(18), 1, None) == -1
    p = ctypes.c_void_p(0)
    assert L.qgd_ipc_malloc(0, ctypes.byref(p), ctypes.create_string_buffer(64)) == -1
    assert L.qgd_ipc_malloc(256, None, ctypes.create_string_buffer(64)) == -1
    assert L.qgd_ipc_open(None, ctypes.byref(p)) == -1
    assert L.qgd_ipc_close(None) == -1 and L.qgd_ipc_free(None) == -1


def test_pdl_setting_is_validated_and_cached():
    L = qgd.lib()
    for bad in (-2, 2, 7):
        assert L.qgd_set_pdl(bad) == -1
    for ok in (0, 1, -1):
        assert L.qgd_set_pdl(ok) == 0
