"""The FP8_Dynamic GEMM entry point that allocates nothing.

Some callers cannot allocate device memory while they run the layer: a
serving engine that carved all device memory into fixed pools at start-up
has none left for a per-call workspace, and a latency-critical loop cannot
afford a cudaMalloc that may wait for the device to go idle.  For them
qlinear_fp8_dynamic_noalloc takes no workspace and uses a fixed scratch array
built into the library.  These checks call it through the C ABI, on two
calls in a row, and hold its output both to the regular entry point's (same
plan, caller-provided workspace) and to the oracle's, with the FP8 tolerance
the other GPU tests use.

This file is named to run last, so that a run stopping at the first failure
has already run every other test; it sets and clears its own plan overrides,
so it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200.workloads import FP8_DYNAMIC
from paritylib import Case, bf16_to_f64, check_fp8_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _plan_overrides_cleared():
    qgd.lib()
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)
    yield
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)


def _noalloc(case: Case, y: torch.Tensor) -> int:
    L = qgd.lib()
    P = ctypes.c_void_p
    st = L.qlinear_fp8_dynamic_noalloc(P(case.xq.data_ptr()), P(case.sx.data_ptr()), P(case.wq.data_ptr()),
                                       P(case.sw.data_ptr()), P(y.data_ptr()), case.M, case.N, case.K,
                                       P(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("split,reduce", [(None, None), (8, qgd.REDUCE_LAST_CTA), (4, qgd.REDUCE_TWO_PASS),
                                          (8, qgd.REDUCE_ATOMIC), (1, qgd.REDUCE_LAST_CTA)])
def test_noalloc_matches_workspace_entry_point_twice(split, reduce):
    case = Case(FP8_DYNAMIC, 8, 1024, 4096, seed=21)
    if split is not None:
        qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, split, reduce, 0, 0, qgd.SCHEDULE_GRID)
    # the regular entry point, with a workspace the caller allocated
    ws = qgd.Workspace(qgd.qgd_workspace_size(qgd.FMT_FP8_DYNAMIC, case.M, case.N, case.K))
    y_ws = bf16_to_f64(case.run(ws=ws))
    yref, bound = case.oracle_gemm(*case.oracle_quant())
    for call in range(2):
        y = torch.full((case.M, case.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(case, y) == 0, qgd.lib().qgd_last_error_message()
        torch.cuda.synchronize()
        got = bf16_to_f64(y)
        check_fp8_tolerance(got, yref, bound, case.K, f"no-alloc call {call} vs the oracle")
        check_fp8_tolerance(got, y_ws, bound, case.K, f"no-alloc call {call} vs the workspace entry point")
    assert qgd.qgd_device_error() == 0


def test_noalloc_rejects_scratch_beyond_its_size():
    # 8 splits x 32 tokens x 16384 columns of fp32 partials is 16 MiB, more
    # than the 8 MiB built-in scratch: refused before anything is launched
    case = Case(FP8_DYNAMIC, 32, 16384, 1024, seed=22)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 8, qgd.REDUCE_LAST_CTA, 0, 0,
                         qgd.SCHEDULE_GRID)
    y = torch.zeros((case.M, case.N), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(case, y) == -3
    assert b"built-in scratch" in qgd.lib().qgd_last_error_message()
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
