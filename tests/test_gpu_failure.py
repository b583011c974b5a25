"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every mbarrier wait in the GEMM kernels gives up after about one second,
records an error code for qgd_device_error(), waits for the copies and MMAs
its CTA issued, frees tensor memory and returns.  Here a test hook withholds
the signal the epilogue waits for (a flag that nothing sets), so that wait
runs out for real.  Nothing is left in flight when it does: the producer's
copies and the MMAs complete on their own.  The call must return, report the
epilogue-wait code, write nothing, and leave the context usable for a normal
call that matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200.workloads import FP8_DYNAMIC
from paritylib import Case

pytestmark = pytest.mark.gpu

ERR_WAIT_EPILOGUE = 3


@pytest.fixture(autouse=True)
def _clean():
    qgd.lib()
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)
    qgd.qgd_test_withhold_accumulator(False)
    qgd.qgd_clear_device_error()
    yield
    qgd.qgd_test_withhold_accumulator(False)
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC)
    qgd.qgd_clear_device_error()


def test_epilogue_wait_runs_out_and_is_reported():
    case = Case(FP8_DYNAMIC, 4, 512, 1024, seed=31)
    # one segment per CTA (grid schedule, no split): the MMA issuer never
    # waits on the epilogue, so only the epilogue's wait runs out
    qgd.qgd_set_override(qgd.FMT_FP8_DYNAMIC, qgd.VARIANT_SWAP_AB, 1, qgd.REDUCE_LAST_CTA, 0, 0,
                         qgd.SCHEDULE_GRID)
    y = torch.full((case.M, case.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    qgd.qgd_test_withhold_accumulator(True)
    try:
        qgd.qlinear_fp8_dynamic(case.xq, case.sx, case.wq, case.sw, y=y)
    finally:
        qgd.qgd_test_withhold_accumulator(False)
    t0 = time.time()
    code = qgd.qgd_device_error()  # synchronizes: the kernel has returned
    waited = time.time() - t0
    assert code == ERR_WAIT_EPILOGUE, code
    assert waited < 30.0
    assert torch.isnan(y.float()).all(), "an aborted call wrote output"
    qgd.qgd_clear_device_error()
    assert qgd.qgd_device_error() == 0
    # the context is still usable: the same call, unhooked, matches the oracle
    yref, bound = case.oracle_gemm(*case.oracle_quant())
    case.check_output(case.run(), yref, bound, "after the aborted call")
    assert qgd.qgd_device_error() == 0
