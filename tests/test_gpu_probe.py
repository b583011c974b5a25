"""The dense tensor-core peak probe: it runs to completion without a device
error, reports the FLOP count of its launch, and its timed rate is in a
physically plausible band (well above the bf16 rate the large-M roofline
would otherwise scale, below the e4m3/int8 data-sheet figure plus margin)."""
import pytest
import torch

import quantized_gemm_decode_b200 as qgd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("qtype", [qgd.QTYPE_E4M3, qgd.QTYPE_INT8])
def test_probe_rate_is_plausible(qtype):
    qgd.qgd_clear_device_error()
    flops = qgd.qgd_mma_peak_probe(qtype, 64)  # warm-up
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert flops == 2 * 128 * 256 * 128 * 64 * sms
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    flops = qgd.qgd_mma_peak_probe(qtype, 8192)
    e1.record()
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 0
    tflops = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert 1000.0 < tflops < 6000.0, tflops


def test_ring_probe_runs_and_waited_wide_groups_keep_the_rate():
    qgd.qgd_clear_device_error()
    rates = {}
    for n, slots, wait in ((256, 2, True), (128, 4, True), (128, 4, False), (128, 1, True), (256, 1, False)):
        qgd.qgd_mma_ring_probe(n, slots, wait, 64)  # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        flops = qgd.qgd_mma_ring_probe(n, slots, wait, 4096)
        e1.record()
        torch.cuda.synchronize()
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert flops == 2 * 128 * n * 128 * 4096 * sms
        rates[(n, slots, wait)] = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert qgd.qgd_device_error() == 0
    assert all(500.0 < r < 6000.0 for r in rates.values()), rates
