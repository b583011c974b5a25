"""CPU checks of the benchmark's bookkeeping: the byte counts the roofline
fractions divide by, and the rule that DRAM traffic is reported only for the
kernel source it was captured on."""
import hashlib
import os

import bench
from quantized_gemm_decode_b200 import workloads
from quantized_gemm_decode_b200.workloads import BLOCK_FP8, FP8_DYNAMIC, W8A8_INT8


def test_gemm_algorithmic_bytes():
    # weight codes + activation codes + scales + bf16 output
    assert workloads.algorithmic_bytes(FP8_DYNAMIC, 1, 24576, 4096) == 24576 * 4096 + 4096 + 4 * 24576 + 4 + 2 * 24576
    assert workloads.algorithmic_bytes(W8A8_INT8, 32, 5120, 5120) == 5120 * 5120 + 32 * 5120 + 4 * 5120 + 4 * 32 + 2 * 32 * 5120
    kb = 5120 // 128
    assert workloads.algorithmic_bytes(BLOCK_FP8, 8, 10240, 5120) == (
        10240 * 5120 + 8 * 5120 + 4 * (10240 // 128) * kb + 4 * 8 * kb + 2 * 8 * 10240)
    assert workloads.flops(8, 10240, 5120) == 2 * 8 * 10240 * 5120


def test_path_and_quantizer_bytes():
    # whole path: bf16 X in (the codes between the two kernels are not counted)
    assert bench.path_bytes(FP8_DYNAMIC, 4, 4096, 4096) == 4096 * 4096 + 2 * 4 * 4096 + 4 * 4096 + 2 * 4 * 4096
    assert bench.path_bytes(BLOCK_FP8, 4, 4096, 4096) == 4096 * 4096 + 2 * 4 * 4096 + 4 * 32 * 32 + 2 * 4 * 4096
    # quantizer: bf16 in, codes and scales out
    assert bench.quant_bytes(FP8_DYNAMIC, 4, 4096) == 3 * 4 * 4096 + 4 * 4
    assert bench.quant_bytes(BLOCK_FP8, 4, 4096) == 3 * 4 * 4096 + 4 * 4 * 32


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    h = hashlib.sha256()
    for f in ("gemm.cu", "sm100.cuh"):
        h.update(open(os.path.join(bench.ROOT, "quantized_gemm_decode_b200", "csrc", f), "rb").read())
    rec = tmp_path / "profiles"
    rec.mkdir()
    body = "case = test\ndram_over_algorithmic = 1.05\nkernel_source_sha256 = {}\n"
    (rec / "gemm_traffic.txt").write_text(body.format(h.hexdigest()))
    root = tmp_path
    (root / "quantized_gemm_decode_b200").symlink_to(os.path.join(bench.ROOT, "quantized_gemm_decode_b200"))
    monkeypatch.setattr(bench, "ROOT", str(root))
    ok, _ = bench.traffic_record()
    assert ok is not None and float(ok["dram_over_algorithmic"]) == 1.05
    (rec / "gemm_traffic.txt").write_text(body.format("0" * 64))
    stale, rec2 = bench.traffic_record()
    assert stale is None and rec2["kernel_source_sha256"] == "0" * 64


def test_decode_sweeps_match_the_configured_shapes():
    assert list(workloads.FP8_DECODE.shapes) == [(6144, 4096), (4096, 4096), (24576, 4096), (4096, 12288)]
    assert list(workloads.FP8_DECODE.ms) == [1, 2, 4, 8, 16, 24, 32]
    for wl in (workloads.FP8_DECODE, workloads.INT8_DECODE, workloads.BLOCK_DECODE):
        for n, k in wl.shapes:
            assert n % 128 == 0 and k % 128 == 0
