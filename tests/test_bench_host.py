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
    # MXFP8: one E8M0 byte per 32 values of each operand row
    assert workloads.algorithmic_bytes(workloads.MXFP8, 4, 4096, 4096) == (
        4096 * 4096 + 4 * 4096 + 4096 * 128 + 4 * 128 + 2 * 4 * 4096)
    assert bench.path_bytes(workloads.MXFP8, 4, 4096, 4096) == 4096 * 4096 + 2 * 4 * 4096 + 4096 * 128 + 2 * 4 * 4096
    # NVFP4: half a byte per value, one E4M3 byte per 16 values, one fp32 per row
    assert workloads.algorithmic_bytes(workloads.NVFP4, 4, 4096, 4096) == (
        4096 * 2048 + 4 * 2048 + (4096 + 4) * 256 + 4 * (4096 + 4) + 2 * 4 * 4096)
    assert bench.path_bytes(workloads.NVFP4, 4, 4096, 4096) == (
        4096 * 2048 + 4096 * 256 + 4 * 4096 + 2 * 4 * 4096 + 2 * 4 * 4096)
    assert bench.quant_bytes(workloads.NVFP4, 4, 4096) == 2 * 4 * 4096 + 4 * 2048 + 4 * 256 + 4 * 4


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


def _fake_result():
    """A result shaped like a full run's: three formats' per-call tables,
    the larger-M rows, the CPU baseline, clocks and the roofline."""
    row = {"M": 8, "N": 4096, "K": 12288, "us": 14.37, "median_us": 14.082, "p90_us": 15.1, "gbs": 3515.0,
           "frac": 0.5371, "tflops": 56.04, "layer_us": 14.835, "layer_gbs": 3411.4, "plan": "swap/s8/r3/st2/k2"}
    per_call = [dict(row) for _ in range(28)]
    lrow = {"M": 8192, "N": 24576, "K": 4096, "us": 700.0, "tflops": 2300.0, "gbs": 900.0, "bound": "tensor",
            "frac": 0.66, "frac_spec": 0.5, "plan": "std/pers1/r0/st4/k1", "frac_probe": 0.5}
    large = {f: [dict(lrow, M=m) for m in workloads.LARGE_M for _ in range(4)] for f in workloads.FORMATS}
    fmts = {f: {"workload": f + "_decode_sweep", "ms_per_step": 0.4, "gbs": 3400.0, "frac": 0.52,
                "quantizer": {"us_per_call": 1.9, "bytes_per_step": 1000, "gbs": 100.0}, "per_call": per_call}
            for f in workloads.FORMATS}
    return {
        "metric": bench.METRIC, "value": 3455.1, "unit": "GB/s", "n_gpus": 1, "steps": 20, "warmup": 5,
        "ms_per_step": 0.394, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": workloads.FP8_DECODE.name, "format": FP8_DYNAMIC,
                   "shapes": [list(s) for s in workloads.FP8_DECODE.shapes], "ms": list(workloads.FP8_DECODE.ms),
                   "calls_per_step": 28, "graph": "one CUDA graph per step", "l2": "inputs larger than L2 " * 4,
                   "parallelism": "replicas x1"},
        "tflops": 20.0, "frac_of_hbm_peak": 0.53, "frac_of_8tbs": 0.43,
        "roofline": {"bound": "hbm", "kernel": "GEMM", "achieved": 3777.0, "peak": 6545.0, "unit": "GB/s",
                     "frac": 0.577, "peak_source": "measured", "traffic": 50_000_000, "traffic_case": "x" * 80,
                     "avg_launch_us": 12.866, "algorithmic_bytes_per_launch": 48_590_000},
        "e2e": {"value": 2782.0, "unit": "GB/s", "h2d_bytes_per_step": 1_000_000, "d2h_bytes_per_step": 3_000_000,
                "ms_per_step": 0.49, "how": "y" * 200},
        "gpu_launches": 1120, "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "power_w_max": 700.0,
                                         "samples": 40, "reasons": []},
        "formats": fmts, "tensor_probe": {"e4m3_tflops": 4443.0, "int8_tops": 4588.0, "how": "z" * 120},
        "large_m": large, "per_call": per_call,
        "tensor_parallel": [{"M": 1, "N": 4096, "K": 4096, "ranks": 8, "shard_n": 512, "layer_us": 4.1,
                             "tp_us": 4.3}, {"M": 1, "N": 4096, "K": 4096, "ranks": 1, "shard_n": 4096,
                                             "layer_us": 8.4, "tp_us": 8.5, "tp_wait_us": 9.9}],
        "cpu_baseline": {"value": 0.047, "unit": "GB/s", "cores": 16, "kind": "oracle", "sample": "s" * 200,
                         "cpu_model": "Some CPU @ 2.70GHz",
                         "single_thread": {"value": 0.006, "unit": "GB/s", "cores": 1, "seconds": 5.0},
                         "large_m": {"full_s_extrapolated": 4000.0, "label": "extrapolated"}},
    }


def test_result_line_is_compact_and_last(tmp_path):
    import io
    import json

    detail = tmp_path / "detail.json"
    out = io.StringIO()
    line = bench.emit(_fake_result(), str(detail), stream=out)
    lines = out.getvalue().splitlines()
    assert lines[-1] == line
    assert len(line) < bench.HEADLINE_MAX_BYTES, len(line)
    parsed = json.loads(line)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "dtype", "config", "roofline", "e2e", "cpu_baseline", "clocks", "gpu_launches"):
        assert k in parsed, k
    assert parsed["value"] > 0 and parsed["config"]["workload"] == workloads.FP8_DECODE.name
    for k in ("achieved", "peak", "frac", "traffic", "bound", "unit"):
        assert k in parsed["roofline"]
    assert parsed["e2e"]["h2d_bytes_per_step"] > 0 and parsed["e2e"]["d2h_bytes_per_step"] > 0
    assert parsed["cpu_baseline"]["cores"] == 16 and parsed["cpu_baseline"]["single_thread"]["cores"] == 1
    # every earlier line is a detail section, none of which parses as a result
    assert all(ln.startswith("detail ") for ln in lines[:-1])
    # the full record went to the detail file
    full = json.loads(detail.read_text())
    assert len(full["per_call"]) == 28 and len(full["large_m"][FP8_DYNAMIC]) == 20
    assert len(full["tensor_parallel"]) == 2


def test_report_renders_every_section():
    rep = bench.render_report(_fake_result())
    assert "Column-parallel calls on one GPU" in rep and "| 1 | 4096 x 4096 | 8 | 512 | 4.1 | 4.3 |  |" in rep
    assert "Larger M" in rep and "CPU baseline" in rep
