"""The decode workloads the library is measured and parity-tested on.

Layer shapes (N, K) follow the linear layers of dense decoder models of three
sizes (qkv, o, gate_up, down); token counts M are the decode buckets the
method tunes separately: 1, 2, 4, 8, 16, 24, 32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

FP8_DYNAMIC = "fp8_dynamic"
W8A8_INT8 = "w8a8_int8"
BLOCK_FP8 = "block_fp8"
MXFP8 = "mxfp8"
NVFP4 = "nvfp4"
FORMATS = (FP8_DYNAMIC, W8A8_INT8, BLOCK_FP8)  # the three formats of the method; MXFP8 and NVFP4 are additions

DECODE_M = (1, 2, 4, 8, 16, 24, 32)
LARGE_M = (64, 128, 512, 2048, 8192)

# (N, K) of the qkv, o, gate_up and down projections
SHAPES_8B = ((6144, 4096), (4096, 4096), (24576, 4096), (4096, 12288))
SHAPES_14B = ((7168, 5120), (5120, 5120), (34816, 5120), (5120, 17408))
SHAPES_32B = ((10240, 5120), (5120, 8192), (51200, 5120), (5120, 25600))


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str
    shapes: tuple
    ms: tuple
    seed: int
    outliers: bool
    description: str = field(default="", compare=False)

    def calls(self):
        """(M, N, K) of every GEMM in one pass, M outer so each weight is
        re-read only after every other weight of the pass has streamed."""
        return [(m, n, k) for m in self.ms for (n, k) in self.shapes]


TINY = Workload("fp8_dynamic_tiny_m4_n512_k1024", FP8_DYNAMIC, ((512, 1024),), (4,), 0, False,
                "FP8_Dynamic, X 4x1024 ~N(0,1), W 512x1024 ~N(0,0.02)")
FP8_DECODE = Workload("fp8_dynamic_decode_sweep_8b_shapes", FP8_DYNAMIC, SHAPES_8B, DECODE_M, 1001, True,
                      "FP8_Dynamic, 8B-class shapes x M in 1..32, 1% x20 outlier channels")
INT8_DECODE = Workload("w8a8_int8_decode_sweep_14b_shapes", W8A8_INT8, SHAPES_14B, DECODE_M, 1002, False,
                       "W8A8_INT8, 14B-class shapes x M in 1..32")
BLOCK_DECODE = Workload("block_fp8_decode_sweep_32b_shapes", BLOCK_FP8, SHAPES_32B, DECODE_M, 1003, True,
                        "Block_FP8, 32B-class shapes x M in 1..32, 1% x20 outlier channels")
MX_DECODE = Workload("mxfp8_decode_sweep_8b_shapes", MXFP8, SHAPES_8B, DECODE_M, 1005, True,
                     "MXFP8 (E8M0 scales per 32 values along K), 8B-class shapes x M in 1..32, "
                     "1% x20 outlier channels")
LARGE = tuple(
    Workload(f"{fmt}_large_m_8b_shapes", fmt, SHAPES_8B, LARGE_M, 1004, fmt != W8A8_INT8,
             f"{fmt}, 8B-class shapes x M in 64..8192")
    for fmt in FORMATS)

NV_DECODE = Workload("nvfp4_decode_sweep_8b_shapes", NVFP4, SHAPES_8B, DECODE_M, 1006, True,
                     "NVFP4 (E2M1 values, E4M3 scale per 16 along K, fp32 per row), 8B-class shapes x M in 1..32, "
                     "1% x20 outlier channels")
# the block-scaled formats past the decode buckets: their kernels cover up to 128 tokens
MID_M = (64, 128)
LARGE_BS = tuple(
    Workload(f"{fmt}_mid_m_8b_shapes", fmt, SHAPES_8B, MID_M, 1008, True, f"{fmt}, 8B-class shapes x M in 64, 128")
    for fmt in (MXFP8, NVFP4))

# one rank's weight shard of the 8B-class layers split column-parallel over 8 GPUs
SHAPES_8B_TP8 = tuple((n // 8, k) for (n, k) in SHAPES_8B)
FP8_TP8 = Workload("fp8_dynamic_decode_tp8_shards_8b", FP8_DYNAMIC, SHAPES_8B_TP8, DECODE_M, 1007, True,
                   "FP8_Dynamic, one of 8 column-parallel shards of the 8B-class shapes x M in 1..32")
ALL = (TINY, FP8_DECODE, INT8_DECODE, BLOCK_DECODE, MX_DECODE, NV_DECODE, FP8_TP8) + LARGE + LARGE_BS


def algorithmic_bytes(fmt: str, M: int, N: int, K: int) -> int:
    """Bytes a GEMM call must move at minimum: 1-byte weight and activation
    codes, fp32 scales, bf16 output."""
    if fmt == BLOCK_FP8:
        scales = 4 * (N // 128) * (K // 128) + 4 * M * (K // 128)
    elif fmt == MXFP8:
        scales = N * (K // 32) + M * (K // 32)  # one E8M0 byte per 32 values
    elif fmt == NVFP4:
        # half a byte per value, one E4M3 byte per 16, an fp32 per row
        return (N * K + M * K) // 2 + (N + M) * (K // 16) + 4 * (N + M) + 2 * M * N
    else:
        scales = 4 * N + 4 * M
    return N * K + M * K + scales + 2 * M * N


def flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K
