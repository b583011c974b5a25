"""CPU oracle for the quantized linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, exact int64 / fp64); this
module only builds that file with gcc and marshals numpy arrays into it.
Every function's source passage is cited in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

E4M3 = 0
INT8 = 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str) -> ctypes.CDLL:
    """Load a build of oracle.c and declare its signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lg = ctypes.c_long
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_double]
    L.orc_int8_encode.restype = ctypes.c_int8
    L.orc_int8_encode.argtypes = [ctypes.c_double]
    L.orc_quant_rows.restype = None
    L.orc_quant_rows.argtypes = [P, lg, lg, ctypes.c_int, P, P]
    L.orc_quant_groups.restype = None
    L.orc_quant_groups.argtypes = [P, lg, lg, lg, P, P]
    L.orc_quant_blocks.restype = None
    L.orc_quant_blocks.argtypes = [P, lg, lg, lg, P, P]
    L.orc_gemm_rowscaled.restype = None
    L.orc_gemm_rowscaled.argtypes = [P, P, P, P, lg, lg, lg, ctypes.c_int, P, P, P]
    L.orc_gemm_blockscaled.restype = None
    L.orc_gemm_blockscaled.argtypes = [P, P, P, P, lg, lg, lg, lg, P, P]
    L.orc_dot_split.restype = ctypes.c_int64
    L.orc_dot_split.argtypes = [P, lg, P, lg, lg, ctypes.c_int, lg]
    L.orc_num_threads.restype = ctypes.c_int
    L.orc_num_threads.argtypes = []
    L.orc_set_num_threads.restype = ctypes.c_int
    L.orc_set_num_threads.argtypes = [ctypes.c_int]
    L.orc_quant_mx.restype = None
    L.orc_quant_mx.argtypes = [P, lg, lg, P, P]
    L.orc_gemm_mx.restype = None
    L.orc_gemm_mx.argtypes = [P, P, P, P, lg, lg, lg, P, P]
    L.orc_e2m1_decode.restype = ctypes.c_double
    L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.orc_e2m1_encode.restype = ctypes.c_uint8
    L.orc_e2m1_encode.argtypes = [ctypes.c_double]
    L.orc_quant_nv.restype = None
    L.orc_quant_nv.argtypes = [P, lg, lg, P, P, P]
    L.orc_gemm_nv.restype = None
    L.orc_gemm_nv.argtypes = [P, P, P, P, P, P, lg, lg, lg, P, P]
    return L


def compile_source(src_path: str, out_path: str) -> str:
    """Compile a copy of oracle.c (the tests compile deliberately broken
    copies to show that the pins catch them)."""
    subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                    src_path, "-o", out_path, "-lm"], check=True)
    return out_path


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB_PATH)
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a numpy uint16 array of bf16 bit patterns or a torch bf16 tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for unpacking bf16 tensors handed in by tests
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(v))


def int8_encode(v: float) -> int:
    return lib().orc_int8_encode(float(v))


def quant_rows(x, qtype: int):
    """Per-row scaling: x [R, K] bf16 -> (codes [R, K], scales fp32 [R])."""
    xb = _bf16_bits(x)
    R, K = xb.shape
    q = np.empty((R, K), dtype=np.uint8 if qtype == E4M3 else np.int8)
    s = np.empty((R,), dtype=np.float32)
    lib().orc_quant_rows(_ptr(xb), R, K, qtype, _ptr(q), _ptr(s))
    return q, s


def quant_groups(x, G: int = 128):
    """1 x G groups: x [M, K] -> (e4m3 codes [M, K], scales [M, K/G])."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    assert K % G == 0
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // G), dtype=np.float32)
    lib().orc_quant_groups(_ptr(xb), M, K, G, _ptr(q), _ptr(s))
    return q, s


def quant_blocks(w, B: int = 128):
    """B x B blocks: w [N, K] -> (e4m3 codes [N, K], scales [N/B, K/B])."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    assert N % B == 0 and K % B == 0
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // B, K // B), dtype=np.float32)
    lib().orc_quant_blocks(_ptr(wb), N, K, B, _ptr(q), _ptr(s))
    return q, s


def gemm_rowscaled(xq, sx, wq, sw, qtype: int, want_acc: bool = False):
    """Y [M, N] fp64 (and bound, and exact acc when asked) for per-row scales."""
    xq = np.ascontiguousarray(xq)
    wq = np.ascontiguousarray(wq)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2 and sx.shape == (M,) and sw.shape == (N,)
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    acc = np.empty((M, N), dtype=np.int64) if want_acc else None
    lib().orc_gemm_rowscaled(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, qtype,
                             _ptr(y), _ptr(bound), _ptr(acc) if want_acc else None)
    return (y, bound, acc) if want_acc else (y, bound)


def gemm_blockscaled(xq, sx, wq, sw, G: int = 128):
    """Y [M, N] fp64 and bound for 1 x G activation / G x G weight scales."""
    xq = np.ascontiguousarray(xq)
    wq = np.ascontiguousarray(wq)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N, _ = wq.shape
    assert sx.shape == (M, K // G) and sw.shape == (N // G, K // G)
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm_blockscaled(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, G,
                               _ptr(y), _ptr(bound))
    return y, bound


def quant_mx(x):
    """MXFP8 (OCP MX v1.0): x [R, K] bf16, K % 32 == 0 -> (e4m3 codes [R, K],
    E8M0 scale bytes [R, K/32])."""
    xb = _bf16_bits(x)
    R, K = xb.shape
    assert K % 32 == 0
    q = np.empty((R, K), dtype=np.uint8)
    se = np.empty((R, K // 32), dtype=np.uint8)
    lib().orc_quant_mx(_ptr(xb), R, K, _ptr(q), _ptr(se))
    return q, se


def gemm_mx(xq, sx, wq, sw):
    """MXFP8 product: Y [M, N] fp64 and bound from e4m3 codes and E8M0 block
    scales (sx [M, K/32], sw [N, K/32])."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.uint8)
    M, K = xq.shape
    N, _ = wq.shape
    assert sx.shape == (M, K // 32) and sw.shape == (N, K // 32)
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm_mx(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), _ptr(bound))
    return y, bound


def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def quant_nv(x):
    """NVFP4: x [R, K] bf16, K % 16 == 0 -> (packed E2M1 codes [R, K/2], two per
    byte with element 2i in the low nibble; E4M3 block scales [R, K/16]; fp32
    row scales [R])."""
    xb = _bf16_bits(x)
    R, K = xb.shape
    assert K % 16 == 0
    q = np.empty((R, K // 2), dtype=np.uint8)
    s = np.empty((R, K // 16), dtype=np.uint8)
    g = np.empty((R,), dtype=np.float32)
    lib().orc_quant_nv(_ptr(xb), R, K, _ptr(q), _ptr(s), _ptr(g))
    return q, s, g


def gemm_nv(xq, sx, gx, wq, sw, gw):
    """NVFP4 product: Y [M, N] fp64 and bound from packed codes, block scales
    and row scales of both operands."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.uint8)
    gx = np.ascontiguousarray(gx, dtype=np.float32)
    gw = np.ascontiguousarray(gw, dtype=np.float32)
    M, K2 = xq.shape
    N, _ = wq.shape
    K = 2 * K2
    assert sx.shape == (M, K // 16) and sw.shape == (N, K // 16) and gx.shape == (M,) and gw.shape == (N,)
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm_nv(_ptr(xq), _ptr(sx), _ptr(gx), _ptr(wq), _ptr(sw), _ptr(gw), M, N, K, _ptr(y), _ptr(bound))
    return y, bound


def dot_split(xq, m: int, wq, n: int, qtype: int, splits: int) -> int:
    xq = np.ascontiguousarray(xq)
    wq = np.ascontiguousarray(wq)
    K = xq.shape[1]
    return lib().orc_dot_split(_ptr(xq), m, _ptr(wq), n, K, qtype, splits)


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> int:
    """Run the GEMMs on n threads from now on; returns the count in force."""
    return lib().orc_set_num_threads(int(n))


def cpu_model() -> str:
    """Model name of the host CPU (from /proc/cpuinfo), or '' if unknown."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""
