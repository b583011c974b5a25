"""Python binding of libqgd.so, the B200 (sm_100a) quantized linear-layer library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI (include/qgd.h).  PyTorch supplies device memory and
streams.  The functions keep the C names:

    quant_act_per_token, quant_act_group128, quant_weight_block128,
    qlinear_fp8_dynamic, qlinear_w8a8_int8, qlinear_block_fp8,
    qgd_w8a8_int8_acc32, qgd_workspace_size, qgd_load_dispatch_table,
    qgd_clear_dispatch_table, qgd_set_override, qgd_get_plan, qgd_m_bucket,
    qgd_device_error, qgd_clear_device_error

There is no fallback: if libqgd.so is missing or cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

__all__ = [
    "QGDError", "lib", "FMT_FP8_DYNAMIC", "FMT_W8A8_INT8", "FMT_BLOCK_FP8", "QTYPE_E4M3", "QTYPE_INT8",
    "VARIANT_STANDARD", "VARIANT_SWAP_AB", "VARIANT_STANDARD_PAIR", "REDUCE_LAST_CTA", "REDUCE_TWO_PASS", "REDUCE_ATOMIC", "REDUCE_CLUSTER",
    "SCHEDULE_GRID", "SCHEDULE_PERSISTENT",
    "quant_act_per_token", "quant_act_group128", "quant_weight_block128", "quant_weight_per_channel",
    "quant_act_per_token_strided", "quant_act_group128_strided", "quant_mx", "qlinear_mxfp8", "FMT_MXFP8",
    "quant_nv", "qlinear_nvfp4", "qlinear_nvfp4_bf16", "FMT_NVFP4",
    "qlinear_fp8_dynamic", "qlinear_w8a8_int8", "qlinear_block_fp8", "qgd_w8a8_int8_acc32",
    "qlinear_fp8_dynamic_noalloc",
    "qgd_workspace_size", "qgd_load_dispatch_table", "qgd_clear_dispatch_table", "qgd_set_override",
    "qgd_get_plan", "qgd_m_bucket", "qgd_device_error", "qgd_clear_device_error", "qgd_version",
    "qgd_mma_peak_probe", "qgd_mma_ring_probe", "qgd_test_withhold_accumulator", "qgd_set_pdl",
    "qlinear_bf16", "qgd_layer_workspace_size", "qgd_get_layer_plan", "qgd_set_fused_override",
    "qgd_test_capture_fused",
    "MAX_TP_RANKS", "qlinear_tp_bf16", "qgd_tp_workspace_size", "qgd_tp_wait", "ipc_malloc", "ipc_open",
    "ipc_close", "ipc_free", "tensor_at",
    "Workspace", "DEFAULT_TABLE",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
# QGD_LIBRARY points the binding at another build of the same C ABI (for
# example a build with developer tracing compiled in).
LIB_PATH = os.environ.get("QGD_LIBRARY") or os.path.join(_PKG, "libqgd.so")
DEFAULT_TABLE = os.path.join(_PKG, "tables", "b200.tsv")

FMT_FP8_DYNAMIC, FMT_W8A8_INT8, FMT_BLOCK_FP8, FMT_MXFP8, FMT_NVFP4 = 0, 1, 2, 3, 4
QTYPE_E4M3, QTYPE_INT8 = 0, 1
VARIANT_STANDARD, VARIANT_SWAP_AB, VARIANT_STANDARD_PAIR = 0, 1, 2
REDUCE_LAST_CTA, REDUCE_TWO_PASS, REDUCE_ATOMIC, REDUCE_CLUSTER = 0, 1, 2, 3
SCHEDULE_GRID, SCHEDULE_PERSISTENT = 0, 1
FORMAT_NAMES = {"fp8_dynamic": 0, "w8a8_int8": 1, "block_fp8": 2, "mxfp8": 3}

_lock = threading.Lock()
_lib = None


class QGDError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {message} (status {status})")
        self.status = status


MAX_TP_RANKS = 8
IPC_HANDLE_BYTES = 64


class _Tp(ctypes.Structure):
    _fields_ = [("ranks", ctypes.c_int), ("rank", ctypes.c_int), ("col0", ctypes.c_int), ("ldy", ctypes.c_int),
                ("y", ctypes.c_void_p * MAX_TP_RANKS), ("flags", ctypes.c_void_p * MAX_TP_RANKS)]


class _Plan(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int), ("split_k", ctypes.c_int), ("reduce", ctypes.c_int),
                ("stages", ctypes.c_int), ("tile_n", ctypes.c_int), ("schedule", ctypes.c_int),
                ("occupancy", ctypes.c_int), ("source", ctypes.c_int), ("k_slices", ctypes.c_int),
                ("fused", ctypes.c_int)]


def lib() -> ctypes.CDLL:
    """Load libqgd.so (built in-tree by quantized_gemm_decode_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise QGDError(-4, "load", f"{LIB_PATH} is missing; run `python -m quantized_gemm_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "quant_act_per_token": [P, I, I, I, P, P, P],
            "quant_act_group128": [P, I, I, P, P, P],
            "quant_act_per_token_strided": [P, I, I, I, I, P, P, P],
            "quant_act_group128_strided": [P, I, I, I, P, P, P],
            "quant_weight_block128": [P, I, I, P, P, P],
            "qlinear_fp8_dynamic": [P, P, P, P, P, I, I, I, P, S, P],
            "qlinear_w8a8_int8": [P, P, P, P, P, I, I, I, P, S, P],
            "qlinear_block_fp8": [P, P, P, P, P, I, I, I, P, S, P],
            "qgd_w8a8_int8_acc32": [P, P, P, I, I, I, P, S, P],
            "qlinear_fp8_dynamic_noalloc": [P, P, P, P, P, I, I, I, P],
            "qgd_load_dispatch_table": [ctypes.c_char_p],
            "qgd_clear_dispatch_table": [],
            "qgd_set_override": [I, I, I, I, I, I, I, I, I],
            "qgd_get_plan": [I, I, I, I, ctypes.POINTER(_Plan)],
            "qgd_device_error": [ctypes.POINTER(ctypes.c_uint)],
            "qgd_clear_device_error": [],
            "qgd_mma_peak_probe": [I, I, ctypes.POINTER(ctypes.c_double), P],
            "qgd_mma_ring_probe": [I, I, I, I, ctypes.POINTER(ctypes.c_double), P],
            "qgd_test_withhold_accumulator": [I],
            "qgd_set_pdl": [I],
            "qlinear_fp8_dynamic_bf16": [P, I, P, P, P, I, I, I, P, S, P],
            "qlinear_w8a8_int8_bf16": [P, I, P, P, P, I, I, I, P, S, P],
            "qlinear_block_fp8_bf16": [P, I, P, P, P, I, I, I, P, S, P],
            "qgd_get_layer_plan": [I, I, I, I, ctypes.POINTER(_Plan)],
            "qgd_set_fused_override": [I, I],
            "qgd_test_capture_fused": [P, P],
            "quant_act_mx": [P, I, I, I, P, P, P],
            "qlinear_mxfp8": [P, P, P, P, P, I, I, I, P, S, P],
            "qlinear_mxfp8_bf16": [P, I, P, P, P, I, I, I, P, S, P],
            "quant_nvfp4": [P, I, I, I, P, P, P, P],
            "qlinear_nvfp4": [P, P, P, P, P, P, P, I, I, I, P, S, P],
            "qlinear_nvfp4_bf16": [P, I, P, P, P, P, I, I, I, P, S, P],
            "qlinear_tp_bf16": [I, P, I, P, P, P, I, I, I, ctypes.POINTER(_Tp), P, S, P],
            "qgd_tp_wait": [P, I, P],
            "qgd_ipc_malloc": [S, ctypes.POINTER(ctypes.c_void_p), P],
            "qgd_ipc_open": [P, ctypes.POINTER(ctypes.c_void_p)],
            "qgd_ipc_close": [P],
            "qgd_ipc_free": [P],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.qgd_workspace_size.argtypes = [I, I, I, I]
        L.qgd_workspace_size.restype = S
        L.qgd_layer_workspace_size.argtypes = [I, I, I, I]
        L.qgd_layer_workspace_size.restype = S
        L.qgd_tp_workspace_size.argtypes = [I, I, I, I]
        L.qgd_tp_workspace_size.restype = S
        L.qgd_m_bucket.argtypes = [I]
        L.qgd_m_bucket.restype = I
        L.qgd_status_string.argtypes = [I]
        L.qgd_status_string.restype = ctypes.c_char_p
        L.qgd_last_error_message.argtypes = []
        L.qgd_last_error_message.restype = ctypes.c_char_p
        L.qgd_version.argtypes = []
        L.qgd_version.restype = ctypes.c_char_p
        _lib = L
        if os.path.exists(DEFAULT_TABLE) and not os.environ.get("QGD_NO_TABLE"):
            _check(L.qgd_load_dispatch_table(os.environ.get("QGD_TABLE", DEFAULT_TABLE).encode()),
                   "qgd_load_dispatch_table")
        return L


def _check(status: int, where: str) -> None:
    if status != 0:
        L = _lib
        msg = L.qgd_last_error_message().decode() if L is not None else ""
        raise QGDError(status, where, msg or (L.qgd_status_string(status).decode() if L else "error"))


def _ptr(t) -> ctypes.c_void_p | None:
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda_2d(t: torch.Tensor, name: str, dtypes) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")


_BYTE_TYPES = (torch.uint8, torch.int8, torch.float8_e4m3fn)


# ---------------------------------------------------------------------------
# Quantizers
# ---------------------------------------------------------------------------
def _activation_rows(x: torch.Tensor) -> int:
    """Row stride (elements) of a bf16 activation: dense rows, or a view of
    the first K columns of a wider matrix (unit column stride)."""
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    if x.stride(1) != 1 or (x.shape[0] > 1 and x.stride(0) < x.shape[1]):
        raise ValueError("x rows must be contiguous (unit column stride, row stride >= K)")
    return x.stride(0) if x.shape[0] > 1 else x.shape[1]


def quant_act_per_token(x: torch.Tensor, qtype: int = QTYPE_E4M3, xq=None, sx=None, stream=None):
    """Per-row dynamic quantization: x bf16 [M, K] -> (xq [M, K], sx fp32 [M]).
    x may be a column slice of a wider matrix (rows any stride apart)."""
    ldx = _activation_rows(x)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.float8_e4m3fn if qtype == QTYPE_E4M3 else torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().quant_act_per_token_strided(_ptr(x), M, K, ldx, qtype, _ptr(xq), _ptr(sx), _stream(stream)),
           "quant_act_per_token")
    return xq, sx


def quant_act_per_token_strided(x: torch.Tensor, qtype: int = QTYPE_E4M3, xq=None, sx=None, stream=None):
    """Alias of quant_act_per_token, which already takes column slices."""
    return quant_act_per_token(x, qtype, xq=xq, sx=sx, stream=stream)


def quant_act_group128_strided(x: torch.Tensor, xq=None, sx=None, stream=None):
    """Alias of quant_act_group128, which already takes column slices."""
    return quant_act_group128(x, xq=xq, sx=sx, stream=stream)


def quant_weight_per_channel(w: torch.Tensor, qtype: int = QTYPE_E4M3, stream=None):
    """Per-output-channel weight quantization (the per-row quantizer over N rows)."""
    return quant_act_per_token(w, qtype, stream=stream)


def quant_act_group128(x: torch.Tensor, xq=None, sx=None, stream=None):
    """1x128 group quantization: x bf16 [M, K] -> (xq e4m3 [M, K], sx fp32 [M, K/128]).
    x may be a column slice of a wider matrix (rows any stride apart)."""
    ldx = _activation_rows(x)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if sx is None:
        sx = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check(lib().quant_act_group128_strided(_ptr(x), M, K, ldx, _ptr(xq), _ptr(sx), _stream(stream)),
           "quant_act_group128")
    return xq, sx


def quant_mx(x: torch.Tensor, xq=None, sx=None, stream=None):
    """MXFP8 quantization (OCP MX v1.0): x bf16 [R, K] -> (e4m3 codes [R, K],
    E8M0 scale bytes uint8 [R, K/32]).  Activations and weights alike; x may
    be a column slice of a wider matrix."""
    ldx = _activation_rows(x)
    R, K = x.shape
    if xq is None:
        xq = torch.empty((R, K), dtype=torch.float8_e4m3fn, device=x.device)
    if sx is None:
        sx = torch.empty((R, K // 32), dtype=torch.uint8, device=x.device)
    _check(lib().quant_act_mx(_ptr(x), R, K, ldx, _ptr(xq), _ptr(sx), _stream(stream)), "quant_act_mx")
    return xq, sx


def quant_nv(x: torch.Tensor, q=None, s=None, g=None, stream=None):
    """NVFP4 quantization: x bf16 [R, K] (K % 16 == 0) -> (packed E2M1 codes
    uint8 [R, K/2], two per byte with value 2i in the low nibble; E4M3 block
    scales uint8 [R, K/16], one per 16 values; fp32 row scales [R]).
    Activations and weights alike; x may be a column slice of a wider matrix."""
    ldx = _activation_rows(x)
    R, K = x.shape
    if q is None:
        q = torch.empty((R, K // 2), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty((R, K // 16), dtype=torch.uint8, device=x.device)
    if g is None:
        g = torch.empty((R,), dtype=torch.float32, device=x.device)
    for t, name, shape, dt in ((q, "q", (R, K // 2), torch.uint8), (s, "s", (R, K // 16), torch.uint8),
                               (g, "g", (R,), torch.float32)):
        if not isinstance(t, torch.Tensor) or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() \
                or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor of shape {shape}")
    _check(lib().quant_nvfp4(_ptr(x), R, K, ldx, _ptr(q), _ptr(s), _ptr(g), _stream(stream)), "quant_nvfp4")
    return q, s, g


def _check_nv(q, s, g, rows, K, name):
    for t, nm, shape, dt in ((q, name + "q", (rows, K // 2), torch.uint8), (s, "s" + name, (rows, K // 16), torch.uint8),
                             (g, "g" + name, (rows,), torch.float32)):
        if not isinstance(t, torch.Tensor) or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() \
                or not t.is_cuda:
            raise ValueError(f"{nm} must be a contiguous CUDA {dt} tensor of shape {shape}")


def quant_weight_block128(w: torch.Tensor, wq=None, sw=None, stream=None):
    """128x128 block quantization: w bf16 [N, K] -> (wq e4m3 [N, K], sw fp32 [N/128, K/128])."""
    _cuda_2d(w, "w", (torch.bfloat16,))
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if sw is None:
        sw = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    _check(lib().quant_weight_block128(_ptr(w), N, K, _ptr(wq), _ptr(sw), _stream(stream)), "quant_weight_block128")
    return wq, sw


# ---------------------------------------------------------------------------
# Workspace
# ---------------------------------------------------------------------------
class Workspace:
    """A zero-filled device buffer for Split-K partials and tile counters.

    The kernels leave its counters zero after every call, so it is zeroed only
    when it is (re)allocated.  Not to be shared by calls running concurrently.
    """

    def __init__(self, nbytes: int = 0, device=None):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def ensure(self, nbytes: int) -> "Workspace":
        if nbytes > self.nbytes:
            self.buf = torch.zeros(int(nbytes), dtype=torch.uint8, device=self.device)
        return self


_default_ws: dict = {}


def _workspace(fmt: int, M: int, N: int, K: int, ws, device):
    need = qgd_workspace_size(fmt, M, N, K)
    if ws is None:
        key = (device.index if device.index is not None else torch.cuda.current_device())
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(need, device)
    if isinstance(ws, Workspace):
        ws.ensure(need)
        return ws.buf.data_ptr(), ws.nbytes
    return ws.data_ptr(), ws.numel() * ws.element_size()


# ---------------------------------------------------------------------------
# GEMMs
# ---------------------------------------------------------------------------
def _check_operands(fmt: int, xq, sx, wq, sw, y) -> tuple:
    """Shapes, dtypes and placement of a GEMM's operands, checked before
    anything reaches the library (which sees only pointers and sizes).
    Returns (M, N, K)."""
    for t, name in ((xq, "xq"), (wq, "wq")):
        if not isinstance(t, torch.Tensor) or t.dim() != 2:
            raise ValueError(f"{name} must be a 2-D tensor")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"K mismatch: xq {tuple(xq.shape)} vs wq {tuple(wq.shape)}")
    want_x = (torch.int8,) if fmt == FMT_W8A8_INT8 else (torch.uint8, torch.float8_e4m3fn)
    for t, name in ((xq, "xq"), (wq, "wq")):
        if t.dtype not in want_x:
            raise ValueError(f"{name} has dtype {t.dtype}, expected one of {want_x}")
    if fmt == FMT_BLOCK_FP8:
        sx_shape, sw_shape = (M, K // 128), (N // 128, K // 128)
    else:
        sx_shape, sw_shape = (M,), (N,)
    for t, name, shape in ((sx, "sx", sx_shape), (sw, "sw", sw_shape)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 tensor")
        if t.numel() < math.prod(shape):
            raise ValueError(f"{name} holds {t.numel()} scales, {shape} = {math.prod(shape)} needed")
    if y is not None:
        if not isinstance(y, torch.Tensor) or y.dtype != torch.bfloat16 or tuple(y.shape) != (M, N) \
                or not y.is_contiguous():
            raise ValueError(f"y must be a contiguous bfloat16 tensor of shape {(M, N)}")
    for t, name in ((xq, "xq"), (wq, "wq"), (sx, "sx"), (sw, "sw"), (y, "y")):
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    _cuda_2d(xq, "xq", _BYTE_TYPES)
    _cuda_2d(wq, "wq", _BYTE_TYPES)
    return M, N, K


def _qlinear(fn_name: str, fmt: int, xq, sx, wq, sw, y, ws, stream):
    M, N, K = _check_operands(fmt, xq, sx, wq, sw, y)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    wsp, wsn = _workspace(fmt, M, N, K, ws, xq.device)
    fn = getattr(lib(), fn_name)
    _check(fn(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(y), M, N, K, ctypes.c_void_p(wsp), wsn, _stream(stream)),
           fn_name)
    return y


def qlinear_fp8_dynamic(xq, sx, wq, sw, y=None, ws=None, stream=None):
    """Y bf16 [M, N] = (Xq . Wq^T) * sx[m] * sw[n], e4m3 operands."""
    return _qlinear("qlinear_fp8_dynamic", FMT_FP8_DYNAMIC, xq, sx, wq, sw, y, ws, stream)


def qlinear_w8a8_int8(xq, sx, wq, sw, y=None, ws=None, stream=None):
    """Y bf16 [M, N] = (Xq . Wq^T) * sx[m] * sw[n], int8 operands, int32 accumulation."""
    return _qlinear("qlinear_w8a8_int8", FMT_W8A8_INT8, xq, sx, wq, sw, y, ws, stream)


def qlinear_block_fp8(xq, sx, wq, sw, y=None, ws=None, stream=None):
    """Y bf16 [M, N] with 1x128 activation and 128x128 weight block scales."""
    return _qlinear("qlinear_block_fp8", FMT_BLOCK_FP8, xq, sx, wq, sw, y, ws, stream)


_LAYER_FN = {FMT_FP8_DYNAMIC: "qlinear_fp8_dynamic_bf16", FMT_W8A8_INT8: "qlinear_w8a8_int8_bf16",
             FMT_BLOCK_FP8: "qlinear_block_fp8_bf16", FMT_MXFP8: "qlinear_mxfp8_bf16"}


def qlinear_bf16(fmt: int, x: torch.Tensor, wq, sw, y=None, ws=None, stream=None):
    """Layer call from bf16 activations: dynamic quantization and the GEMM,
    fused into one kernel when the layer plan says so (qgd_get_layer_plan).
    x [M, K] bf16 may be a column slice of a wider matrix."""
    ldx = _activation_rows(x)
    M, K = x.shape
    want_w = (torch.int8,) if fmt == FMT_W8A8_INT8 else (torch.uint8, torch.float8_e4m3fn)
    if not isinstance(wq, torch.Tensor) or wq.dim() != 2 or wq.shape[1] != K or wq.dtype not in want_w:
        raise ValueError(f"wq must be a 2-D {want_w} tensor with K={K} columns")
    N = wq.shape[0]
    sw_n = (N // 128) * (K // 128) if fmt == FMT_BLOCK_FP8 else (N * (K // 32) if fmt == FMT_MXFP8 else N)
    sw_t = torch.uint8 if fmt == FMT_MXFP8 else torch.float32
    if not isinstance(sw, torch.Tensor) or sw.dtype != sw_t or sw.numel() < sw_n or not sw.is_contiguous():
        raise ValueError(f"sw must be a contiguous {sw_t} tensor of at least {sw_n} scales")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif y.dtype != torch.bfloat16 or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous bfloat16 tensor of shape {(M, N)}")
    for t, name in ((wq, "wq"), (sw, "sw"), (y, "y")):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    need = qgd_layer_workspace_size(fmt, M, N, K)
    if ws is None:
        key = (x.device.index if x.device.index is not None else torch.cuda.current_device())
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(need, x.device)
    if isinstance(ws, Workspace):
        ws.ensure(need)
        wsp, wsn = ws.buf.data_ptr(), ws.nbytes
    else:
        wsp, wsn = ws.data_ptr(), ws.numel() * ws.element_size()
    fn = _LAYER_FN[fmt]
    _check(getattr(lib(), fn)(_ptr(x), ldx, _ptr(wq), _ptr(sw), _ptr(y), M, N, K, ctypes.c_void_p(wsp), wsn,
                              _stream(stream)), fn)
    return y


def qlinear_mxfp8(xq, sx, wq, sw, y=None, ws=None, stream=None):
    """Y bf16 [M, N] from MXFP8 operands: e4m3 codes with E8M0 block scales
    (uint8 [M, K/32] and [N, K/32]), scaled by the tensor core."""
    for t, name in ((xq, "xq"), (wq, "wq")):
        if not isinstance(t, torch.Tensor) or t.dim() != 2 or t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise ValueError(f"{name} must be a 2-D e4m3 tensor")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"K mismatch: xq {tuple(xq.shape)} vs wq {tuple(wq.shape)}")
    for t, name, rows in ((sx, "sx", M), (sw, "sw", N)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or tuple(t.shape) != (rows, K // 32) \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous uint8 tensor of shape {(rows, K // 32)}")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    elif y.dtype != torch.bfloat16 or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous bfloat16 tensor of shape {(M, N)}")
    for t, name in ((xq, "xq"), (wq, "wq"), (sx, "sx"), (sw, "sw"), (y, "y")):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    wsp, wsn = _workspace(FMT_MXFP8, M, N, K, ws, xq.device)
    _check(lib().qlinear_mxfp8(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(y), M, N, K, ctypes.c_void_p(wsp), wsn,
                               _stream(stream)), "qlinear_mxfp8")
    return y


def qlinear_nvfp4(xq, sx, gx, wq, sw, gw, y=None, ws=None, stream=None):
    """Y bf16 [M, N] from NVFP4 operands (quant_nv's outputs for X and W):
    packed E2M1 codes, E4M3 block scales applied by the tensor core, fp32 row
    scales applied in the epilogue."""
    if not isinstance(xq, torch.Tensor) or xq.dim() != 2 or not isinstance(wq, torch.Tensor) or wq.dim() != 2:
        raise ValueError("xq and wq must be 2-D packed uint8 tensors")
    M, K = xq.shape[0], 2 * xq.shape[1]
    N = wq.shape[0]
    if 2 * wq.shape[1] != K:
        raise ValueError(f"K mismatch: xq {tuple(xq.shape)} vs wq {tuple(wq.shape)} (two values per byte)")
    _check_nv(xq, sx, gx, M, K, "x")
    _check_nv(wq, sw, gw, N, K, "w")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    elif not isinstance(y, torch.Tensor) or y.dtype != torch.bfloat16 or tuple(y.shape) != (M, N) \
            or not y.is_contiguous() or not y.is_cuda:
        raise ValueError(f"y must be a contiguous CUDA bfloat16 tensor of shape {(M, N)}")
    wsp, wsn = _workspace(FMT_NVFP4, M, N, K, ws, xq.device)
    _check(lib().qlinear_nvfp4(_ptr(xq), _ptr(sx), _ptr(gx), _ptr(wq), _ptr(sw), _ptr(gw), _ptr(y), M, N, K,
                               ctypes.c_void_p(wsp), wsn, _stream(stream)), "qlinear_nvfp4")
    return y


def qlinear_nvfp4_bf16(x: torch.Tensor, wq, sw, gw, y=None, ws=None, stream=None):
    """NVFP4 layer call: x bf16 [M, K] quantized into the workspace, then the
    GEMM against quant_nv's weight outputs (wq, sw, gw)."""
    ldx = _activation_rows(x)
    M, K = x.shape
    if not isinstance(wq, torch.Tensor) or wq.dim() != 2:
        raise ValueError("wq must be a 2-D packed uint8 tensor")
    N = wq.shape[0]
    _check_nv(wq, sw, gw, N, K, "w")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif not isinstance(y, torch.Tensor) or y.dtype != torch.bfloat16 or tuple(y.shape) != (M, N) \
            or not y.is_contiguous() or not y.is_cuda:
        raise ValueError(f"y must be a contiguous CUDA bfloat16 tensor of shape {(M, N)}")
    need = qgd_layer_workspace_size(FMT_NVFP4, M, N, K)
    if ws is None:
        key = (x.device.index if x.device.index is not None else torch.cuda.current_device())
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(need, x.device)
    if isinstance(ws, Workspace):
        ws.ensure(need)
        wsp, wsn = ws.buf.data_ptr(), ws.nbytes
    else:
        wsp, wsn = ws.data_ptr(), ws.numel() * ws.element_size()
    _check(lib().qlinear_nvfp4_bf16(_ptr(x), ldx, _ptr(wq), _ptr(sw), _ptr(gw), _ptr(y), M, N, K,
                                    ctypes.c_void_p(wsp), wsn, _stream(stream)), "qlinear_nvfp4_bf16")
    return y


# ---------------------------------------------------------------------------
# Column-parallel layer call (all-gather fused into the output stores)
# ---------------------------------------------------------------------------
def _layer_weight_operands(fmt: int, wq, sw, sw_block, K: int) -> int:
    """Check a layer call's weight operands for format fmt; returns N."""
    if not isinstance(wq, torch.Tensor) or wq.dim() != 2 or not wq.is_cuda or not wq.is_contiguous():
        raise ValueError("wq must be a contiguous 2-D CUDA tensor")
    N = wq.shape[0]
    if fmt == FMT_NVFP4:
        _check_nv(wq, sw_block, sw, N, K, "w")
        return N
    if sw_block is not None:
        raise ValueError("sw_block is for NVFP4 weights only")
    want_w = (torch.int8,) if fmt == FMT_W8A8_INT8 else (torch.uint8, torch.float8_e4m3fn)
    if wq.shape[1] != K or wq.dtype not in want_w:
        raise ValueError(f"wq must be a {want_w} tensor with K={K} columns")
    sw_n = (N // 128) * (K // 128) if fmt == FMT_BLOCK_FP8 else (N * (K // 32) if fmt == FMT_MXFP8 else N)
    sw_t = torch.uint8 if fmt == FMT_MXFP8 else torch.float32
    if not isinstance(sw, torch.Tensor) or sw.dtype != sw_t or sw.numel() < sw_n or not sw.is_contiguous() \
            or not sw.is_cuda:
        raise ValueError(f"sw must be a contiguous CUDA {sw_t} tensor of at least {sw_n} scales")
    return N


def qgd_tp_workspace_size(fmt: int, M: int, N: int, K: int) -> int:
    return int(lib().qgd_tp_workspace_size(fmt, M, N, K))


def qlinear_tp_bf16(fmt: int, x: torch.Tensor, wq, sw, sw_block, *, ranks: int, rank: int, col0: int, ldy: int,
                    ys, flags, ws, stream=None) -> None:
    """Column-parallel layer call: this rank's weight shard (wq [N, K] with
    its scales; NVFP4: sw = fp32 row scales, sw_block = E4M3 block scales)
    against the replicated bf16 activations x [M, K].  Every finished output
    element goes to columns [col0, col0 + N) of all ranks' full outputs
    ys[r] (bf16 [>= M, ldy], device pointers or tensors as addressed from this
    process); when the call is done, its new call count (word `ranks` of this
    rank's own flag array, advanced on the device) goes to entry `rank` of
    every rank's flag array flags[r] (ranks + 1 uint32 words each).  Follow
    with qgd_tp_wait on this rank's own flags before reading its full output."""
    ldx = _activation_rows(x)
    M, K = x.shape
    N = _layer_weight_operands(fmt, wq, sw, sw_block, K)
    if len(ys) != ranks or len(flags) != ranks or not 1 <= ranks <= MAX_TP_RANKS:
        raise ValueError(f"need one output and one flag array per rank (1..{MAX_TP_RANKS} ranks)")
    tp = _Tp()
    tp.ranks, tp.rank, tp.col0, tp.ldy = ranks, rank, col0, ldy
    for r in range(ranks):
        tp.y[r] = _ptr(ys[r]).value
        tp.flags[r] = _ptr(flags[r]).value
    if isinstance(ws, Workspace):
        ws.ensure(qgd_tp_workspace_size(fmt, M, N, K))
        wsp, wsn = ws.buf.data_ptr(), ws.nbytes
    else:
        wsp, wsn = ws.data_ptr(), ws.numel() * ws.element_size()
    _check(lib().qlinear_tp_bf16(fmt, _ptr(x), ldx, _ptr(wq), _ptr(sw), _ptr(sw_block), M, N, K, ctypes.byref(tp),
                                 ctypes.c_void_p(wsp), wsn, _stream(stream)), "qlinear_tp_bf16")


def qgd_tp_wait(flags, ranks: int, stream=None) -> None:
    """Enqueue the wait for every rank's entry in this rank's own flag array
    (a tensor or a device pointer) to reach this rank's call count."""
    _check(lib().qgd_tp_wait(_ptr(flags), ranks, _stream(stream)), "qgd_tp_wait")


def ipc_malloc(nbytes: int) -> tuple:
    """A zero-filled device buffer on the current device that other processes
    can map: returns (device pointer, handle bytes)."""
    ptr = ctypes.c_void_p(0)
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().qgd_ipc_malloc(nbytes, ctypes.byref(ptr), handle), "qgd_ipc_malloc")
    return int(ptr.value), handle.raw


def ipc_open(handle: bytes) -> int:
    """Map another process's buffer from its handle; returns the pointer."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes")
    ptr = ctypes.c_void_p(0)
    _check(lib().qgd_ipc_open(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES), ctypes.byref(ptr)),
           "qgd_ipc_open")
    return int(ptr.value)


def ipc_close(ptr: int) -> None:
    _check(lib().qgd_ipc_close(ctypes.c_void_p(ptr)), "qgd_ipc_close")


def ipc_free(ptr: int) -> None:
    _check(lib().qgd_ipc_free(ctypes.c_void_p(ptr)), "qgd_ipc_free")


class _DeviceArray:
    """__cuda_array_interface__ of a raw device pointer (no ownership)."""

    def __init__(self, ptr: int, shape: tuple, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 2, "strides": None}


_TYPESTR = {torch.bfloat16: ("<i2", torch.int16), torch.int16: ("<i2", torch.int16),
            torch.int32: ("<i4", torch.int32), torch.uint8: ("|u1", torch.uint8)}


def tensor_at(ptr: int, shape: tuple, dtype: torch.dtype, device) -> torch.Tensor:
    """A tensor over device memory this library allocated or mapped (no copy,
    no ownership: the memory must outlive the tensor)."""
    typestr, carrier = _TYPESTR[dtype]
    with torch.cuda.device(device):
        t = torch.as_tensor(_DeviceArray(ptr, shape, typestr), device=device)
    assert t.dtype == carrier and t.data_ptr() == ptr
    return t.view(dtype)


def qlinear_fp8_dynamic_noalloc(xq, sx, wq, sw, y, stream=None):
    """FP8_Dynamic GEMM into a caller-provided y that allocates nothing: no
    workspace argument, no allocation by the binding or the library (the
    library's built-in Split-K scratch is used).  y must be a bf16 [M, N]
    CUDA tensor; every operand is checked before the call."""
    if y is None:
        raise ValueError("qlinear_fp8_dynamic_noalloc writes into a caller-provided y; y is None")
    M, N, K = _check_operands(FMT_FP8_DYNAMIC, xq, sx, wq, sw, y)
    _check(lib().qlinear_fp8_dynamic_noalloc(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(y), M, N, K,
                                             _stream(stream)), "qlinear_fp8_dynamic_noalloc")
    return y


def qgd_w8a8_int8_acc32(xq, wq, acc=None, ws=None, stream=None):
    """Exact int32 accumulator [M, N] of the W8A8_INT8 mainloop (test hook)."""
    _cuda_2d(xq, "xq", (torch.int8,))
    _cuda_2d(wq, "wq", (torch.int8,))
    M, K = xq.shape
    N = wq.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    wsp, wsn = _workspace(FMT_W8A8_INT8, M, N, K, ws, xq.device)
    _check(lib().qgd_w8a8_int8_acc32(_ptr(xq), _ptr(wq), _ptr(acc), M, N, K, ctypes.c_void_p(wsp), wsn,
                                     _stream(stream)), "qgd_w8a8_int8_acc32")
    return acc


# ---------------------------------------------------------------------------
# Dispatch and status (host only)
# ---------------------------------------------------------------------------
def qgd_workspace_size(fmt: int, M: int, N: int, K: int) -> int:
    return int(lib().qgd_workspace_size(fmt, M, N, K))


def qgd_load_dispatch_table(path: str) -> None:
    _check(lib().qgd_load_dispatch_table(str(path).encode()), "qgd_load_dispatch_table")


def qgd_clear_dispatch_table() -> None:
    _check(lib().qgd_clear_dispatch_table(), "qgd_clear_dispatch_table")


def qgd_set_override(fmt: int, variant: int = -1, split_k: int = -1, reduce: int = -1, stages: int = 0,
                     tile_n: int = 0, schedule: int = -1, occupancy: int = 0, k_slices: int = 0) -> None:
    """Force plan fields for one format; every default argument leaves that
    field to the dispatch table / built-in default."""
    _check(lib().qgd_set_override(fmt, variant, split_k, reduce, stages, tile_n, schedule, occupancy, k_slices),
           "qgd_set_override")


def qgd_get_plan(fmt: int, M: int, N: int, K: int) -> dict:
    p = _Plan()
    _check(lib().qgd_get_plan(fmt, M, N, K, ctypes.byref(p)), "qgd_get_plan")
    return {f: getattr(p, f) for f, _ in _Plan._fields_}


def qgd_layer_workspace_size(fmt: int, M: int, N: int, K: int) -> int:
    return int(lib().qgd_layer_workspace_size(fmt, M, N, K))


def qgd_get_layer_plan(fmt: int, M: int, N: int, K: int) -> dict:
    p = _Plan()
    _check(lib().qgd_get_layer_plan(fmt, M, N, K, ctypes.byref(p)), "qgd_get_layer_plan")
    return {f: getattr(p, f) for f, _ in _Plan._fields_}


def qgd_set_fused_override(fmt: int, fused: int = -1) -> None:
    """Force layer plans' `fused` field for one format (-1 = table / default)."""
    _check(lib().qgd_set_fused_override(fmt, fused), "qgd_set_fused_override")


def qgd_test_capture_fused(xq=None, sx=None) -> None:
    """Test hook: fused launches also write their activation codes / scales
    into these device tensors (None, None turns it off)."""
    _check(lib().qgd_test_capture_fused(_ptr(xq), _ptr(sx)), "qgd_test_capture_fused")


def qgd_m_bucket(M: int) -> int:
    return int(lib().qgd_m_bucket(M))


def qgd_device_error() -> int:
    code = ctypes.c_uint(0)
    _check(lib().qgd_device_error(ctypes.byref(code)), "qgd_device_error")
    return int(code.value)


def qgd_clear_device_error() -> None:
    _check(lib().qgd_clear_device_error(), "qgd_clear_device_error")


def qgd_mma_peak_probe(qtype: int = QTYPE_E4M3, iters: int = 4096, stream=None) -> float:
    """Launch the dense tensor-core peak probe on `stream` (one CTA per SM,
    back-to-back tcgen05.mma from shared memory) and return its FLOP count;
    the caller times the launch."""
    flops = ctypes.c_double(0.0)
    _check(lib().qgd_mma_peak_probe(qtype, iters, ctypes.byref(flops), _stream(stream)), "qgd_mma_peak_probe")
    return float(flops.value)


def qgd_mma_ring_probe(n: int = 256, slots: int = 2, wait: bool = True, iters: int = 4096, stream=None) -> float:
    """Launch the accumulator-ring probe on `stream` (groups of four e4m3
    tcgen05.mma of 128 x n x 32 into `slots` TMEM slots in turn, waiting for a
    slot's previous group before reusing it when `wait`) and return its FLOP
    count; the caller times the launch."""
    flops = ctypes.c_double(0.0)
    _check(lib().qgd_mma_ring_probe(n, slots, 1 if wait else 0, iters, ctypes.byref(flops), _stream(stream)),
           "qgd_mma_ring_probe")
    return float(flops.value)


def qgd_set_pdl(on: int = -1) -> None:
    """Programmatic dependent launch on (1), off (0), or as QGD_PDL says (-1)."""
    _check(lib().qgd_set_pdl(on), "qgd_set_pdl")


def qgd_test_withhold_accumulator(on: bool) -> None:
    """Failure-detection test hook: while on, Swap-AB GEMMs never signal a
    finished accumulator, so their epilogue's bounded wait runs out."""
    _check(lib().qgd_test_withhold_accumulator(1 if on else 0), "qgd_test_withhold_accumulator")


def qgd_version() -> str:
    return lib().qgd_version().decode()
