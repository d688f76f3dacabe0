"""Thin ctypes binding over libw4a8.so (the C ABI declared in include/w4a8.h).

Argument marshalling only: torch tensors -> device pointers, strides and the
current CUDA stream. Every step of the layer runs in the library's kernels;
torch only allocates device memory. If the library is missing this module
raises at import time: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a8.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)

RELU = 0x01
OUT_F32, OUT_BF16, OUT_S32 = 0x00, 0x02, 0x04
STATIC_WEIGHTS = 0x08
PATH_AUTO, PATH_GENERIC, PATH_DECODE, PATH_TC = 0x00, 0x10, 0x20, 0x30
PATH_DECODE_RING, PATH_DECODE_REGS, PATH_DECODE_SPLIT = 0x40, 0x50, 0x60
PATH_TC_PAIR = 0x70
MAX_K = 2097152

_OUT = {"f32": OUT_F32, "bf16": OUT_BF16, "s32": OUT_S32}
_OUT_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "s32": torch.int32}
_PATH = {"auto": PATH_AUTO, "generic": PATH_GENERIC, "decode": PATH_DECODE, "tc": PATH_TC,
         "ring": PATH_DECODE_RING, "regs": PATH_DECODE_REGS, "split": PATH_DECODE_SPLIT,
         "tc2": PATH_TC_PAIR}
PATH_NAMES = {v: k for k, v in _PATH.items()}

class Problem(ctypes.Structure):
    """struct w4a8_problem of include/w4a8.h."""
    _fields_ = [("X", ctypes.c_void_p), ("Wp", ctypes.c_void_p), ("sw", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("M", ctypes.c_int),
                ("K", ctypes.c_int), ("ldx", ctypes.c_int), ("ldp", ctypes.c_int), ("N", ctypes.c_int),
                ("ldy", ctypes.c_int)]


# Every symbol include/w4a8.h declares, with its ctypes signature.
_P, _I, _U, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
SIGNATURES = {
    "w4a8_packed_ld": (_I, [_I]),
    "w4a8_act_ld": (_I, [_I]),
    "w4a8_workspace_size": (_S, [_I, _I]),
    "w4_quantize_pack": (_I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    "a8_quantize_rows": (_I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    "w4a8_linear": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _U, _P, _I, _P, _S, _P]),
    "w4a8_linear_q": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _I, _P, _U, _P, _I, _P]),
    "w4a8_linear_noalloc": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _U, _P, _I, _P]),
    "w4a8_noalloc_scratch_bytes": (_S, []),
    "w4a8_amax_parts": (_I, [_I]),
    "w4a8_linear_chain": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _U, _P, _I, _P, _P, _S, _P]),
    "w8a8_ld": (_I, [_I]),
    "w8_quantize": (_I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    "w8a8_linear": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _U, _P, _I, _P, _S, _P]),
    "w8a8_linear_q": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _I, _P, _U, _P, _I, _P]),
    "w4z_quantize_pack": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P]),
    "w4z_workspace_size": (_S, [_I, _I, _I]),
    "w4z_linear": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _I, _P, _U, _P, _I, _P, _S, _P]),
    "w4z_linear_q": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _U, _P, _I, _P, _S, _P]),
    "w4g_groups": (_I, [_I]),
    "w4g_quantize_pack": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P]),
    "w4g_linear": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _I, _P, _U, _P, _I, _P, _S, _P]),
    "w4g_linear_q": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _U, _P, _I, _P]),
    "w4a8_last_path": (_U, []),
    "w4a8_last_launch_count": (_U, []),
    "w4a8_last_kernel": (ctypes.c_char_p, []),
    "w4a8_selftest_timeout": (_I, [ctypes.c_longlong, _P]),
    "w4a8_linear_grouped": (_I, [ctypes.POINTER(Problem), _I, _U, _P]),
    "w4a8_get_device_status": (_I, [_I, _P]),
    "w4a8_status_string": (ctypes.c_char_p, [_I]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libw4a8.so not found at {LIB_PATH}; build it with "
            "`python -m w4a8_quantized_gemm_channel_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class W4A8Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.w4a8_status_string(status).decode()} (status {status})")


def _check(status: int, what: str):
    if status != OK:
        raise W4A8Error(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _rowmajor(t: torch.Tensor, name: str):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    return t.stride(0)


def packed_ld(k: int) -> int:
    return lib.w4a8_packed_ld(k)


def act_ld(k: int) -> int:
    return lib.w4a8_act_ld(k)


def workspace_size(m: int, k: int) -> int:
    return lib.w4a8_workspace_size(m, k)


def flags_for(relu: bool = False, out: str = "f32", path: str = "auto",
              static_weights: bool = False) -> int:
    return (RELU if relu else 0) | _OUT[out] | _PATH[path] | (STATIC_WEIGHTS if static_weights else 0)


def w4_quantize_pack(w: torch.Tensor, wp: torch.Tensor | None = None,
                     sw: torch.Tensor | None = None, stream=None):
    """W[K][N] float32 (CUDA) -> (Wp[N][ldp] uint8, sw[N] float32)."""
    ldw = _rowmajor(w, "W")
    k, n = w.shape
    if wp is None:
        wp = torch.empty((n, packed_ld(k)), dtype=torch.uint8, device=w.device)
    if sw is None:
        sw = torch.empty(n, dtype=torch.float32, device=w.device)
    ldp = _rowmajor(wp, "Wp")
    _check(lib.w4_quantize_pack(_ptr(w), k, n, ldw, _ptr(wp), ldp, _ptr(sw), _stream(stream)),
           "w4_quantize_pack")
    return wp, sw


def a8_quantize_rows(x: torch.Tensor, xq: torch.Tensor | None = None,
                     sx: torch.Tensor | None = None, stream=None):
    """X[M][K] float32 (CUDA) -> (Xq[M][ldq] int8, sx[M] float32)."""
    ldx = _rowmajor(x, "X")
    m, k = x.shape
    if xq is None:
        xq = torch.empty((m, act_ld(k)), dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty(m, dtype=torch.float32, device=x.device)
    ldq = _rowmajor(xq, "Xq")
    _check(lib.a8_quantize_rows(_ptr(x), m, k, ldx, _ptr(xq), ldq, _ptr(sx), _stream(stream)),
           "a8_quantize_rows")
    return xq, sx


def _out_tensor(y, m, n, out, device):
    if y is None:
        y = torch.empty((m, n), dtype=_OUT_DTYPE[out], device=device)
    return y, _rowmajor(y, "Y")


def w4a8_linear(x: torch.Tensor, wp: torch.Tensor, sw: torch.Tensor,
                bias: torch.Tensor | None = None, relu: bool = False, out: str = "f32",
                path: str = "auto", y: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None,
                static_weights: bool = False) -> torch.Tensor:
    """Y[M][N] = dequant(quant8(X) @ unpack(Wp)^T) (+bias, ReLU) for X[M][K] float32.

    static_weights: promise that wp, sw and bias are final and not written by
    work still pending on the stream (W4A8_STATIC_WEIGHTS)."""
    ldx = _rowmajor(x, "X")
    ldp = _rowmajor(wp, "Wp")
    m, k = x.shape
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, x.device)
    need = workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(lib.w4a8_linear(_ptr(x), m, k, ldx, _ptr(wp), ldp, _ptr(sw), n, _ptr(bias),
                           flags_for(relu, out, path, static_weights), _ptr(y), ldy, _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "w4a8_linear")
    return y


def w4a8_linear_q(xq: torch.Tensor, sx: torch.Tensor, k: int, wp: torch.Tensor,
                  sw: torch.Tensor, bias: torch.Tensor | None = None, relu: bool = False,
                  out: str = "f32", path: str = "auto", y: torch.Tensor | None = None,
                  stream=None, static_weights: bool = False) -> torch.Tensor:
    """Y from INT8 activations Xq[M][ldq] (first k bytes of each row) and sx[M]."""
    ldq = _rowmajor(xq, "Xq")
    ldp = _rowmajor(wp, "Wp")
    m = xq.shape[0]
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, xq.device)
    _check(lib.w4a8_linear_q(_ptr(xq), m, k, ldq, _ptr(sx), _ptr(wp), ldp, _ptr(sw), n,
                             _ptr(bias), flags_for(relu, out, path, static_weights), _ptr(y), ldy,
                             _stream(stream)),
           "w4a8_linear_q")
    return y


def amax_parts(n: int) -> int:
    return lib.w4a8_amax_parts(n)


def w4a8_linear_chain(x: torch.Tensor, wp: torch.Tensor, sw: torch.Tensor,
                      x_amax: torch.Tensor | None = None, bias: torch.Tensor | None = None,
                      relu: bool = False, emit_amax: bool = True, path: str = "auto",
                      y: torch.Tensor | None = None, y_amax: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, stream=None,
                      static_weights: bool = False):
    """One chained Dense layer: Y[M][N] float32 as w4a8_linear, taking the
    input's per-row abs-max parts x_amax [M][parts] (or None) and returning
    (Y, y_amax) with y_amax [M][amax_parts(N)] (None if emit_amax is False)."""
    ldx = _rowmajor(x, "X")
    ldp = _rowmajor(wp, "Wp")
    m, k = x.shape
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, "f32", x.device)
    if emit_amax and y_amax is None:
        y_amax = torch.empty((m, amax_parts(n)), dtype=torch.float32, device=x.device)
    if not emit_amax:
        y_amax = None
    x_parts = 0
    if x_amax is not None:
        if x_amax.dim() != 2 or x_amax.shape[0] != m or not x_amax.is_contiguous():
            raise ValueError("x_amax must be a contiguous [M][parts] tensor")
        x_parts = x_amax.shape[1]
    need = workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(lib.w4a8_linear_chain(_ptr(x), m, k, ldx, _ptr(x_amax), x_parts, _ptr(wp), ldp, _ptr(sw), n,
                                 _ptr(bias), flags_for(relu, "f32", path, static_weights), _ptr(y), ldy,
                                 _ptr(y_amax), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream)),
           "w4a8_linear_chain")
    return y, y_amax


def w4a8_linear_grouped(problems, relu: bool = False, out: str = "f32", stream=None,
                        static_weights: bool = False):
    """Many independent few-row linears in as few launches as possible.
    problems: list of (x, wp, sw, bias_or_None) with x [M][K] float32, M <= 4.
    Returns the list of outputs Y [M][N]."""
    arr = (Problem * max(1, len(problems)))()
    ys = []
    for i, (x, wp, sw, bias) in enumerate(problems):
        ldx = _rowmajor(x, "X")
        ldp = _rowmajor(wp, "Wp")
        m, k = x.shape
        n = wp.shape[0]
        y, ldy = _out_tensor(None, m, n, out, x.device)
        ys.append(y)
        arr[i] = Problem(x.data_ptr(), wp.data_ptr(), sw.data_ptr(), None if bias is None else bias.data_ptr(),
                         y.data_ptr(), m, k, ldx, ldp, n, ldy)
    flags = (RELU if relu else 0) | _OUT[out] | (STATIC_WEIGHTS if static_weights else 0)
    _check(lib.w4a8_linear_grouped(arr, len(problems), flags, _stream(stream)), "w4a8_linear_grouped")
    return ys


# the library's own figure, so Python and C cannot drift apart
NOALLOC_SCRATCH_BYTES = lib.w4a8_noalloc_scratch_bytes()


def w4a8_linear_noalloc(x: torch.Tensor, wp: torch.Tensor, sw: torch.Tensor,
                        bias: torch.Tensor | None = None, relu: bool = False, out: str = "f32",
                        path: str = "auto", y: torch.Tensor | None = None,
                        stream=None, static_weights: bool = False) -> torch.Tensor:
    """w4a8_linear without a caller workspace: the INT8 activations live in the
    library's fixed per-device scratch array (see include/w4a8.h)."""
    ldx = _rowmajor(x, "X")
    ldp = _rowmajor(wp, "Wp")
    m, k = x.shape
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, x.device)
    _check(lib.w4a8_linear_noalloc(_ptr(x), m, k, ldx, _ptr(wp), ldp, _ptr(sw), n, _ptr(bias),
                                   flags_for(relu, out, path, static_weights), _ptr(y), ldy,
                                   _stream(stream)),
           "w4a8_linear_noalloc")
    return y


# ------------------------------------------------------------------ W8A8 ---
# The INT8 path the INT4 scheme extends: one INT8 weight code per byte
# (scale 127 / abs-max), the same activation step and epilogue.

def w8a8_ld(k: int) -> int:
    return lib.w8a8_ld(k)


def w8_quantize(w: torch.Tensor, wq: torch.Tensor | None = None,
                sw: torch.Tensor | None = None, stream=None):
    """W[K][N] float32 (CUDA) -> (Wq[N][ldw8] int8, sw[N] float32)."""
    ldw = _rowmajor(w, "W")
    k, n = w.shape
    if wq is None:
        wq = torch.empty((n, w8a8_ld(k)), dtype=torch.int8, device=w.device)
    if sw is None:
        sw = torch.empty(n, dtype=torch.float32, device=w.device)
    ldw8 = _rowmajor(wq, "Wq")
    _check(lib.w8_quantize(_ptr(w), k, n, ldw, _ptr(wq), ldw8, _ptr(sw), _stream(stream)), "w8_quantize")
    return wq, sw


def w8a8_linear(x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                bias: torch.Tensor | None = None, relu: bool = False, out: str = "f32",
                path: str = "auto", y: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None,
                static_weights: bool = False) -> torch.Tensor:
    """Y[M][N] = dequant(quant8(X) @ Wq^T) (+bias, ReLU) for X[M][K] float32."""
    ldx = _rowmajor(x, "X")
    ldw8 = _rowmajor(wq, "Wq")
    m, k = x.shape
    n = wq.shape[0]
    y, ldy = _out_tensor(y, m, n, out, x.device)
    need = workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(lib.w8a8_linear(_ptr(x), m, k, ldx, _ptr(wq), ldw8, _ptr(sw), n, _ptr(bias),
                           flags_for(relu, out, path, static_weights), _ptr(y), ldy, _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "w8a8_linear")
    return y


def w8a8_linear_q(xq: torch.Tensor, sx: torch.Tensor, k: int, wq: torch.Tensor,
                  sw: torch.Tensor, bias: torch.Tensor | None = None, relu: bool = False,
                  out: str = "f32", path: str = "auto", y: torch.Tensor | None = None,
                  stream=None, static_weights: bool = False) -> torch.Tensor:
    """Y from INT8 activations Xq[M][ldq] (first k bytes of each row) and sx[M]."""
    ldq = _rowmajor(xq, "Xq")
    ldw8 = _rowmajor(wq, "Wq")
    m = xq.shape[0]
    n = wq.shape[0]
    y, ldy = _out_tensor(y, m, n, out, xq.device)
    _check(lib.w8a8_linear_q(_ptr(xq), m, k, ldq, _ptr(sx), _ptr(wq), ldw8, _ptr(sw), n,
                             _ptr(bias), flags_for(relu, out, path, static_weights), _ptr(y), ldy,
                             _stream(stream)),
           "w8a8_linear_q")
    return y


# --------------------------------------------------- zero-point INT4 ---
# Asymmetric per-channel INT4 weights (scale 15 / range, integer zero point),
# stored as q - 8 nibbles in the W4A8 packed layout.

def w4z_quantize_pack(w: torch.Tensor, stream=None):
    """W[K][N] float32 (CUDA) -> (Wp[N][ldp] uint8, sa[N] float32, zp[N] int32)."""
    ldw = _rowmajor(w, "W")
    k, n = w.shape
    wp = torch.empty((n, packed_ld(k)), dtype=torch.uint8, device=w.device)
    sa = torch.empty(n, dtype=torch.float32, device=w.device)
    zp = torch.empty(n, dtype=torch.int32, device=w.device)
    _check(lib.w4z_quantize_pack(_ptr(w), k, n, ldw, _ptr(wp), wp.stride(0), _ptr(sa), _ptr(zp),
                                 _stream(stream)), "w4z_quantize_pack")
    return wp, sa, zp


def _zworkspace(workspace, m, k, n, device):
    need = lib.w4z_workspace_size(m, k, n)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def w4z_linear(x: torch.Tensor, wp: torch.Tensor, sa: torch.Tensor, zp: torch.Tensor,
               bias: torch.Tensor | None = None, relu: bool = False, out: str = "f32",
               path: str = "auto", y: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None,
               static_weights: bool = False) -> torch.Tensor:
    """Y[M][N] of the zero-point layer for X[M][K] float32."""
    ldx = _rowmajor(x, "X")
    ldp = _rowmajor(wp, "Wp")
    m, k = x.shape
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, x.device)
    workspace, wsb = _zworkspace(workspace, m, k, n, x.device)
    _check(lib.w4z_linear(_ptr(x), m, k, ldx, _ptr(wp), ldp, _ptr(sa), _ptr(zp), n, _ptr(bias),
                          flags_for(relu, out, path, static_weights), _ptr(y), ldy, _ptr(workspace), wsb,
                          _stream(stream)), "w4z_linear")
    return y


def w4z_linear_q(xq: torch.Tensor, sx: torch.Tensor, k: int, wp: torch.Tensor, sa: torch.Tensor,
                 zp: torch.Tensor, bias: torch.Tensor | None = None, relu: bool = False,
                 out: str = "f32", path: str = "auto", y: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None,
                 static_weights: bool = False) -> torch.Tensor:
    """The zero-point layer on INT8 activations Xq[M][ldq] and sx[M]."""
    ldq = _rowmajor(xq, "Xq")
    ldp = _rowmajor(wp, "Wp")
    m = xq.shape[0]
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, xq.device)
    workspace, wsb = _zworkspace(workspace, m, k, n, xq.device)
    _check(lib.w4z_linear_q(_ptr(xq), m, k, ldq, _ptr(sx), _ptr(wp), ldp, _ptr(sa), _ptr(zp), n, _ptr(bias),
                            flags_for(relu, out, path, static_weights), _ptr(y), ldy, _ptr(workspace), wsb,
                            _stream(stream)), "w4z_linear_q")
    return y


# ---------------------------------------------------- group-wise INT4 ---
# Per (output channel, group of 128 k) scale and zero point; float32 outputs.

def w4g_quantize_pack(w: torch.Tensor, stream=None):
    """W[K][N] float32 (CUDA) -> (Wp[N][ldp] uint8, sa[N][ng] float32, zp[N][ng] int32)."""
    ldw = _rowmajor(w, "W")
    k, n = w.shape
    ng = lib.w4g_groups(k)
    wp = torch.empty((n, packed_ld(k)), dtype=torch.uint8, device=w.device)
    sa = torch.empty((n, ng), dtype=torch.float32, device=w.device)
    zp = torch.empty((n, ng), dtype=torch.int32, device=w.device)
    _check(lib.w4g_quantize_pack(_ptr(w), k, n, ldw, _ptr(wp), wp.stride(0), _ptr(sa), _ptr(zp),
                                 _stream(stream)), "w4g_quantize_pack")
    return wp, sa, zp


def w4g_linear(x: torch.Tensor, wp: torch.Tensor, sa: torch.Tensor, zp: torch.Tensor,
               bias: torch.Tensor | None = None, relu: bool = False, out: str = "f32",
               path: str = "auto", y: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None,
               static_weights: bool = False) -> torch.Tensor:
    """Y[M][N] of the group-wise layer for X[M][K] float32."""
    ldx = _rowmajor(x, "X")
    ldp = _rowmajor(wp, "Wp")
    m, k = x.shape
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, x.device)
    need = workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(lib.w4g_linear(_ptr(x), m, k, ldx, _ptr(wp), ldp, _ptr(sa), _ptr(zp), n, _ptr(bias),
                          flags_for(relu, out, path, static_weights), _ptr(y), ldy, _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream)), "w4g_linear")
    return y


def w4g_linear_q(xq: torch.Tensor, sx: torch.Tensor, k: int, wp: torch.Tensor, sa: torch.Tensor,
                 zp: torch.Tensor, bias: torch.Tensor | None = None, relu: bool = False,
                 out: str = "f32", path: str = "auto", y: torch.Tensor | None = None, stream=None,
                 static_weights: bool = False) -> torch.Tensor:
    """The group-wise layer on INT8 activations Xq[M][ldq] and sx[M]."""
    ldq = _rowmajor(xq, "Xq")
    ldp = _rowmajor(wp, "Wp")
    m = xq.shape[0]
    n = wp.shape[0]
    y, ldy = _out_tensor(y, m, n, out, xq.device)
    _check(lib.w4g_linear_q(_ptr(xq), m, k, ldq, _ptr(sx), _ptr(wp), ldp, _ptr(sa), _ptr(zp), n, _ptr(bias),
                            flags_for(relu, out, path, static_weights), _ptr(y), ldy, _stream(stream)),
           "w4g_linear_q")
    return y


def last_path() -> str:
    return PATH_NAMES.get(lib.w4a8_last_path(), "none")


def last_launch_count() -> int:
    return lib.w4a8_last_launch_count()


def last_kernel() -> str:
    """Name of the product kernel of this thread's last call ("" if none)."""
    return lib.w4a8_last_kernel().decode()


def selftest_timeout(cycles: int = 1_000_000, stream=None):
    """Enqueue the bounded-wait self-test (see include/w4a8.h)."""
    _check(lib.w4a8_selftest_timeout(cycles, _stream(stream)), "w4a8_selftest_timeout")


def get_device_status(clear: bool = False, stream=None) -> int:
    return lib.w4a8_get_device_status(int(clear), _stream(stream))
