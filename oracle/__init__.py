"""CPU oracle for the W4A8 per-channel quantized linear layer (test infrastructure).

TEST INFRASTRUCTURE ONLY: the test-suite, the package smoke check and the
benchmark's CPU-baseline leg are the only users. The CUDA product path never
imports this package, and this package never imports the product.

The arithmetic lives in plain C (``w4a8_oracle.c``, built with gcc at
``-O2 -ffp-contract=off -fno-fast-math``); this module only marshals numpy
arrays into it. Method: Keras guide "INT4 quantization in Keras", section
"How it works", steps 1-6 (see the C file's header for the readings of the
constants the page leaves open).

Parity of the page's absolute minimal-model MSE value is unpinned: the page
draws its data and weights from an unseeded generator and Keras' own
initialiser, so only its order of magnitude can be checked.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None

OK, BAD_ARG, OVERFLOW = 0, 1, 2


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            for name, args in {
                "oracle_weight_scales": [P, I, I, I, P],
                "oracle_w4_quantize_pack": [P, I, I, I, P, I, P],
                "oracle_w4_unpack": [P, I, I, I, P],
                "oracle_w4_pack": [P, I, I, P, I],
                "oracle_w4_quantize": [P, I, I, I, P, P],
                "oracle_a8_quantize_rows": [P, I, I, I, P, I, P],
                "oracle_gemm_s32": [P, I, I, I, P, I, I, P, I],
                "oracle_dequant": [P, I, I, I, P, P, P, I, P, I],
                "oracle_f32_to_bf16_array": [P, ctypes.c_size_t, P],
                "oracle_quantize_weight": [ctypes.c_float, ctypes.c_float],
                "oracle_w8_quantize": [P, I, I, I, P, I, P],
                "oracle_gemm8_s32": [P, I, I, I, P, I, I, P, I],
                "oracle_w4z_quantize_pack": [P, I, I, I, P, I, P, P],
                "oracle_gemm_z_s32": [P, I, I, I, P, I, I, P, P, I],
                "oracle_w4g_quantize_pack": [P, I, I, I, I, P, I, P, P],
                "oracle_linear_g_q": [P, P, I, I, I, P, I, I, I, P, P, P, I, P, P, I],
            }.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = I
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc == OVERFLOW:
        raise OracleError(f"{what}: INT32 accumulator overflow")
    if rc != OK:
        raise OracleError(f"{what}: invalid argument (rc={rc})")


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def packed_ld(k: int) -> int:
    """Bytes per packed output-channel row: ceil(K/2) rounded up to 16."""
    return ((k + 1) // 2 + 15) // 16 * 16


def weight_scales(w: np.ndarray) -> np.ndarray:
    w = _f32(w)
    k, n = w.shape
    sw = np.empty(n, np.float32)
    _check(_load().oracle_weight_scales(_ptr(w), k, n, n, _ptr(sw)), "weight_scales")
    return sw


def quantize_weight(w: float, sw: float) -> int:
    return int(_load().oracle_quantize_weight(ctypes.c_float(w), ctypes.c_float(sw)))


def w4_quantize_pack(w: np.ndarray, ldp: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """W[K][N] float32 -> (Wp[N][ldp] uint8, sw[N] float32)."""
    w = _f32(w)
    k, n = w.shape
    ldp = packed_ld(k) if ldp is None else ldp
    wp = np.empty((n, ldp), np.uint8)
    sw = np.empty(n, np.float32)
    _check(_load().oracle_w4_quantize_pack(_ptr(w), k, n, n, _ptr(wp), ldp, _ptr(sw)),
           "w4_quantize_pack")
    return wp, sw


def w4_quantize(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """W[K][N] float32 -> (Q[N][K] int8 codes, sw[N] float32), before packing."""
    w = _f32(w)
    k, n = w.shape
    q = np.empty((n, k), np.int8)
    sw = np.empty(n, np.float32)
    _check(_load().oracle_w4_quantize(_ptr(w), k, n, n, _ptr(q), _ptr(sw)), "w4_quantize")
    return q, sw


def w4_pack(q: np.ndarray, ldp: int | None = None) -> np.ndarray:
    """Q[N][K] int8 codes in [-8, 7] -> Wp[N][ldp] uint8."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    n, k = q.shape
    ldp = packed_ld(k) if ldp is None else ldp
    wp = np.empty((n, ldp), np.uint8)
    _check(_load().oracle_w4_pack(_ptr(q), k, n, _ptr(wp), ldp), "w4_pack")
    return wp


def w4_unpack(wp: np.ndarray, k: int) -> np.ndarray:
    """Wp[N][ldp] -> Q[N][K] int8 (sign-extended nibbles)."""
    wp = np.ascontiguousarray(wp, dtype=np.uint8)
    n, ldp = wp.shape
    q = np.empty((n, k), np.int8)
    _check(_load().oracle_w4_unpack(_ptr(wp), k, n, ldp, _ptr(q)), "w4_unpack")
    return q


def a8_quantize_rows(x: np.ndarray, ldq: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """X[M][K] float32 -> (Xq[M][ldq] int8, sx[M] float32)."""
    x = _f32(x)
    m, k = x.shape
    ldq = k if ldq is None else ldq
    xq = np.empty((m, ldq), np.int8)
    sx = np.empty(m, np.float32)
    _check(_load().oracle_a8_quantize_rows(_ptr(x), m, k, k, _ptr(xq), ldq, _ptr(sx)),
           "a8_quantize_rows")
    return xq, sx


def gemm_s32(xq: np.ndarray, k: int, wp: np.ndarray) -> np.ndarray:
    """acc[M][N] = sum_k xq[m][k] * q[n][k] (exact, must fit INT32)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wp = np.ascontiguousarray(wp, dtype=np.uint8)
    m, ldq = xq.shape
    n, ldp = wp.shape
    acc = np.empty((m, n), np.int32)
    _check(_load().oracle_gemm_s32(_ptr(xq), m, k, ldq, _ptr(wp), n, ldp, _ptr(acc), n),
           "gemm_s32")
    return acc


def dequant(acc: np.ndarray, sx: np.ndarray, sw: np.ndarray,
            bias: np.ndarray | None = None, relu: bool = False) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    m, n = acc.shape
    sx, sw = _f32(sx), _f32(sw)
    b = None if bias is None else _f32(bias)
    y = np.empty((m, n), np.float32)
    _check(_load().oracle_dequant(_ptr(acc), m, n, n, _ptr(sx), _ptr(sw), _ptr(b),
                                  int(bool(relu)), _ptr(y), n), "dequant")
    return y


def to_bf16_bits(y: np.ndarray) -> np.ndarray:
    y = _f32(y)
    out = np.empty(y.shape, np.uint16)
    _check(_load().oracle_f32_to_bf16_array(_ptr(y), y.size, _ptr(out)), "to_bf16")
    return out


def linear(x: np.ndarray, wp: np.ndarray, sw: np.ndarray, k: int,
           bias: np.ndarray | None = None, relu: bool = False,
           out: str = "f32"):
    """One quantized Dense layer on float32 input: steps 3-6 of the page.

    out = "f32" (float32 Y), "bf16" (uint16 bf16 bits of Y) or "s32" (raw acc).
    """
    xq, sx = a8_quantize_rows(x)
    acc = gemm_s32(xq, k, wp)
    if out == "s32":
        return acc
    y = dequant(acc, sx, sw, bias, relu)
    return to_bf16_bits(y) if out == "bf16" else y


def linear_q(xq: np.ndarray, sx: np.ndarray, wp: np.ndarray, sw: np.ndarray, k: int,
             bias: np.ndarray | None = None, relu: bool = False, out: str = "f32"):
    """Steps 4-6 on already-quantized activations."""
    acc = gemm_s32(xq, k, wp)
    if out == "s32":
        return acc
    y = dequant(acc, sx, sw, bias, relu)
    return to_bf16_bits(y) if out == "bf16" else y


# ----------------------------------------------------------------- W8A8 ---
# The INT8 path that the page presents INT4 as an extension of: the same steps
# with 8-bit weight codes (scale 127 / max|W[:,n]|, range [-127, 127]) stored
# one per byte. Activation quantization and dequantization are steps 3 and 6
# above, unchanged.

def w8_ld(k: int) -> int:
    """Bytes per INT8 weight row: K rounded up to 16."""
    return (k + 15) // 16 * 16


def w8_quantize(w: np.ndarray, ldw8: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """W[K][N] float32 -> (Q8[N][ldw8] int8 codes, pad 0; sw[N] float32)."""
    w = _f32(w)
    k, n = w.shape
    ldw8 = w8_ld(k) if ldw8 is None else ldw8
    q8 = np.empty((n, ldw8), np.int8)
    sw = np.empty(n, np.float32)
    _check(_load().oracle_w8_quantize(_ptr(w), k, n, n, _ptr(q8), ldw8, _ptr(sw)), "w8_quantize")
    return q8, sw


def gemm8_s32(xq: np.ndarray, k: int, q8: np.ndarray) -> np.ndarray:
    """acc[M][N] = sum_k xq[m][k] * q8[n][k] (exact, must fit INT32)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    q8 = np.ascontiguousarray(q8, dtype=np.int8)
    m, ldq = xq.shape
    n, ldw8 = q8.shape
    acc = np.empty((m, n), np.int32)
    _check(_load().oracle_gemm8_s32(_ptr(xq), m, k, ldq, _ptr(q8), n, ldw8, _ptr(acc), n),
           "gemm8_s32")
    return acc


def linear8(x: np.ndarray, q8: np.ndarray, sw: np.ndarray, k: int,
            bias: np.ndarray | None = None, relu: bool = False, out: str = "f32"):
    """One W8A8 Dense layer on float32 input (steps 3, 5, 6)."""
    xq, sx = a8_quantize_rows(x)
    return linear8_q(xq, sx, q8, sw, k, bias=bias, relu=relu, out=out)


def linear8_q(xq: np.ndarray, sx: np.ndarray, q8: np.ndarray, sw: np.ndarray, k: int,
              bias: np.ndarray | None = None, relu: bool = False, out: str = "f32"):
    """W8A8 steps 5-6 on already-quantized activations."""
    acc = gemm8_s32(xq, k, q8)
    if out == "s32":
        return acc
    y = dequant(acc, sx, sw, bias, relu)
    return to_bf16_bits(y) if out == "bf16" else y


# ------------------------------------------------ asymmetric INT4 (zero point) ---
# Uniform asymmetric quantization of the weights per output channel ("INT4"
# concept page, section 4.1; "4-bit Integer Quantization for LLMs" page,
# section "Weight quantization"): multiplier sa = 15 / (max - min), integer
# zero point zp = -rne(min * sa), codes q = clamp(rne(w * sa) + zp, 0, 15)
# packed as unsigned nibbles; activations as in step 3.

def w4z_quantize_pack(w: np.ndarray, ldp: int | None = None):
    """W[K][N] float32 -> (Wp[N][ldp] uint8, sa[N] float32, zp[N] int32)."""
    w = _f32(w)
    k, n = w.shape
    ldp = packed_ld(k) if ldp is None else ldp
    wp = np.empty((n, ldp), np.uint8)
    sa = np.empty(n, np.float32)
    zp = np.empty(n, np.int32)
    _check(_load().oracle_w4z_quantize_pack(_ptr(w), k, n, n, _ptr(wp), ldp, _ptr(sa), _ptr(zp)),
           "w4z_quantize_pack")
    return wp, sa, zp


def gemm_z_s32(xq: np.ndarray, k: int, wp: np.ndarray, zp: np.ndarray) -> np.ndarray:
    """acc[M][N] = sum_k xq[m][k] * (q[n][k] - zp[n]) (exact, must fit INT32)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wp = np.ascontiguousarray(wp, dtype=np.uint8)
    zp = np.ascontiguousarray(zp, dtype=np.int32)
    m, ldq = xq.shape
    n, ldp = wp.shape
    acc = np.empty((m, n), np.int32)
    _check(_load().oracle_gemm_z_s32(_ptr(xq), m, k, ldq, _ptr(wp), n, ldp, _ptr(zp), _ptr(acc), n),
           "gemm_z_s32")
    return acc


def linear_z(x: np.ndarray, wp: np.ndarray, sa: np.ndarray, zp: np.ndarray, k: int,
             bias: np.ndarray | None = None, relu: bool = False, out: str = "f32"):
    """One Dense layer with zero-point INT4 weights on float32 input."""
    xq, sx = a8_quantize_rows(x)
    acc = gemm_z_s32(xq, k, wp, zp)
    if out == "s32":
        return acc
    y = dequant(acc, sx, sa, bias, relu)
    return to_bf16_bits(y) if out == "bf16" else y


# ---------------------------------------------------- group-wise INT4 ---
# "INT4" concept page, section 4.2: every group of G consecutive k of an
# output channel has its own scale and zero point (the zero-point rule above
# per group); partial INT32 sums per group, dequantized per group and summed
# over the groups in float32.

def w4g_quantize_pack(w: np.ndarray, group: int, ldp: int | None = None):
    """W[K][N] float32 -> (Wp[N][ldp] uint8, sa[N][ng] float32, zp[N][ng] int32)."""
    w = _f32(w)
    k, n = w.shape
    ng = -(-k // group)
    ldp = packed_ld(k) if ldp is None else ldp
    wp = np.empty((n, ldp), np.uint8)
    sa = np.empty((n, ng), np.float32)
    zp = np.empty((n, ng), np.int32)
    _check(_load().oracle_w4g_quantize_pack(_ptr(w), k, n, n, group, _ptr(wp), ldp, _ptr(sa), _ptr(zp)),
           "w4g_quantize_pack")
    return wp, sa, zp


def linear_g(x: np.ndarray, wp: np.ndarray, sa: np.ndarray, zp: np.ndarray, k: int, group: int,
             bias: np.ndarray | None = None, relu: bool = False, partials: bool = False):
    """One group-wise INT4 Dense layer on float32 input; with partials=True
    also returns the INT32 partial sums [M][N][ng]."""
    xq, sx = a8_quantize_rows(x)
    m = xq.shape[0]
    n, ldp = wp.shape
    ng = sa.shape[1]
    acc_g = np.empty((m, n, ng), np.int32)
    y = np.empty((m, n), np.float32)
    b = None if bias is None else _f32(bias)
    _check(_load().oracle_linear_g_q(_ptr(xq), _ptr(sx), m, k, xq.shape[1], _ptr(np.ascontiguousarray(wp)), n,
                                     ldp, group, _ptr(_f32(sa)), _ptr(np.ascontiguousarray(zp, np.int32)), _ptr(b),
                                     int(bool(relu)), _ptr(acc_g), _ptr(y), n), "linear_g")
    return (y, acc_g) if partials else y


def mlp(x: np.ndarray, w1, b1, w2, b2) -> np.ndarray:
    """The page's minimal model, quantized: Dense(K->H, ReLU) then Dense(H->1).

    Each layer quantizes its own float32 input dynamically (step 3); the hidden
    activations stay float32 between the layers.
    """
    k1 = w1.shape[0]
    wp1, sw1 = w4_quantize_pack(w1)
    wp2, sw2 = w4_quantize_pack(w2)
    h = linear(x, wp1, sw1, k1, bias=b1, relu=True)
    return linear(h, wp2, sw2, w2.shape[0], bias=b2, relu=False)
