"""Scalar CPU oracle for the NVFP4 QAD hot path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check (``__graft_entry__.smoke``) and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``nvfp4_quantization_aware_b200``) never imports it and shares no code with
it: the two meet only in the seeded input generators, which hold none of the
method's arithmetic.

The arithmetic lives in ``nvfp4_oracle.c``; this module marshals numpy arrays
into it.  Every function follows the definitions of the NVFP4 format
(Nemotron-3-Nano-30B NVFP4 article, "NVFP4-Format und warum es wichtig ist?"),
the two scale strategies (Nemotron 3.5 Lightning NVFP4 article, "量化尺度处理策略")
and the KL distillation loss (same article, "QAD的工作原理").

Parity status of each function (what pins it is in the tests under
``tests/test_oracle_*.py``): e2m1/e4m3 encode and decode, bf16 rounding,
quantize, dequantize, fake_quant, swizzled_scale_offset, gemm_w4a4, gemm_w4a16,
kl and calibrate_mse are all pinned; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

DYNAMIC = 0
FROZEN_GLOBAL = 1
FROZEN_ALL = 2

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_i64, c_f, c_d, c_p = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        L.oracle_e2m1_encode.argtypes = [c_f]
        L.oracle_e2m1_encode.restype = ctypes.c_int
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e2m1_value.restype = c_d
        L.oracle_e4m3_encode_nonneg.argtypes = [c_f]
        L.oracle_e4m3_encode_nonneg.restype = ctypes.c_int
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = c_d
        L.oracle_bf16_round.argtypes = [c_d]
        L.oracle_bf16_round.restype = ctypes.c_uint16
        L.oracle_bf16_round_array.argtypes = [c_p, c_i64, c_p]
        L.oracle_bf16_round_array.restype = None
        L.oracle_tensor_amax.argtypes = [c_p, c_i64, c_i64, c_i64]
        L.oracle_tensor_amax.restype = c_f
        L.oracle_global_scale_from_amax.argtypes = [c_f]
        L.oracle_global_scale_from_amax.restype = c_f
        L.oracle_quantize.argtypes = [c_p, c_i64, c_i64, c_i64, ctypes.c_int, c_p, c_p, c_p]
        L.oracle_quantize.restype = ctypes.c_int
        L.oracle_dequantize.argtypes = [c_p, c_p, c_f, c_i64, c_i64, c_p, c_p]
        L.oracle_dequantize.restype = ctypes.c_int
        L.oracle_fake_quant.argtypes = [c_p, c_i64, c_i64, c_i64, ctypes.c_int, c_p, c_p, c_p, c_p, c_p]
        L.oracle_fake_quant.restype = ctypes.c_int
        L.oracle_swizzled_scale_offset.argtypes = [c_i64, c_i64, c_i64]
        L.oracle_swizzled_scale_offset.restype = c_i64
        L.oracle_swizzle_scales.argtypes = [c_p, c_i64, c_i64, c_p]
        L.oracle_swizzle_scales.restype = ctypes.c_int
        L.oracle_gemm_w4a4.argtypes = [c_p, c_p, c_f, c_p, c_p, c_f, c_i64, c_i64, c_i64, c_p]
        L.oracle_gemm_w4a4.restype = ctypes.c_int
        L.oracle_gemm_w4a4_rows.argtypes = [c_p, c_p, c_f, c_p, c_p, c_f, c_i64, c_i64, c_p, c_i64, c_p]
        L.oracle_gemm_w4a4_rows.restype = ctypes.c_int
        L.oracle_calibrate_mse.argtypes = [c_p, c_i64, c_i64, c_i64, c_f, c_p, c_p]
        L.oracle_calibrate_mse.restype = ctypes.c_int
        L.oracle_kl.argtypes = [c_p, c_p, c_i64, c_i64, c_i64, c_d, c_d, c_p, c_p, c_p, c_p, ctypes.c_int]
        L.oracle_kl.restype = ctypes.c_int
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_get_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(st: int, what: str):
    if st != 0:
        raise ValueError(f"oracle {what} failed with status {st}")


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# --------------------------------------------------------------------------
# bf16 <-> float helpers (bit-level, no rounding except bf16_round)
# --------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bf16 (RNE); returns uint16 bit patterns."""
    a = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_bf16_round_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_round_scalar(v: float) -> int:
    return int(lib().oracle_bf16_round(float(v)))


# --------------------------------------------------------------------------
# scalar format functions
# --------------------------------------------------------------------------

def e2m1_encode(v: float) -> int:
    return int(lib().oracle_e2m1_encode(float(v)))


def e2m1_value(code: int) -> float:
    return float(lib().oracle_e2m1_value(int(code)))


def e4m3_encode(t: float) -> int:
    return int(lib().oracle_e4m3_encode_nonneg(float(t)))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e4m3_table() -> np.ndarray:
    """Values of all 256 E4M3 codes (NaN for 0x7F / 0xFF)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def swizzled_scale_offset(r: int, kb: int, cols: int) -> int:
    return int(lib().oracle_swizzled_scale_offset(int(r), int(kb), int(cols)))


def swizzled_scale_bytes(rows: int, cols: int) -> int:
    return ((rows + 127) // 128) * 128 * ((cols // 16 + 3) // 4) * 4


def swizzle_scales(s_b: np.ndarray, cols: int) -> np.ndarray:
    """Scatter row-major block scales [rows, cols/16] into the tensor-core
    layout (oracle_swizzled_scale_offset); padding bytes are 0."""
    s_b = np.ascontiguousarray(s_b, dtype=np.uint8)
    out = np.zeros(swizzled_scale_bytes(s_b.shape[0], cols), dtype=np.uint8)
    _check(lib().oracle_swizzle_scales(_ptr(s_b), s_b.shape[0], cols, _ptr(out)), "swizzle_scales")
    return out


# --------------------------------------------------------------------------
# tensor functions
# --------------------------------------------------------------------------

def tensor_amax(x: np.ndarray) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return float(lib().oracle_tensor_amax(_ptr(x), x.shape[0], x.shape[1], x.shape[1]))


def quantize(x: np.ndarray, mode: int = DYNAMIC, s_g: float | None = None,
             s_b: np.ndarray | None = None):
    """x: float32 [rows, cols] (exact copies of the bf16/f32 input).
    Returns (codes uint8 [rows, cols/2], s_b uint8 [rows, cols/16], s_g float)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    sg = np.array([0.0 if s_g is None else s_g], dtype=np.float32)
    if mode == FROZEN_ALL:
        if s_b is None or s_g is None:
            raise ValueError("FROZEN_ALL needs s_g and s_b")
        sb = np.ascontiguousarray(s_b, dtype=np.uint8).copy()
    else:
        if mode == FROZEN_GLOBAL and s_g is None:
            raise ValueError("FROZEN_GLOBAL needs s_g")
        sb = np.zeros((rows, cols // 16), dtype=np.uint8)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    _check(lib().oracle_quantize(_ptr(x), rows, cols, cols, mode, _ptr(sg), _ptr(sb), _ptr(codes)),
           "quantize")
    return codes, sb, float(sg[0])


def dequantize(codes: np.ndarray, s_b: np.ndarray, s_g: float, cols: int):
    """Returns (float32 [rows, cols], bf16 bits uint16 [rows, cols])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    s_b = np.ascontiguousarray(s_b, dtype=np.uint8)
    rows = codes.shape[0]
    f32 = np.zeros((rows, cols), dtype=np.float32)
    b16 = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().oracle_dequantize(_ptr(codes), _ptr(s_b), float(s_g), rows, cols, _ptr(f32), _ptr(b16)),
           "dequantize")
    return f32, b16


def fake_quant(x: np.ndarray, mode: int = DYNAMIC, s_g: float | None = None,
               s_b: np.ndarray | None = None):
    """Returns (y float32, y bf16 bits, s_b, s_g)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    sg = np.array([0.0 if s_g is None else s_g], dtype=np.float32)
    sb = (np.ascontiguousarray(s_b, dtype=np.uint8).copy() if mode == FROZEN_ALL
          else np.zeros((rows, cols // 16), dtype=np.uint8))
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    f32 = np.zeros((rows, cols), dtype=np.float32)
    b16 = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().oracle_fake_quant(_ptr(x), rows, cols, cols, mode, _ptr(sg), _ptr(sb), _ptr(codes),
                                   _ptr(f32), _ptr(b16)), "fake_quant")
    return f32, b16, sb, float(sg[0])


def calibrate_mse(x: np.ndarray, s_g: float):
    """MSE block-scale calibration with the tensor scale s_g given.
    Returns (s_b uint8 [rows, cols/16], least squared error float32 per block)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    sb = np.zeros((rows, cols // 16), dtype=np.uint8)
    err = np.zeros((rows, cols // 16), dtype=np.float32)
    _check(lib().oracle_calibrate_mse(_ptr(x), rows, cols, cols, float(s_g), _ptr(sb), _ptr(err)), "calibrate_mse")
    return sb, err


def gemm_w4a4(a_codes, a_sb, a_sg, b_codes, b_sb, b_sg, K: int) -> np.ndarray:
    """C = A_hat @ B_hat^T in float64 (A: M x K, B: N x K)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    b_codes = np.ascontiguousarray(b_codes, dtype=np.uint8)
    a_sb = np.ascontiguousarray(a_sb, dtype=np.uint8)
    b_sb = np.ascontiguousarray(b_sb, dtype=np.uint8)
    M, N = a_codes.shape[0], b_codes.shape[0]
    c = np.zeros((M, N), dtype=np.float64)
    _check(lib().oracle_gemm_w4a4(_ptr(a_codes), _ptr(a_sb), float(a_sg), _ptr(b_codes), _ptr(b_sb),
                                  float(b_sg), M, N, K, _ptr(c)), "gemm_w4a4")
    return c


def gemm_w4a16(a: np.ndarray, b_codes, b_sb, b_sg: float, K: int) -> np.ndarray:
    """Weight-only NVFP4 product in float64: C = A @ W_hat^T with A the bf16
    activations (given as their exact float32/float64 values, M x K) and
    W_hat the bf16 dequantized weights (N x K): value(q) * (s_b * s_g) in
    binary32, rounded to bf16 -- the weights a bf16 fake-quant produces
    (Qwen3.6-35B-A3B W4A4 tutorial, section "为什么目标是 W4A4 而不是 W4A16":
    W4A16 multiplies 16-bit activations with weights dequantized to 16 bits)."""
    _, w_bits = dequantize(b_codes, b_sb, b_sg, K)
    w_hat = bf16_bits_to_f32(w_bits).astype(np.float64)
    return np.asarray(a, dtype=np.float64) @ w_hat.T


def gemm_w4a4_rows(a_codes, a_sb, a_sg, b_codes, b_sb, b_sg, K: int, rows) -> np.ndarray:
    """Rows `rows` of A_hat @ B_hat^T in float64."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    b_codes = np.ascontiguousarray(b_codes, dtype=np.uint8)
    a_sb = np.ascontiguousarray(a_sb, dtype=np.uint8)
    b_sb = np.ascontiguousarray(b_sb, dtype=np.uint8)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N = b_codes.shape[0]
    c = np.zeros((rows.shape[0], N), dtype=np.float64)
    _check(lib().oracle_gemm_w4a4_rows(_ptr(a_codes), _ptr(a_sb), float(a_sg), _ptr(b_codes), _ptr(b_sb),
                                       float(b_sg), N, K, _ptr(rows), rows.shape[0], _ptr(c)),
           "gemm_w4a4_rows")
    return c


def kl(teacher: np.ndarray, student: np.ndarray, T: float = 1.0, grad_scale: float | None = None,
       want_grad: bool = True, threads: int | None = None):
    """Forward KL(p_t || p_s) per row in float64.
    Returns (loss, row_kl [rows], grad [rows, V] or None)."""
    t = np.ascontiguousarray(teacher, dtype=np.float64)
    s = np.ascontiguousarray(student, dtype=np.float64)
    rows, V = t.shape
    if grad_scale is None:
        grad_scale = 1.0 / rows if rows else 1.0
    nthr = threads or get_threads()
    work = np.zeros(nthr * 2 * V, dtype=np.float64)
    row_kl = np.zeros(rows, dtype=np.float64)
    loss = np.zeros(1, dtype=np.float64)
    grad = np.zeros((rows, V), dtype=np.float64) if want_grad else None
    _check(lib().oracle_kl(_ptr(t), _ptr(s), rows, V, V, float(T), float(grad_scale), _ptr(row_kl),
                           _ptr(loss), _ptr(grad), _ptr(work), nthr), "kl")
    return float(loss[0]), row_kl, grad
