"""CPU oracle for the NVFP4 W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline /
reference leg may import this package.  The product path (the CUDA library
and its Python binding) never does; the two share no code.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp32 steps written out
one operation at a time, fp64 GEMM); this module only marshals numpy arrays.
It follows the pages on the method:

* NVFP4 = 4-bit E2M1 codes, each group of 16 consecutive codes sharing one
  E4M3 scale
  ("NVFP4 W4A4 quantization compresses 27B hybrid models", thevalue.engineering,
  section "Challenging the Recurrence Fragility Assumption"; "Quantizing All
  Layers Reveals Recurrent Memory Is Robust", freegardner.com, section "Block
  Scaling and the Geography of Outliers").
* W4A4 on every linear layer, one FP32 global scale per calibrated module, and
  the fused-module GEMM whose global-scale mismatch the paper repairs ("Why
  Gated DeltaNet Survives 4-Bit Quantization", kipquest.com, sections "The
  abstract" and "The deep dive").

Readings of what the pages leave open are written in ``nvfp4_oracle.c``'s
header.  Every function here is pinned by ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

E4M3_MAX = 448.0
E2M1_MAX = 6.0
GLOBAL_DIVISOR = 2688.0  # 6 * 448


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, no FMA
    contraction, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        c_i64, c_f, c_d, c_p = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        lib.oracle_e2m1_decode.restype = c_d
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_int]
        lib.oracle_e4m3_decode.restype = c_d
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_int]
        lib.oracle_e2m1_encode.restype = ctypes.c_int
        lib.oracle_e2m1_encode.argtypes = [c_f]
        lib.oracle_e4m3_encode_nonneg.restype = ctypes.c_int
        lib.oracle_e4m3_encode_nonneg.argtypes = [c_f]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_double_to_bf16.argtypes = [c_d]
        lib.oracle_rows_amax.restype = c_f
        lib.oracle_rows_amax.argtypes = [c_p, c_i64, c_i64, c_i64, c_i64]
        lib.oracle_global_scale.restype = c_f
        lib.oracle_global_scale.argtypes = [c_f]
        lib.oracle_quantize_rows.restype = None
        lib.oracle_quantize_rows.argtypes = [c_p, c_i64, c_i64, c_i64, c_p, c_p, c_p]
        lib.oracle_dequant_rows.restype = None
        lib.oracle_dequant_rows.argtypes = [c_p, c_p, c_i64, c_i64, c_p, c_p]
        lib.oracle_sf_offset.restype = c_i64
        lib.oracle_sf_offset.argtypes = [c_i64, c_i64, c_i64]
        lib.oracle_sf_bytes.restype = c_i64
        lib.oracle_sf_bytes.argtypes = [c_i64, c_i64]
        lib.oracle_swizzle_scales.restype = None
        lib.oracle_swizzle_scales.argtypes = [c_p, c_i64, c_i64, c_p]
        lib.oracle_unswizzle_scales.restype = None
        lib.oracle_unswizzle_scales.argtypes = [c_p, c_i64, c_i64, c_p]
        lib.oracle_linear_sampled.restype = None
        lib.oracle_linear_sampled.argtypes = [c_p, c_p, c_f, c_p, c_p, c_p, c_i64, c_p, c_p, c_i64, c_p, c_p]
        lib.oracle_swiglu.restype = None
        lib.oracle_swiglu.argtypes = [c_p, c_i64, c_i64, c_i64, c_p]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [c_f]
        lib.oracle_fp8_kv_scale.restype = c_f
        lib.oracle_fp8_kv_scale.argtypes = [c_f]
        lib.oracle_fp8_kv_quantize.restype = None
        lib.oracle_fp8_kv_quantize.argtypes = [c_p, c_i64, c_i64, c_i64, c_f, c_p, c_i64]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------ formats

def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code."""
    return _L().oracle_e2m1_decode(int(code))


def e4m3_decode(byte: int) -> float:
    """Value of an E4M3 byte (NaN for 0x7F / 0xFF)."""
    return _L().oracle_e4m3_decode(int(byte))


def e2m1_encode(y: float) -> int:
    """E2M1 code of an fp32 value: round to nearest, ties to the even code,
    saturate at +-6, keep the sign of zero."""
    return _L().oracle_e2m1_encode(float(np.float32(y)))


def e4m3_encode(v: float) -> int:
    """E4M3 byte of a non-negative fp32 scale: round to nearest even,
    saturate at 448."""
    return _L().oracle_e4m3_encode_nonneg(float(np.float32(v)))


def e2m1_table() -> np.ndarray:
    return np.array([e2m1_decode(c) for c in range(16)], dtype=np.float64)


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_decode(b) for b in range(256)], dtype=np.float64)


def double_to_bf16(x: float) -> int:
    return int(_L().oracle_double_to_bf16(float(x)))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16/int16) -> float32 values (exact)."""
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# -------------------------------------------------------------- quantization

def amax(x_bits: np.ndarray, r0: int = 0, r1: int | None = None) -> float:
    """max |x| over rows [r0, r1) of a bf16 matrix given as uint16 bits."""
    x = np.ascontiguousarray(x_bits).view(np.uint16)
    rows, K = x.shape
    r1 = rows if r1 is None else r1
    return float(np.float32(_L().oracle_rows_amax(_ptr(x), r0, r1, K, K)))


def global_scale(a: float) -> float:
    """FP32 global scale g = amax / (6 * 448) (1.0 when amax == 0)."""
    return float(np.float32(_L().oracle_global_scale(float(np.float32(a)))))


def quantize(x_bits: np.ndarray, g_row) -> tuple[np.ndarray, np.ndarray]:
    """Block-quantize a bf16 matrix [rows, K] (uint16 bits) with global scale
    g_row (scalar or one fp32 per row).  Returns packed codes [rows, K/2]
    (uint8) and logical scale bytes [rows, K/16] (uint8)."""
    x = np.ascontiguousarray(x_bits).view(np.uint16)
    rows, K = x.shape
    assert K % 16 == 0
    g = np.broadcast_to(np.asarray(g_row, dtype=np.float32), (rows,)).copy()
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, K // 16), dtype=np.uint8)
    _L().oracle_quantize_rows(_ptr(x), rows, K, K, _ptr(g), _ptr(codes), _ptr(scales))
    return codes, scales


def segment_scales(x_bits: np.ndarray, segments) -> np.ndarray:
    """One global scale per module segment (half-open row ranges)."""
    return np.array([global_scale(amax(x_bits, a, b)) for a, b in segments], dtype=np.float32)


def rows_scale(segments, g_seg, rows: int) -> np.ndarray:
    g = np.zeros(rows, dtype=np.float32)
    for (a, b), gs in zip(segments, g_seg):
        g[a:b] = gs
    return g


def quantize_tensor(x_bits: np.ndarray):
    """Dynamic per-tensor quantization: returns (codes, logical scales, g)."""
    g = global_scale(amax(x_bits))
    c, s = quantize(x_bits, g)
    return c, s, np.float32(g)


def quantize_segments(x_bits: np.ndarray, segments):
    """Per-module quantization of a fused weight: returns (codes, logical
    scales, g per segment)."""
    g_seg = segment_scales(x_bits, segments)
    c, s = quantize(x_bits, rows_scale(segments, g_seg, x_bits.shape[0]))
    return c, s, g_seg


def dequant(codes: np.ndarray, scales: np.ndarray, g_row) -> np.ndarray:
    """fp64 values code * scale * g, shape [rows, K]."""
    rows, half = codes.shape
    K = half * 2
    g = np.broadcast_to(np.asarray(g_row, dtype=np.float32), (rows,)).copy()
    out = np.zeros((rows, K), dtype=np.float64)
    _L().oracle_dequant_rows(_ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)),
                             rows, K, _ptr(g), _ptr(out))
    return out


# ----------------------------------------------------- scale-factor layout

def sf_offset(r: int, c: int, K: int) -> int:
    return int(_L().oracle_sf_offset(r, c, K))


def sf_bytes(rows: int, K: int) -> int:
    return int(_L().oracle_sf_bytes(rows, K))


def swizzle(logical: np.ndarray, K: int) -> np.ndarray:
    rows = logical.shape[0]
    out = np.zeros(sf_bytes(rows, K), dtype=np.uint8)
    _L().oracle_swizzle_scales(_ptr(np.ascontiguousarray(logical)), rows, K, _ptr(out))
    return out


def unswizzle(swz: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.zeros((rows, K // 16), dtype=np.uint8)
    _L().oracle_unswizzle_scales(_ptr(np.ascontiguousarray(swz)), rows, K, _ptr(out))
    return out


# --------------------------------------------------------------------- GEMM

def linear_full(a_codes, a_scales, g_a, w_codes, w_scales, g_w_row):
    """Full fp64 GEMM over the dequantised operands: C = A^ @ W^.T and the
    error-bound reference B = |A^| @ |W^|.T (a library matmul is one step)."""
    A = dequant(a_codes, a_scales, g_a)
    W = dequant(w_codes, w_scales, g_w_row)
    return A @ W.T, np.abs(A) @ np.abs(W).T


def linear_sampled(a_codes, a_scales, g_a, w_codes, w_scales, g_w_row, ms, ns):
    """C[i], B[i] for the outputs (ms[i], ns[i]) only, by sequential fp64
    dot products."""
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    K = a_codes.shape[1] * 2
    g = np.ascontiguousarray(np.broadcast_to(np.asarray(g_w_row, dtype=np.float32), (w_codes.shape[0],)))
    C = np.zeros(len(ms), dtype=np.float64)
    B = np.zeros(len(ms), dtype=np.float64)
    _L().oracle_linear_sampled(_ptr(np.ascontiguousarray(a_codes)), _ptr(np.ascontiguousarray(a_scales)),
                               float(np.float32(g_a)), _ptr(np.ascontiguousarray(w_codes)),
                               _ptr(np.ascontiguousarray(w_scales)), _ptr(g), K, _ptr(ms), _ptr(ns),
                               len(ms), _ptr(C), _ptr(B))
    return C, B


def gemm_tolerance(B: np.ndarray) -> np.ndarray:
    """Per-element bound |gpu - oracle| <= 1e-5 * sum|a*b| + 1e-6."""
    return 1e-5 * B + 1e-6


# ------------------------------------------------------- MLP intermediate

def swiglu(gate_up_bits: np.ndarray) -> np.ndarray:
    """h = bf16(silu(gate) * up) in fp64 from a [rows, 2F] bf16 matrix whose
    first F columns are the gate and last F the up projection."""
    x = np.ascontiguousarray(gate_up_bits).view(np.uint16)
    rows, F2 = x.shape
    F = F2 // 2
    h = np.zeros((rows, F), dtype=np.uint16)
    _L().oracle_swiglu(_ptr(x), rows, F, F2, _ptr(h))
    return h


# ------------------------------------------------------ gated MLP (fused)

def gated_stored_row(r: int, F: int) -> int:
    """Row at which the gated weight layout stores input row r of a [gate F |
    up F] weight: 128-row blocks alternate gate, up, gate, up, ..."""
    module, i = divmod(r, F)
    block, within = divmod(i, 128)
    return (2 * block + module) * 128 + within


def interleave_gate_up(rows_data: np.ndarray, F: int) -> np.ndarray:
    """Reorder the rows of a [2F, ...] array into the gated storage order."""
    out = np.empty_like(rows_data)
    for r in range(2 * F):
        out[gated_stored_row(r, F)] = rows_data[r]
    return out


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """silu(g) * u = g / (1 + exp(-g)) * u, in fp64."""
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g)) * np.asarray(u, dtype=np.float64)


# ------------------------------------------------------ FP8 KV-cache codec
# The KV cache in FP8 (E4M3) with one calibrated FP32 decode scale per cache
# tensor (the recipe ships calibrated KV-cache scales: freegardner.com, section
# "The Calibrated Cache That Ships for Free"; thevalue.engineering, section
# "Efficiency Gains and Serving Optimization").  Readings: s = amax / 448,
# code = E4M3_RNE_satfinite(x / s), sign kept.

def e4m3_encode_signed(y: float) -> int:
    """E4M3 byte of a signed fp32 value: nearest even magnitude, saturating
    at 448, sign bit from the input (so -0 and small negatives give 0x80)."""
    return _L().oracle_e4m3_encode(float(np.float32(y)))


def fp8_kv_scale(a: float) -> float:
    """Calibrated FP32 decode scale s = amax / 448 (1.0 when amax == 0)."""
    return float(np.float32(_L().oracle_fp8_kv_scale(float(np.float32(a)))))


def fp8_kv_quantize(x_bits: np.ndarray, s: float) -> np.ndarray:
    """FP8 codes [rows, cols] (uint8) of a bf16 matrix (uint16 bits)."""
    x = np.ascontiguousarray(x_bits).view(np.uint16)
    rows, cols = x.shape
    out = np.empty((rows, cols), dtype=np.uint8)
    _L().oracle_fp8_kv_quantize(_ptr(x), rows, cols, cols, float(np.float32(s)), _ptr(out), cols)
    return out
