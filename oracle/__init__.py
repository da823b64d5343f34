"""CPU oracle for block-wise microscaling FP4 quantization.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product package
(``microscaling_fp4_quantization_block_b200``) never imports this module, and
this module never imports the product package; they share no code.

The arithmetic lives in ``fp4q_oracle.c`` (plain single-threaded C, built with
``gcc -O2 -ffp-contract=off``); this file only builds/loads it and marshals
numpy arrays.  ``theory.py`` holds the Gaussian three-term MSE model.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4q_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

E8M0, UE4M3, UE5M3 = 0, 1, 2
G_NONE, G_COMPUTE, G_GIVEN = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, no GPU needed)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I, F, U32, U64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                  ctypes.c_uint32, ctypes.c_uint64)
        sig = {
            "orc_version": (I, []),
            "orc_bf16_to_f32": (F, [ctypes.c_uint16]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [F]),
            "orc_f32_to_bf16_array": (None, [P, I64, P]),
            "orc_bf16_to_f32_array": (None, [P, I64, P]),
            "orc_e2m1_decode": (F, [ctypes.c_uint8]),
            "orc_e2m1_encode": (ctypes.c_uint8, [F]),
            "orc_e8m0_decode": (F, [ctypes.c_uint8]),
            "orc_e8m0_from_amax": (ctypes.c_uint8, [F]),
            "orc_ue4m3_decode": (F, [ctypes.c_uint8]),
            "orc_ue4m3_encode": (ctypes.c_uint8, [F]),
            "orc_ue5m3_decode": (F, [ctypes.c_uint8]),
            "orc_ue5m3_encode": (ctypes.c_uint8, [F]),
            "orc_e2m1_encode_bits_range": (None, [U32, U64, P]),
            "orc_ue4m3_encode_bits_range": (None, [U32, U64, P]),
            "orc_e2m1_encode_array": (None, [P, I64, P]),
            "orc_ue4m3_encode_array": (None, [P, I64, P]),
            "orc_ue5m3_encode_array": (None, [P, I64, P]),
            "orc_hadamard": (I, [P, I64, I, P]),
            "orc_tensor_amax": (F, [P, I64]),
            "orc_global_scale_from_amax": (F, [F]),
            "orc_quantize_f32": (I, [P, I64, I64, I, I, I, I, P, P, P]),
            "orc_quantize_bf16": (I, [P, I64, I64, I, I, I, I, P, P, P]),
            "orc_dequantize": (I, [P, P, F, I64, I64, I, I, I, P]),
            "orc_quantize_search_f32": (I, [P, I64, I64, I, I, I, I, I, I, P, P, P]),
            "orc_quantize_search_bf16": (I, [P, I64, I64, I, I, I, I, I, I, P, P, P]),
            "orc_quantize_with_scales_f32": (I, [P, I64, I64, I, I, I, P, F, P]),
            "orc_quantize_with_scales_bf16": (I, [P, I64, I64, I, I, I, P, F, P]),
            "orc_nearest_rank": (I64, [ctypes.c_double, I64]),
            "orc_fp4_gemm": (I, [P, P, F, I64, P, P, F, I64, I64, I, I, P]),
            "orc_outlier_stats_bf16": (I, [P, I64, I64, ctypes.c_double, P, P]),
            "orc_global_scale_search_f32": (I, [P, I64, I64, I, I, I, I, I, P, P, P, P]),
            "orc_global_scale_search_bf16": (I, [P, I64, I64, I, I, I, I, I, P, P, P, P]),
            "orc_block_mse_f32": (I, [P, P, P, F, I64, I64, I, I, I, P, P]),
            "orc_block_mse_bf16": (I, [P, P, P, F, I64, I64, I, I, I, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(st: int, what: str) -> None:
    if st != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {st})")


# --------------------------------------------------------------------------- codecs
def e2m1_encode(r) -> np.ndarray:
    """One E2M1 nibble (sign in bit 3) per fp32 value, one nibble per byte."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    out = np.empty(r.shape, np.uint8)
    lib().orc_e2m1_encode_array(_ptr(r), r.size, _ptr(out))
    return out


def ue4m3_encode_array(s) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty(s.shape, np.uint8)
    lib().orc_ue4m3_encode_array(_ptr(s), s.size, _ptr(out))
    return out


def ue5m3_encode_array(s) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty(s.shape, np.uint8)
    lib().orc_ue5m3_encode_array(_ptr(s), s.size, _ptr(out))
    return out


def e2m1_encode_bits_range(lo: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint8)
    lib().orc_e2m1_encode_bits_range(lo, count, _ptr(out))
    return out


def ue4m3_encode_bits_range(lo: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint8)
    lib().orc_ue4m3_encode_bits_range(lo, count, _ptr(out))
    return out


def e2m1_decode(nibble: int) -> float:
    return lib().orc_e2m1_decode(nibble)


def ue4m3_encode(s: float) -> int:
    return lib().orc_ue4m3_encode(s)


def ue4m3_decode(c: int) -> float:
    return lib().orc_ue4m3_decode(c)


def ue5m3_encode(s: float) -> int:
    return lib().orc_ue5m3_encode(s)


def ue5m3_decode(c: int) -> float:
    return lib().orc_ue5m3_decode(c)


def e8m0_from_amax(m: float) -> int:
    return lib().orc_e8m0_from_amax(m)


def e8m0_decode(c: int) -> float:
    return lib().orc_e8m0_decode(c)


def bf16_bits_to_f32(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float32)
    lib().orc_bf16_to_f32_array(_ptr(bits), bits.size, _ptr(out))
    return out


def f32_to_bf16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


# --------------------------------------------------------------------------- path
def hadamard(x, k: int) -> np.ndarray:
    """H_k x / sqrt(k) on every run of k consecutive elements (fp64 dense -> fp32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    _check(lib().orc_hadamard(_ptr(x), x.size, k, _ptr(y)), "hadamard")
    return y


def tensor_amax(y) -> float:
    y = np.ascontiguousarray(y, dtype=np.float32)
    return lib().orc_tensor_amax(_ptr(y), y.size)


def global_scale_from_amax(amax: float) -> float:
    return lib().orc_global_scale_from_amax(amax)


def quantize(x, fmt: int, block: int, rot: int = 0, gmode: int = G_NONE, gscale: float = 1.0):
    """Quantize a 2-D tensor given as fp32 values or as bf16 bit patterns (uint16).

    Returns ``(codes uint8[rows, cols/2], scales uint8[rows, cols/block], G float)``.
    """
    x = np.ascontiguousarray(x)
    if x.ndim != 2:
        raise ValueError("expected a 2-D array")
    rows, cols = x.shape
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // block if block else 0), np.uint8)
    g = np.array([gscale], np.float32)
    fn = lib().orc_quantize_bf16 if x.dtype == np.uint16 else lib().orc_quantize_f32
    if x.dtype not in (np.uint16, np.float32):
        raise TypeError("x must be float32 values or uint16 bf16 bit patterns")
    _check(fn(_ptr(x), rows, cols, fmt, block, rot, gmode, _ptr(g), _ptr(codes), _ptr(scales)),
           "quantize")
    return codes, scales, float(g[0])


def quantize_search(x, fmt: int, block: int, rot: int = 0, gmode: int = G_NONE, gscale: float = 1.0,
                    below: int = 1, above: int = 1):
    """Quantize with MSE-optimised block scales: per block, the max-rule code and
    the codes up to `above` above and `below` below it are tried (in that order)
    and the one of least squared error is kept (ties keep the earlier one).

    Returns ``(codes, scales, G)`` like :func:`quantize`.
    """
    x = np.ascontiguousarray(x)
    if x.ndim != 2:
        raise ValueError("expected a 2-D array")
    if x.dtype not in (np.uint16, np.float32):
        raise TypeError("x must be float32 values or uint16 bf16 bit patterns")
    rows, cols = x.shape
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // block if block else 0), np.uint8)
    g = np.array([gscale], np.float32)
    fn = lib().orc_quantize_search_bf16 if x.dtype == np.uint16 else lib().orc_quantize_search_f32
    _check(fn(_ptr(x), rows, cols, fmt, block, rot, gmode, below, above, _ptr(g), _ptr(codes), _ptr(scales)),
           "quantize_search")
    return codes, scales, float(g[0])


def global_scale_search(x, fmt: int, block: int, rot: int = 0, below: int = 4, above: int = 4):
    """MSE-optimised per-tensor scale: candidates G_j = fp32(G0 (16 + j) / 16),
    j in [-below, above], the max rule for the block scales under each.
    Returns ``(codes, scales, G*, errs)`` with errs[j + below] the candidate's
    per-tensor MSE (fp64)."""
    x = np.ascontiguousarray(x)
    if x.ndim != 2:
        raise ValueError("expected a 2-D array")
    rows, cols = x.shape
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // block if block else 0), np.uint8)
    g = np.zeros(1, np.float32)
    errs = np.full(below + above + 1, np.nan, np.float64)
    fn = lib().orc_global_scale_search_bf16 if x.dtype == np.uint16 else lib().orc_global_scale_search_f32
    _check(fn(_ptr(x), rows, cols, fmt, block, rot, below, above, _ptr(g), _ptr(errs), _ptr(codes), _ptr(scales)),
           "global_scale_search")
    return codes, scales, float(g[0]), errs


def quantize_with_scales(x, scales, G: float, fmt: int, block: int, rot: int = 0) -> np.ndarray:
    """Codes of x for given scale bytes (each block quantized with its own S)."""
    x = np.ascontiguousarray(x)
    if x.dtype not in (np.uint16, np.float32):
        raise TypeError("x must be float32 values or uint16 bf16 bit patterns")
    rows, cols = x.shape
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    codes = np.empty((rows, cols // 2), np.uint8)
    fn = lib().orc_quantize_with_scales_bf16 if x.dtype == np.uint16 else lib().orc_quantize_with_scales_f32
    _check(fn(_ptr(x), rows, cols, fmt, block, rot, _ptr(scales), G, _ptr(codes)), "quantize_with_scales")
    return codes


def dequantize(codes, scales, G: float, rows: int, cols: int, fmt: int, block: int,
               rot: int = 0) -> np.ndarray:
    """fp32 values decode(nibble) * S (rotated back when rot > 0)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.empty((rows, cols), np.float32)
    _check(lib().orc_dequantize(_ptr(codes), _ptr(scales), G, rows, cols, fmt, block, rot,
                                _ptr(out)), "dequantize")
    return out


def block_mse(x, codes, scales, G: float, fmt: int, block: int, rot: int = 0):
    """Per-block MSE (fp64) and tensor terms [total, non-max, max, zero-rounded]."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    bm = np.empty((rows, cols // block), np.float64)
    terms = np.zeros(4, np.float64)
    fn = lib().orc_block_mse_bf16 if x.dtype == np.uint16 else lib().orc_block_mse_f32
    _check(fn(_ptr(x), _ptr(codes), _ptr(scales), G, rows, cols, fmt, block, rot, _ptr(bm),
              _ptr(terms)), "block_mse")
    return bm, terms


def unpack_nibbles(codes) -> np.ndarray:
    """Packed code bytes -> one nibble per element (low nibble = even element)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def nearest_rank(p: float, n: int) -> int:
    """k = ceil(p n) clamped to [1, n] (0 for n = 0): the rank of the p-quantile."""
    return lib().orc_nearest_rank(p, n)


def outlier_stats(xb, p: float = 0.999):
    """Max |x|, the nearest-rank p-quantile of |x| and the per-column max |x| of
    a 2-D bf16 tensor given as uint16 bit patterns."""
    xb = np.ascontiguousarray(xb, dtype=np.uint16)
    rows, cols = xb.shape
    stats = np.zeros(2, np.float32)
    col = np.zeros(cols, np.float32)
    _check(lib().orc_outlier_stats_bf16(_ptr(xb), rows, cols, p, _ptr(stats), _ptr(col)), "outlier_stats")
    return float(stats[0]), float(stats[1]), col


def fp4_gemm(codes_a, scales_a, ga: float, codes_b, scales_b, gb: float, k: int, fmt: int, block: int):
    """Y = G_A G_B sum_k q_A s_A q_B s_B (fp64, [rows_A][rows_B]) of two quantized
    operands, each [rows][k] with blocks of `block` along k."""
    if k <= 0:
        raise ValueError("k must be positive")
    codes_a = np.ascontiguousarray(codes_a, dtype=np.uint8)
    codes_b = np.ascontiguousarray(codes_b, dtype=np.uint8)
    scales_a = np.ascontiguousarray(scales_a, dtype=np.uint8)
    scales_b = np.ascontiguousarray(scales_b, dtype=np.uint8)
    m = codes_a.size * 2 // k
    n = codes_b.size * 2 // k
    y = np.empty((m, n), np.float64)
    _check(lib().orc_fp4_gemm(_ptr(codes_a), _ptr(scales_a), ga, m, _ptr(codes_b), _ptr(scales_b), gb, n, k, fmt,
                              block, _ptr(y)), "fp4_gemm")
    return y
