"""CPU oracle for the NVFP4 block-scaled GEMM (ctypes view of nvfp4_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product package
``nvfp4_block_scaled_gemm_b200`` never imports it, and the two share no code.

Every function here is argument marshalling around the plain C in
``nvfp4_oracle.c``; the arithmetic, and the page citations for it, live there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (IEEE float, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "nvfp4_oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, f32, f64 = ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.oracle_e2m1_value.restype = f64
        L.oracle_e2m1_value.argtypes = [i32]
        L.oracle_e4m3_value.restype = f64
        L.oracle_e4m3_value.argtypes = [i32]
        L.oracle_e4m3_rne_satfinite.restype = i32
        L.oracle_e4m3_rne_satfinite.argtypes = [f32]
        L.oracle_e2m1_rne_satfinite.restype = i32
        L.oracle_e2m1_rne_satfinite.argtypes = [f32]
        L.oracle_quantize.restype = i32
        L.oracle_quantize.argtypes = [P, i32, i32, P, P, P]
        L.oracle_quantize_with_scale.argtypes = [P, i32, i32, f32, P, P]
        L.oracle_quantize_with_scale.restype = i32
        L.oracle_gemm.restype = i32
        L.oracle_gemm.argtypes = [P, P, P, P, f32, i32, i32, i32, P, P, P]
        L.oracle_gemm_sampled.restype = i32
        L.oracle_gemm_sampled.argtypes = [P, P, P, P, f32, i32, i32, i32, P, P, i32, P, P, P]
        L.oracle_grouped_gemm.restype = i32
        L.oracle_grouped_gemm.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, P, P, P]
        L.oracle_bf16_of_scaled.restype = ctypes.c_uint16
        L.oracle_bf16_of_scaled.argtypes = [ctypes.c_int64, ctypes.c_uint64, f32]
        L.oracle_swizzled_bytes.restype = ctypes.c_long
        L.oracle_swizzled_bytes.argtypes = [i32, i32]
        L.oracle_swizzle_scales.restype = i32
        L.oracle_swizzle_scales.argtypes = [P, i32, i32, P]
        L.oracle_dot.restype = ctypes.c_uint16
        L.oracle_dot.argtypes = [P, P, P, P, i32, f32, P, P]
        L.oracle_sparse24_compress.restype = i32
        L.oracle_sparse24_compress.argtypes = [P, i32, i32, P, P]
        L.oracle_sparse24_decompress.restype = i32
        L.oracle_sparse24_decompress.argtypes = [P, P, i32, i32, P]
        L.oracle_quantize_sparse24.restype = i32
        L.oracle_quantize_sparse24.argtypes = [P, i32, i32, P, P, P, P]
        L.oracle_gemm_sparse24.restype = i32
        L.oracle_e8m0_value.restype = ctypes.c_double
        L.oracle_e8m0_value.argtypes = [i32]
        L.oracle_quantize_mxfp4.restype = i32
        L.oracle_quantize_mxfp4.argtypes = [P, i32, i32, P, P]
        L.oracle_gemm_mxfp4.restype = i32
        L.oracle_gemm_mxfp4.argtypes = [P, P, P, P, f32, i32, i32, i32, P, P, P]
        L.oracle_gemm_sparse24.argtypes = [P, P, P, P, P, f32, i32, i32, i32, P, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().oracle_e4m3_value(int(byte))


def e4m3_rne(v: float) -> int:
    return lib().oracle_e4m3_rne_satfinite(float(v))


def e2m1_rne(v: float) -> int:
    return lib().oracle_e2m1_rne_satfinite(float(v))


def quantize(X: np.ndarray):
    """fp32 [rows, K] -> (codes u8 [rows, K/2], scales u8 [rows, K/16], g float)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows, K = X.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    g = np.zeros(1, np.float32)
    rc = lib().oracle_quantize(_p(X), rows, K, _p(codes), _p(scales), _p(g))
    if rc:
        raise ValueError("oracle_quantize rejected its input")
    return codes, scales, float(g[0])


def quantize_with_scale(X: np.ndarray, g: float):
    """fp32 [rows, K] and a given global scale g -> (codes u8 [rows, K/2], scales u8 [rows, K/16])."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows, K = X.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    rc = lib().oracle_quantize_with_scale(_p(X), rows, K, ctypes.c_float(g), _p(codes), _p(scales))
    if rc:
        raise ValueError("oracle_quantize_with_scale rejected its input")
    return codes, scales


def gemm(A, sA, B, sB, alpha: float, M: int, N: int, K: int):
    """-> (D bf16 bits uint16 [M,N], exact value f64 [M,N], |alpha|*sum|a_k b_k| f64 [M,N])."""
    A, sA, B, sB = (np.ascontiguousarray(x, dtype=np.uint8) for x in (A, sA, B, sB))
    D = np.zeros((M, N), np.uint16)
    ref = np.zeros((M, N), np.float64)
    ad = np.zeros((M, N), np.float64)
    rc = lib().oracle_gemm(_p(A), _p(sA), _p(B), _p(sB), float(alpha), M, N, K, _p(D), _p(ref), _p(ad))
    if rc:
        raise ValueError("oracle_gemm rejected its input")
    return D, ref, ad


def gemm_sampled(A, sA, B, sB, alpha: float, M: int, N: int, K: int, rows, cols):
    A, sA, B, sB = (np.ascontiguousarray(x, dtype=np.uint8) for x in (A, sA, B, sB))
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    n = len(rows)
    D = np.zeros(n, np.uint16)
    ref = np.zeros(n, np.float64)
    ad = np.zeros(n, np.float64)
    rc = lib().oracle_gemm_sampled(_p(A), _p(sA), _p(B), _p(sB), float(alpha), M, N, K,
                                   _p(rows), _p(cols), n, _p(D), _p(ref), _p(ad))
    if rc:
        raise ValueError("oracle_gemm_sampled rejected its input")
    return D, ref, ad


def grouped_gemm(A, sA, B, sB, alpha, row_offsets, G: int, M_total: int, N: int, K: int):
    A, sA, B, sB = (np.ascontiguousarray(x, dtype=np.uint8) for x in (A, sA, B, sB))
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    off = np.ascontiguousarray(row_offsets, dtype=np.int32)
    D = np.zeros((M_total, N), np.uint16)
    ref = np.zeros((M_total, N), np.float64)
    ad = np.zeros((M_total, N), np.float64)
    rc = lib().oracle_grouped_gemm(_p(A), _p(sA), _p(B), _p(sB), _p(alpha), _p(off), G, M_total, N, K,
                                   _p(D), _p(ref), _p(ad))
    if rc:
        raise ValueError("oracle_grouped_gemm rejected its input")
    return D, ref, ad


def bf16_of_scaled(S: int, alpha: float) -> int:
    """BF16 bits of the exact value alpha * S * 2^-20 (S a Python int, |S| < 2^127)."""
    u = S & ((1 << 128) - 1)
    hi = (u >> 64) & ((1 << 64) - 1)
    lo = u & ((1 << 64) - 1)
    if hi >= 1 << 63:
        hi -= 1 << 64
    return int(lib().oracle_bf16_of_scaled(hi, lo, float(alpha)))


def swizzle_scales(s: np.ndarray, rows: int, K: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.uint8)
    nbytes = lib().oracle_swizzled_bytes(rows, K)
    if nbytes < 0:
        raise ValueError("bad swizzle shape")
    out = np.zeros(nbytes, np.uint8)
    if lib().oracle_swizzle_scales(_p(s), rows, K, _p(out)):
        raise ValueError("oracle_swizzle_scales rejected its input")
    return out


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to fp32 (a bit shift; no rounding involved)."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- 2:4 sparsity
# Layout and pruning rule: see oracle_sparse24_* in nvfp4_oracle.h.

def sparse24_compress(codes: np.ndarray, K: int):
    """Dense packed codes u8 [rows, K/2] with at most 2 non-zero bytes in every
    4 -> (values u8 [rows, K/4], meta u8 [rows, K/16])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows = codes.shape[0]
    values = np.zeros((rows, K // 4), np.uint8)
    meta = np.zeros((rows, K // 16), np.uint8)
    if lib().oracle_sparse24_compress(_p(codes), rows, K, _p(values), _p(meta)):
        raise ValueError("oracle_sparse24_compress: a group has more than 2 non-zero bytes, or a bad shape")
    return values, meta


def sparse24_decompress(values: np.ndarray, meta: np.ndarray, K: int) -> np.ndarray:
    """(values [rows, K/4], meta [rows, K/16]) -> dense packed codes u8 [rows, K/2]."""
    values = np.ascontiguousarray(values, dtype=np.uint8)
    meta = np.ascontiguousarray(meta, dtype=np.uint8)
    rows = values.shape[0]
    codes = np.zeros((rows, K // 2), np.uint8)
    if lib().oracle_sparse24_decompress(_p(values), _p(meta), rows, K, _p(codes)):
        raise ValueError("oracle_sparse24_decompress: invalid metadata or shape")
    return codes


def quantize_sparse24(X: np.ndarray):
    """fp32 [rows, K] -> pruned to 2:4 over value pairs and quantized:
    (values [rows, K/4], meta [rows, K/16], scales [rows, K/16], g)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows, K = X.shape
    values = np.zeros((rows, K // 4), np.uint8)
    meta = np.zeros((rows, K // 16), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    g = np.zeros(1, np.float32)
    if lib().oracle_quantize_sparse24(_p(X), rows, K, _p(values), _p(meta), _p(scales), _p(g)):
        raise ValueError("oracle_quantize_sparse24 rejected its input")
    return values, meta, scales, float(g[0])


def gemm_sparse24(A, sA, Bv, Bm, sB, alpha: float, M: int, N: int, K: int):
    """Dense A times 2:4-sparse B: (D bf16 bits [M,N], exact f64 [M,N], |alpha| sum|a b| [M,N])."""
    A, sA, Bv, Bm, sB = (np.ascontiguousarray(x, dtype=np.uint8) for x in (A, sA, Bv, Bm, sB))
    D = np.zeros((M, N), np.uint16)
    ref = np.zeros((M, N), np.float64)
    ad = np.zeros((M, N), np.float64)
    rc = lib().oracle_gemm_sparse24(_p(A), _p(sA), _p(Bv), _p(Bm), _p(sB), float(alpha), M, N, K,
                                    _p(D), _p(ref), _p(ad))
    if rc:
        raise ValueError("oracle_gemm_sparse24 rejected its input")
    return D, ref, ad


# ---------------------------------------------------------------- MXFP4
# E2M1 values, one E8M0 scale (2^(byte - 127)) per 32 values: see nvfp4_oracle.h.

def e8m0_value(byte: int) -> float:
    return lib().oracle_e8m0_value(int(byte))


def quantize_mxfp4(X: np.ndarray):
    """fp32 [rows, K] -> (codes u8 [rows, K/2], E8M0 scales u8 [rows, K/32])."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows, K = X.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    if lib().oracle_quantize_mxfp4(_p(X), rows, K, _p(codes), _p(scales)):
        raise ValueError("oracle_quantize_mxfp4 rejected its input")
    return codes, scales


def gemm_mxfp4(A, sA, B, sB, alpha: float, M: int, N: int, K: int):
    """-> (D bf16 bits [M,N], exact value f64 [M,N], |alpha| sum|a_k b_k| f64 [M,N])."""
    A, sA, B, sB = (np.ascontiguousarray(x, dtype=np.uint8) for x in (A, sA, B, sB))
    D = np.zeros((M, N), np.uint16)
    ref = np.zeros((M, N), np.float64)
    ad = np.zeros((M, N), np.float64)
    if lib().oracle_gemm_mxfp4(_p(A), _p(sA), _p(B), _p(sB), float(alpha), M, N, K, _p(D), _p(ref), _p(ad)):
        raise ValueError("oracle_gemm_mxfp4 rejected its input")
    return D, ref, ad
