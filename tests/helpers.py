"""Shared test helpers: oracle-side input preparation and the parity bound."""
from __future__ import annotations

import numpy as np

import oracle
from nvfp4_block_scaled_gemm_b200 import synth

# Elementwise bound between the GPU result and the exact value:
#   |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|
# (half a BF16 ulp of the output, plus an fp32-accumulation allowance that
# scales with the magnitude of the terms being summed).
REL_TOL = 2.0 ** -8
ACC_TOL = 2.0 ** -20


def violations(gpu: np.ndarray, ref: np.ndarray, absdot: np.ndarray) -> np.ndarray:
    gpu = np.asarray(gpu, np.float64)
    bound = REL_TOL * np.abs(ref) + ACC_TOL * absdot
    return ~(np.abs(gpu - ref) <= bound)


def quantized_problem(M: int, N: int, K: int, kind: str, seed: int):
    """fp32 sources from the shared generator, quantised by the ORACLE."""
    A32, B32 = synth.source(kind, M, N, K, seed)
    ca, sa, ga = oracle.quantize(A32)
    cb, sb, gb = oracle.quantize(B32)
    alpha = float(np.float32(ga) * np.float32(gb))
    return ca, sa, cb, sb, alpha
