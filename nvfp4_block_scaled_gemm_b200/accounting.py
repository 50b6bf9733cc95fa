"""FLOP and byte accounting for the NVFP4 GEMM roofline.

The byte model is the one printed on "Peeling the Kernel Onion", section
"The Benchmark Design": FP4 operands packed two per byte (K/2 bytes per row),
one FP8 scale per 16 elements (K/16 bytes per row) and a BF16 output:

    bytes = M*K/2 + K*N/2 + M*K/16 + K*N/16 + 2*M*N,   flops = 2*M*N*K.

With these, the arithmetic-intensity column of that page's results table is
reproduced exactly (section "The Results").  For the grouped MoE GEMM the
weight bytes count each expert that owns at least one row once (the others
are never read), the activation and output bytes count every grouped row.
"""
from __future__ import annotations

from typing import Sequence


def gemm_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


def gemm_bytes(M: int, N: int, K: int) -> int:
    return M * K // 2 + K * N // 2 + M * K // 16 + K * N // 16 + 2 * M * N


def arithmetic_intensity(M: int, N: int, K: int) -> float:
    return gemm_flops(M, N, K) / gemm_bytes(M, N, K)


def grouped_bytes(row_counts: Sequence[int], N: int, K: int) -> int:
    active = sum(1 for c in row_counts if c > 0)
    m_total = sum(row_counts)
    return active * (N * K // 2 + N * K // 16) + m_total * (K // 2 + K // 16) + 2 * m_total * N


def grouped_flops(row_counts: Sequence[int], N: int, K: int) -> int:
    return 2 * sum(row_counts) * N * K


def roofline_time_s(flops: float, nbytes: float, peak_flops: float, peak_bytes_per_s: float) -> float:
    """Lower bound on run time: the slower of compute and memory."""
    return max(flops / peak_flops, nbytes / peak_bytes_per_s)
