"""Byte/FLOP accounting pinned to the printed arithmetic-intensity column of
the results table on "Peeling the Kernel Onion" (section "The Results")."""
import pytest

from nvfp4_block_scaled_gemm_b200 import accounting as acc

# (M, N, K, printed AI) -- MoE up 2K/4K/8K batch, Attn QKV 1K/2K/4K batch
PRINTED = [(2048, 2048, 6144, 2286), (4096, 2048, 6144, 2712), (8192, 2048, 6144, 2990),
           (1024, 6144, 6144, 2070), (2048, 6144, 6144, 2891), (4096, 6144, 6144, 3608)]


@pytest.mark.parametrize("M,N,K,ai", PRINTED)
def test_ai_matches_printed_table(M, N, K, ai):
    # Five of the six printed values are the formula rounded to the nearest
    # integer; the sixth (4096x6144x6144: 3607.49 printed as 3,608) is within
    # one unit, so the check is |AI - printed| < 1.
    assert abs(acc.arithmetic_intensity(M, N, K) - ai) < 1.0


def test_bytes_formula_terms():
    # FP4 operands K/2 bytes per row, one FP8 scale per 16 elements, BF16 out
    assert acc.gemm_bytes(1, 768, 6144) == 3072 + 768 * 3072 + 384 + 768 * 384 + 2 * 768
    assert acc.gemm_flops(2, 3, 64) == 768


def test_grouped_bytes_counts_active_experts_once():
    N, K = 2048, 6144
    counts = [3, 0, 5, 0]
    expect = 2 * (N * K // 2 + N * K // 16) + 8 * (K // 2 + K // 16) + 2 * 8 * N
    assert acc.grouped_bytes(counts, N, K) == expect
    assert acc.grouped_flops(counts, N, K) == 2 * 8 * N * K
