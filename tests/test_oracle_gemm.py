"""Pins of the oracle GEMM, its BF16 rounding, grouped form and scale layout.

Independent references: hand-worked closed forms (tests/golden), brute force
with exact fractions and a decoder written here from the format definitions,
torch's float32 -> bfloat16 conversion (round-to-nearest-even), and structural
invariants (one-hot rows, grouped == per-group, layout bijection).
"""
from fractions import Fraction as F
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1 = [F(x) for x in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]


def e2m1(c):
    v = E2M1[c & 7]
    return -v if c & 8 else v


def e4m3(b):
    e, m = (b >> 3) & 0xF, b & 7
    v = F(m, 512) if e == 0 else F(8 + m, 8) * F(2) ** (e - 7)
    return -v if b & 0x80 else v


def code_at(row_bytes, k):
    return (int(row_bytes[k // 2]) >> (4 * (k % 2))) & 0xF


def exact_dot(a_bytes, sa, b_bytes, sb, K):
    return sum(e2m1(code_at(a_bytes, k)) * e4m3(int(sa[k // 16])) * e2m1(code_at(b_bytes, k)) * e4m3(int(sb[k // 16]))
               for k in range(K))


def bf16_rne(v: F) -> int:
    """BF16 bit pattern of the exact rational v, round to nearest even."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if F(2) ** e > a:
        e -= 1
    quantum = F(2) ** (-133) if e < -126 else F(2) ** (e - 7)
    q = round(a / quantum)                      # Python rounds halves to even
    r = q * quantum
    if r >= F(2) ** 128:
        return sign | 0x7F80
    bits = np.array([float(r)], np.float32).view(np.uint32)[0]
    return sign | int(bits >> 16)


def test_bf16_helper_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000),
                        rng.standard_normal(2000) * 1e-39]).astype(np.float32)
    x = x[np.isfinite(x)]
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    for xi, ti in zip(x[:4000], t[:4000]):
        assert bf16_rne(F(float(xi))) == ti, float(xi)


@pytest.mark.parametrize("seed", range(4))
def test_oracle_bf16_of_scaled(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(1500):
        S = int(rng.integers(-2 ** 62, 2 ** 62)) >> int(rng.integers(0, 62))
        alpha = np.float32(rng.standard_normal() * 2.0 ** int(rng.integers(-60, 40)))
        got = oracle.bf16_of_scaled(S, float(alpha))
        assert got == bf16_rne(F(S) * F(float(alpha)) / 2 ** 20), (S, float(alpha))


def test_oracle_bf16_ties_subnormals_overflow():
    # exact ties: 1 + 2^-8 lies halfway between bf16 1.0 and 1 + 2^-7 -> even (1.0)
    assert oracle.bf16_of_scaled(2 ** 20 + 2 ** 12, 1.0) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert oracle.bf16_of_scaled(2 ** 20 + 3 * 2 ** 12, 1.0) == 0x3F82
    # just above the tie rounds up
    assert oracle.bf16_of_scaled(2 ** 20 + 2 ** 12 + 1, 1.0) == 0x3F81
    # smallest subnormal 2^-133 and half of it (tie to even -> 0)
    tiny = np.float32(2.0 ** -140)
    assert oracle.bf16_of_scaled(2 ** 27, float(tiny)) == 0x0001
    assert oracle.bf16_of_scaled(2 ** 26, float(tiny)) == 0x0000
    # overflow to infinity, with sign
    big = np.float32(2.0 ** 120)
    assert oracle.bf16_of_scaled(2 ** 40, float(big)) == 0x7F80
    assert oracle.bf16_of_scaled(-(2 ** 40), float(big)) == 0xFF80
    assert oracle.bf16_of_scaled(0, -3.0) == 0x0000


def _bytes(h):
    return np.frombuffer(bytes.fromhex(h), np.uint8)


def test_k16_closed_form_golden():
    cases = json.load(open(os.path.join(GOLDEN, "k16_closed_form.json")))["cases"]
    for c in cases:
        K = c["K"]
        a, b = _bytes(c["a_bytes"])[None, :], _bytes(c["b_bytes"])[None, :]
        sa = np.array([int(x, 16) for x in c["sa"]], np.uint8)[None, :]
        sb = np.array([int(x, 16) for x in c["sb"]], np.uint8)[None, :]
        D, ref, ad = oracle.gemm(a, sa, b, sb, c["alpha"], 1, 1, K)
        assert ref[0, 0] == c["expected"], c["name"]
        assert oracle.bf16_bits_to_float(D)[0, 0] == np.float32(c["expected"]), c["name"]


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (2, 3, 16), (3, 2, 32), (3, 3, 64), (1, 2, 48), (2, 1, 64)])
def test_bruteforce_tiny(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = rng.integers(0, 0x7F, (M, K // 16), dtype=np.uint8)
    sB = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
    alpha = np.float32(rng.standard_normal() * 1e-3)
    D, ref, ad = oracle.gemm(A, sA, B, sB, float(alpha), M, N, K)
    for m in range(M):
        for n in range(N):
            s = exact_dot(A[m], sA[m], B[n], sB[n], K)
            v = s * F(float(alpha))
            assert ref[m, n] == float(v)
            assert D[m, n] == bf16_rne(v)
            absd = sum(abs(e2m1(code_at(A[m], k)) * e4m3(int(sA[m][k // 16])) *
                           e2m1(code_at(B[n], k)) * e4m3(int(sB[n][k // 16]))) for k in range(K))
            assert ad[m, n] == pytest.approx(float(absd * abs(F(float(alpha)))), rel=1e-15)


def test_one_hot_rows_select_columns_of_B():
    # Row m of A holds a single 1.0 (code 0x2) at k = km[m]; then
    # D[m, n] = alpha * sA[m, km/16] * e2m1(B[n, km]) * sB[n, km/16].
    M, N, K = 7, 5, 128
    rng = np.random.default_rng(3)
    km = [0, 1, 15, 16, 63, 64, 127]
    A = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(km):
        A[m, k // 2] = 0x2 << (4 * (k % 2))
    sA = rng.integers(0x20, 0x50, (M, K // 16), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sB = rng.integers(0x20, 0x50, (N, K // 16), dtype=np.uint8)
    D, ref, _ = oracle.gemm(A, sA, B, sB, 1.0, M, N, K)
    for m, k in enumerate(km):
        for n in range(N):
            expect = e4m3(int(sA[m, k // 16])) * e2m1(code_at(B[n], k)) * e4m3(int(sB[n, k // 16]))
            assert ref[m, n] == float(expect)


def test_identity_codes_reproduce_B():
    # A = "identity" in 16-blocks: row m has 1.0 at k = m, scale 1.0;
    # D = B's decoded values (times its scales) in the first M columns of K.
    K = 64
    M = 64
    A = np.zeros((M, K // 2), np.uint8)
    for m in range(M):
        A[m, m // 2] |= 0x2 << (4 * (m % 2))
    sA = np.full((M, K // 16), 0x38, np.uint8)
    rng = np.random.default_rng(4)
    N = 9
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sB = rng.integers(0x30, 0x40, (N, K // 16), dtype=np.uint8)
    _, ref, _ = oracle.gemm(A, sA, B, sB, 1.0, M, N, K)
    for m in range(M):
        for n in range(N):
            assert ref[m, n] == float(e2m1(code_at(B[n], m)) * e4m3(int(sB[n, m // 16])))


def test_sampled_matches_full():
    rng = np.random.default_rng(5)
    M, N, K = 9, 11, 96
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = rng.integers(0, 0x7F, (M, K // 16), dtype=np.uint8)
    sB = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
    D, ref, ad = oracle.gemm(A, sA, B, sB, 0.75, M, N, K)
    r = rng.integers(0, M, 30)
    c = rng.integers(0, N, 30)
    Ds, refs, ads = oracle.gemm_sampled(A, sA, B, sB, 0.75, M, N, K, r, c)
    assert (Ds == D[r, c]).all() and (refs == ref[r, c]).all() and (ads == ad[r, c]).all()


def test_grouped_bruteforce_with_empty_groups():
    rng = np.random.default_rng(6)
    G, N, K = 5, 3, 32
    counts = [2, 0, 3, 0, 1]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    Mt = int(off[-1])
    A = rng.integers(0, 256, (Mt, K // 2), dtype=np.uint8)
    sA = rng.integers(0x20, 0x48, (Mt, K // 16), dtype=np.uint8)
    B = rng.integers(0, 256, (G, N, K // 2), dtype=np.uint8)
    sB = rng.integers(0x20, 0x48, (G, N, K // 16), dtype=np.uint8)
    alpha = rng.standard_normal(G).astype(np.float32)
    D, ref, _ = oracle.grouped_gemm(A, sA, B, sB, alpha, off, G, Mt, N, K)
    for g in range(G):
        for m in range(off[g], off[g + 1]):
            for n in range(N):
                v = exact_dot(A[m], sA[m], B[g, n], sB[g, n], K) * F(float(alpha[g]))
                assert ref[m, n] == float(v)
                assert D[m, n] == bf16_rne(v)


def test_oracle_rejects_bad_scales_and_shapes():
    A = np.zeros((1, 8), np.uint8)
    s = np.full((1, 1), 0x7F, np.uint8)       # NaN scale
    with pytest.raises(ValueError):
        oracle.gemm(A, s, A, np.zeros((1, 1), np.uint8), 1.0, 1, 1, 16)
    with pytest.raises(ValueError):
        oracle.gemm(A, np.full((1, 1), 0x80, np.uint8), A, np.zeros((1, 1), np.uint8), 1.0, 1, 1, 16)


def test_swizzle_layout_positions():
    rows, K = 200, 512                     # 2 row blocks, 8 K-steps of 64
    kb = K // 16
    s = np.arange(rows * kb, dtype=np.int64).reshape(rows, kb)
    s8 = (s % 251 + 1).astype(np.uint8)    # distinct-ish non-zero bytes
    out = oracle.swizzle_scales(s8, rows, K)
    assert out.size == 2 * 8 * 512
    steps = K // 64
    # hand-worked positions within the 512-byte atom: 16*(r%32) + 4*(r/32) + j
    for r, b, off in [(0, 0, 0), (1, 0, 16), (32, 0, 4), (33, 3, 16 + 4 + 3), (127, 2, 16 * 31 + 12 + 2),
                      (0, 4, 512), (5, 31, 7 * 512 + 80 + 3), (128, 0, steps * 512), (199, 5, steps * 512 + 512 + 16 * 7 + 8 + 1)]:
        assert out[off] == s8[r, b], (r, b, off)
    # padding rows are zero and every source byte lands exactly once
    counts = np.zeros(256, np.int64)
    np.add.at(counts, out, 1)
    src = np.zeros(256, np.int64)
    np.add.at(src, s8.ravel(), 1)
    assert (counts[1:] == src[1:]).all()
    assert counts[0] == out.size - s8.size
