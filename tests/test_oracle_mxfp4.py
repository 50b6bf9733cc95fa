"""Pins of the oracle's MXFP4 functions (no GPU).

MXFP4 is the other block-scaled FP4 format of the tensor-core instruction
family the pages turn on (they use NVFP4 only): E2M1 values, one E8M0 scale
2^(byte - 127) per 32 values.  Pinned here, independently of the oracle's C:
  * the E8M0 closed form for all 256 bytes;
  * the quantizer on hand-worked blocks and, on random data, against a
    restatement in Python (frexp for the shared exponent, nearest-even on the
    E2M1 grid);
  * the GEMM against exact rational arithmetic (fractions.Fraction) with an
    independent round-to-nearest-even to BF16, including scales at both ends
    of the E8M0 range (underflow to signed zero, overflow to infinity);
  * the GEMM against the pinned NVFP4 oracle when every scale is 1.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from nvfp4_block_scaled_gemm_b200 import synth

MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1(code):
    v = MAGS[code & 7]
    return -v if code & 8 else v


def test_e8m0_closed_form():
    for b in range(255):
        assert oracle.e8m0_value(b) == math.ldexp(1.0, b - 127)
    assert math.isnan(oracle.e8m0_value(255))


def py_e2m1_code(v):
    """Nearest E2M1 code, ties to the even code, saturating at 6, sign kept."""
    sign = 8 if math.copysign(1.0, v) < 0 else 0
    a = min(abs(v), 6.0)
    best = min(range(8), key=lambda i: (abs(MAGS[i] - a), i % 2))
    return sign | best


def py_quantize_mxfp4(X):
    X = np.asarray(X, np.float32)
    rows, K = X.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    for r in range(rows):
        for b in range(K // 32):
            blk = X[r, 32 * b:32 * b + 32]
            amax = float(np.abs(blk).max())
            if amax == 0.0:
                scales[r, b] = 0
                qs = [8 if math.copysign(1.0, float(x)) < 0 else 0 for x in blk]
            else:
                shared = min(max(math.frexp(amax)[1] - 1 - 2, -127), 127)
                scales[r, b] = shared + 127
                Xs = np.float32(math.ldexp(1.0, shared))
                qs = [py_e2m1_code(float(np.float32(x) / Xs)) for x in blk]
            for i, q in enumerate(qs):
                k = 32 * b + i
                codes[r, k // 2] |= q << (4 * (k % 2))
    return codes, scales


def test_quantizer_hand_worked_blocks():
    X = np.zeros((4, 32), np.float32)
    X[0, 0] = 6.0                                   # amax 6: 2^(2-2) = 1, byte 127, code 6
    X[1, :8] = [1.0, 0.3, -0.1, 0.0625, -0.01, 0.875, 0.625, 0.0]
    # amax 1: X = 2^-2.  1 -> 4 (0x6); 1.2 -> 1 (0x2); -0.4 -> -0.5 (0x9); 0.25 -> tie 0|0.5 -> 0;
    # -0.04 -> -0 (0x8); 3.5 -> tie 3|4 -> 4 (0x6); 2.5 -> tie 2|3 -> 2 (0x4)
    X[2, 0] = 7.0                                   # 2^(2-2) = 1: 7 saturates to 6
    X[3, 0] = -0.0                                  # all-zero block: byte 0, -0 keeps its sign
    codes, scales = oracle.quantize_mxfp4(X)
    assert scales[:, 0].tolist() == [127, 125, 127, 0]
    assert codes[0, 0] == 0x07
    assert codes[1, :4].tolist() == [0x6 | 0x2 << 4, 0x9 | 0x0 << 4, 0x8 | 0x6 << 4, 0x4 | 0x0 << 4]
    assert codes[2, 0] == 0x07
    assert codes[3, 0] == 0x08


def test_quantizer_scale_clamps():
    X = np.zeros((2, 32), np.float32)
    X[0, 0] = np.float32(2.0 ** -140)               # floor(log2) - 2 = -142, clamped to -127 (byte 0)
    X[1, 0] = np.float32(3.0e38)                    # 2^127.8: floor 127, shared 125 (byte 252)
    codes, scales = oracle.quantize_mxfp4(X)
    assert scales[:, 0].tolist() == [0, 252]
    assert codes[0, 0] == 0x00                      # 2^-13 rounds to 0
    assert codes[1, 0] == py_e2m1_code(3.0e38 / 2.0 ** 125)


@pytest.mark.parametrize("rows,K,kind,seed", [(4, 64, "normal", 1), (16, 256, "moe", 2), (3, 1024, "uniform", 3)])
def test_quantizer_matches_python_restatement(rows, K, kind, seed):
    X = synth.source(kind, rows, 8, K, seed)[0]
    X[0, :32] *= np.float32(1e-30)                  # a block of tiny values
    c, s = oracle.quantize_mxfp4(X)
    pc, ps = py_quantize_mxfp4(X)
    assert (s == ps).all()
    assert (c == pc).all()


def bf16_bits_of(fr):
    """Round a Fraction to BF16 (nearest even); exact zero -> +0."""
    if fr == 0:
        return 0x0000
    sign = 0x8000 if fr < 0 else 0
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                      # now 2^e <= a < 2^(e+1)
    q_exp = e - 7 if e >= -126 else -133
    m = a / Fraction(2) ** q_exp
    n = math.floor(m)
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    if n == 256:
        n, q_exp = 128, q_exp + 1
    if n >= 128:
        biased = q_exp + 7 + 127
        if biased >= 255:
            return sign | 0x7F80
        return sign | (biased << 7) | (n - 128)
    return sign | n


def exact_dot(a_codes, a_scales, b_codes, b_scales, K):
    s = Fraction(0)
    for k in range(K):
        ca = (int(a_codes[k // 2]) >> (4 * (k % 2))) & 0xF
        cb = (int(b_codes[k // 2]) >> (4 * (k % 2))) & 0xF
        sa = Fraction(2) ** (int(a_scales[k // 32]) - 127)
        sb = Fraction(2) ** (int(b_scales[k // 32]) - 127)
        s += Fraction(e2m1(ca)) * sa * Fraction(e2m1(cb)) * sb
    return s


@pytest.mark.parametrize("M,N,K,seed,lo,hi", [
    (2, 3, 32, 1, 120, 134),      # scales near 1
    (3, 2, 64, 2, 0, 254),        # the whole E8M0 range: sums across wildly different magnitudes
    (1, 4, 128, 3, 100, 160),
])
def test_gemm_against_exact_rationals(M, N, K, seed, lo, hi):
    rng = np.random.default_rng(seed)
    A, B = synth.random_codes(M, K, seed), synth.random_codes(N, K, seed + 1)
    sA = rng.integers(lo, hi + 1, size=(M, K // 32), dtype=np.uint8)
    sB = rng.integers(lo, hi + 1, size=(N, K // 32), dtype=np.uint8)
    alpha = float(np.float32(0.7))
    D, ref, ad = oracle.gemm_mxfp4(A, sA, B, sB, alpha, M, N, K)
    for m in range(M):
        for n in range(N):
            s = exact_dot(A[m], sA[m], B[n], sB[n], K)
            v = s * Fraction(alpha)
            assert D[m, n] == bf16_bits_of(v), (m, n)
            assert ref[m, n] == float(v)  or abs(ref[m, n] - float(v)) <= 1e-15 * abs(float(v))


def test_gemm_underflow_to_signed_zero_and_overflow_to_inf():
    K = 32
    one = 0x2 | 0x2 << 4                            # two codes of 1.0
    A = np.full((1, K // 2), one, np.uint8)
    B = np.full((2, K // 2), one, np.uint8)
    B[1] = 0xA | 0xA << 4                           # -1.0 codes
    tiny = np.zeros((1, 1), np.uint8)               # 2^-127 each side: 32 * 2^-254
    D, _, _ = oracle.gemm_mxfp4(A, tiny, B, np.zeros((2, 1), np.uint8), 1.0, 1, 2, K)
    assert D.tolist() == [[0x0000, 0x8000]]        # rounds to +0 and -0
    huge = np.full((1, 1), 254, np.uint8)           # 2^127 each side: 32 * 2^254
    D, _, _ = oracle.gemm_mxfp4(A, huge, B, np.full((2, 1), 254, np.uint8), 1.0, 1, 2, K)
    assert D.tolist() == [[0x7F80, 0xFF80]]


def test_gemm_reduces_to_nvfp4_with_unit_scales():
    M, N, K = 5, 7, 256
    A, B = synth.random_codes(M, K, 11), synth.random_codes(N, K, 12)
    alpha = 1.0e-3
    Dm, rm, am = oracle.gemm_mxfp4(A, np.full((M, K // 32), 127, np.uint8), B, np.full((N, K // 32), 127, np.uint8),
                                   alpha, M, N, K)
    Dn, rn, an = oracle.gemm(A, np.full((M, K // 16), 0x38, np.uint8), B, np.full((N, K // 16), 0x38, np.uint8),
                             alpha, M, N, K)
    assert (Dm == Dn).all() and (rm == rn).all() and (am == an).all()


def test_rejections():
    A = np.zeros((1, 16), np.uint8)
    with pytest.raises(ValueError):
        oracle.gemm_mxfp4(A, np.full((1, 1), 255, np.uint8), A, np.zeros((1, 1), np.uint8), 1.0, 1, 1, 32)
    with pytest.raises(ValueError):
        oracle.quantize_mxfp4(np.zeros((1, 48), np.float32))
