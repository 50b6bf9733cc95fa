"""Pins of the oracle's 2:4-sparse FP4 operand (no GPU).

The pages name FP4 structured sparsity as a way to cut what small-batch
decode demands ("Peeling the Kernel Onion", sections "Assumptions Embedded in
the Benchmark" and "Knowledge Created and Its Impact") but give no layout.
The reading the oracle takes: 2:4 over packed bytes, i.e. in every 4
consecutive bytes of a row (pairs of E2M1 values) at most 2 are non-zero;
values [rows][K/4] hold the kept bytes, meta [rows][K/16] a nibble
p0 | p1 << 2 per group (even group low), scales stay dense [rows][K/16].

Pinned here, independently of the oracle's C code:
  * a worked layout example, computed by hand from that definition;
  * round trips and rejections;
  * the pruning quantizer against a numpy statement of the pruning rule fed
    to the (separately pinned) dense quantizer;
  * the sparse GEMM against a brute-force sum read straight from values and
    meta, on tiny shapes.
"""
import numpy as np
import pytest

import oracle
from nvfp4_block_scaled_gemm_b200 import synth

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1(code):
    v = E2M1[code & 7]
    return -v if code & 8 else v


def test_layout_worked_example():
    # row 0: group 0 = [00 21 00 43] keeps positions 1, 3 -> nibble 1 | 3<<2 = 0xD
    #        group 1 = [65 00 00 07] keeps positions 0, 3 -> nibble 0 | 3<<2 = 0xC -> meta 0xCD
    # row 1: group 0 = [00 00 5A 00] keeps 2 and the lowest zero, 0 -> nibble 0 | 2<<2 = 0x8
    #        group 1 = [00 00 00 00] keeps 0, 1 -> nibble 0 | 1<<2 = 0x4 -> meta 0x48
    codes = np.array([[0x00, 0x21, 0x00, 0x43, 0x65, 0x00, 0x00, 0x07],
                      [0x00, 0x00, 0x5A, 0x00, 0x00, 0x00, 0x00, 0x00]], np.uint8)
    values, meta = oracle.sparse24_compress(codes, 16)
    assert values.tolist() == [[0x21, 0x43, 0x65, 0x07], [0x00, 0x5A, 0x00, 0x00]]
    assert meta.tolist() == [[0xCD], [0x48]]
    assert (oracle.sparse24_decompress(values, meta, 16) == codes).all()


def test_negative_zero_pairs_count_as_zero():
    # 0x88 is (-0, -0): a zero pair, so [88 10 00 02] has two non-zero bytes
    codes = np.array([[0x88, 0x10, 0x00, 0x02, 0x80, 0x08, 0x33, 0x00]], np.uint8)
    values, meta = oracle.sparse24_compress(codes, 16)
    assert values.tolist() == [[0x10, 0x02, 0x80, 0x33]]
    assert meta.tolist() == [[(1 | 3 << 2) | ((0 | 2 << 2) << 4)]]
    back = oracle.sparse24_decompress(values, meta, 16)
    # the dropped zero pairs come back as +0 bytes; kept ones verbatim
    assert back.tolist() == [[0x00, 0x10, 0x00, 0x02, 0x80, 0x00, 0x33, 0x00]]


def random_sparse_codes(rows, K, seed):
    rng = np.random.default_rng(seed)
    codes = np.zeros((rows, K // 2), np.uint8)
    for r in range(rows):
        for g in range(K // 8):
            nz = rng.integers(0, 3)
            for p in rng.choice(4, size=nz, replace=False):
                b = 0
                while b & 0x77 == 0:
                    b = int(rng.integers(0, 256))
                codes[r, 4 * g + p] = b
    return codes


@pytest.mark.parametrize("rows,K,seed", [(3, 16, 1), (17, 64, 2), (5, 1024, 3)])
def test_round_trip(rows, K, seed):
    codes = random_sparse_codes(rows, K, seed)
    values, meta = oracle.sparse24_compress(codes, K)
    assert values.shape == (rows, K // 4) and meta.shape == (rows, K // 16)
    assert (oracle.sparse24_decompress(values, meta, K) == codes).all()


def test_rejections():
    with pytest.raises(ValueError):      # three non-zero bytes in one group
        oracle.sparse24_compress(np.array([[0x01, 0x10, 0x00, 0x02, 0, 0, 0, 0]], np.uint8), 16)
    values = np.zeros((1, 4), np.uint8)
    for bad in (0x00, 0x01, 0x05, 0x06, 0x0B, 0x0F):  # p0 >= p1 in the low group
        with pytest.raises(ValueError):
            oracle.sparse24_decompress(values, np.array([[0x40 | bad]], np.uint8), 16)


def numpy_prune(X):
    """The pruning rule stated in numpy: per group of 4 value pairs keep the
    2 with the largest max(|x_2p|, |x_2p+1|), ties to the lower position."""
    rows, K = X.shape
    pairs = np.abs(X).reshape(rows, K // 8, 4, 2).max(axis=3)
    pos = np.broadcast_to(np.arange(4), pairs.shape)
    order = np.lexsort((pos, -pairs), axis=-1)        # largest key first, lower position first on ties
    keep = np.zeros(pairs.shape, bool)
    np.put_along_axis(keep, order[..., :2], True, axis=-1)
    mask = np.repeat(keep, 2, axis=-1).reshape(rows, K)
    return np.where(mask, X, np.float32(0)), keep


@pytest.mark.parametrize("rows,K,kind,seed", [(8, 256, "normal", 11), (33, 512, "moe", 12), (4, 6144, "uniform", 13)])
def test_pruning_quantizer_is_dense_quantizer_of_pruned_tensor(rows, K, kind, seed):
    X = synth.source(kind, rows, 8, K, seed)[0]
    values, meta, scales, g = oracle.quantize_sparse24(X)
    Xp, keep = numpy_prune(X)
    cp, sp, gp = oracle.quantize(Xp)
    assert (oracle.sparse24_decompress(values, meta, K) == cp).all()
    assert (scales == sp).all() and np.float32(g) == np.float32(gp)
    # each group keeps its largest value, so scales and g are the unpruned tensor's too
    cd, sd, gd = oracle.quantize(X)
    assert (scales == sd).all() and np.float32(g) == np.float32(gd)
    # the recorded positions are the pruning rule's, read from meta directly
    nib = np.stack([meta & 0x0F, meta >> 4], axis=-1).reshape(rows, K // 8)
    p0, p1 = nib & 3, nib >> 2
    got = np.zeros_like(keep)
    np.put_along_axis(got, p0[..., None].astype(np.int64), True, axis=-1)
    np.put_along_axis(got, p1[..., None].astype(np.int64), True, axis=-1)
    assert (got == keep).all()


def test_pruning_ties_keep_lower_positions():
    X = np.zeros((1, 16), np.float32)
    X[0, :8] = [1, -1, 1, 0, -1, 0, 0.5, 1]     # keys 1, 1, 1, 1: positions 0 and 1 win
    X[0, 8:] = [0, 0, 0, 0, 0, 2, 0, 2]         # keys 0, 0, 2, 2: positions 2 and 3
    values, meta, scales, g = oracle.quantize_sparse24(X)
    assert meta.tolist() == [[(0 | 1 << 2) | ((2 | 3 << 2) << 4)]]


@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 16, 1), (2, 3, 32, 2), (3, 5, 64, 3), (4, 2, 128, 4)])
def test_sparse_gemm_brute_force(M, N, K, seed):
    rng = np.random.default_rng(seed)
    A = synth.random_codes(M, K, seed)
    sA = synth.random_scales(M, K, seed + 10)
    Bv = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    pairs = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]
    nibs = rng.integers(0, 6, size=(N, K // 8))
    Bm = np.zeros((N, K // 16), np.uint8)
    for n in range(N):
        for g in range(K // 8):
            p0, p1 = pairs[nibs[n, g]]
            Bm[n, g // 2] |= (p0 | p1 << 2) << (4 * (g % 2))
    sB = synth.random_scales(N, K, seed + 20)
    D, ref, ad = oracle.gemm_sparse24(A, sA, Bv, Bm, sB, 1.0, M, N, K)
    for m in range(M):
        for n in range(N):
            s = 0.0
            for g in range(K // 8):
                p0, p1 = pairs[nibs[n, g]]
                for j, p in enumerate((p0, p1)):
                    byte = int(Bv[n, 2 * g + j])
                    for h in range(2):                       # low nibble = even k
                        k = 8 * g + 2 * p + h
                        a = e2m1(int(A[m, k // 2]) >> (4 * (k % 2))) * oracle.e4m3_value(int(sA[m, k // 16]))
                        b = e2m1(byte >> (4 * h)) * oracle.e4m3_value(int(sB[n, k // 16]))
                        s += a * b                           # exact: dyadic terms, < 2^53 units
            assert ref[m, n] == s
