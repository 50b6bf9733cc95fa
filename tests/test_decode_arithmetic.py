"""The number facts the CUDA-core decode kernel's exactness rests on, checked
exhaustively on the host (no GPU).

That kernel sums each 16-value block as two halves of an f16x2 fma chain over
products of E2M1 values, adds the halves in fp32, multiplies by sA * sB in
fp32 and only then rounds (adding into the fp32 sum over blocks).  These tests
check, over every value that can occur, that none of those steps before the
sum over blocks can round: E2M1 values are {0, 0.5, 1, 1.5, 2, 3, 4, 6} with
a sign ("The SM120 FP4 Kernel Disaster", section "Input Knowledge Required":
4-bit values with per-block scale factors; one FP8 scale per 16 values in
"Peeling the Kernel Onion", section "The Benchmark Design").
"""
import numpy as np
import torch

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def e4m3_values():
    """Every non-negative, non-NaN E4M3 byte (0x00..0x7E) as float64."""
    b = torch.arange(0, 0x7F, dtype=torch.uint8)
    return b.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_products_are_quarter_multiples_within_36():
    p = np.outer(E2M1, E2M1).ravel()
    assert np.abs(p).max() == 36.0
    assert (p * 4 == np.round(p * 4)).all()
    assert (np.float16(p).astype(np.float64) == p).all()


def test_every_partial_half_sum_is_exact_in_f16():
    # A half of the f16x2 chain holds the sum of up to 8 products: a multiple
    # of 1/4 with magnitude at most 8 * 36 = 288.  Every such value is an f16,
    # so each fma of the chain (exact result, then rounded to f16) is exact.
    q = np.arange(-8 * 36 * 4, 8 * 36 * 4 + 1, dtype=np.float64) / 4.0
    assert (np.float16(q).astype(np.float64) == q).all()
    # and the chain itself, on random and on extreme product sequences
    rng = np.random.default_rng(7)
    p = np.outer(E2M1, E2M1).ravel()
    seqs = rng.choice(p, size=(20000, 8))
    seqs = np.vstack([seqs, np.full((1, 8), 36.0), np.full((1, 8), -36.0)])
    acc = np.zeros(seqs.shape[0], np.float16)
    for i in range(8):
        acc = (acc.astype(np.float64) + seqs[:, i]).astype(np.float16)   # one rounding per fma
    assert (acc.astype(np.float64) == seqs.sum(axis=1)).all()


def test_block_sum_times_scale_product_is_exact_in_fp32():
    # Block sum b: a multiple of 1/4 with |b| <= 576.  sA * sB over every pair
    # of scale bytes, then b * (sA * sB), both in fp32, against float64.
    s = e4m3_values()
    assert s.max() == 448.0 and s[1] == 2.0 ** -9
    sp64 = np.outer(s, s).ravel()
    sp32 = (np.float32(s)[:, None] * np.float32(s)[None, :]).ravel()
    assert (sp32.astype(np.float64) == sp64).all()
    b = (np.arange(-576 * 4, 576 * 4 + 1, dtype=np.float64) / 4.0)
    b32 = b.astype(np.float32)
    for lo in range(0, sp64.size, 1024):
        prod32 = b32[None, :] * sp32[lo:lo + 1024, None]
        assert (prod32.astype(np.float64) == b[None, :] * sp64[lo:lo + 1024, None]).all()
    # the smallest non-zero product stays a normal fp32 number
    assert 0.25 * (2.0 ** -9) ** 2 >= np.finfo(np.float32).tiny
