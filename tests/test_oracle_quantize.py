"""Pins of the oracle quantiser against invariants the recipe implies.

Recipe (per tensor g = amax / (6*448); per 16-block s = E4M3(amax_blk / (6 g));
q = E2M1(x / (g s)), RNE, packed with the even-k element in the low nibble).
Properties checked, each of which a dropped term, a wrong index, a swapped
nibble or a wrong sign breaks:
  * g * 2688 == amax (to one fp32 rounding);
  * every block whose scale is a normal E4M3 number puts its largest element at
    code magnitude 7 (value 6) or 6 (value 4 when the scale rounded up);
  * the decoded value g * s * e2m1(q) is within half an E2M1 step (in units of
    g*s) of x, relative to the block, and keeps x's sign;
  * order within a block is preserved (monotone);
  * packing: element k sits in byte k/2, low nibble for even k;
  * exact reconstructions: inputs already on the grid come back unchanged.
"""
import numpy as np
import pytest

import oracle
from nvfp4_block_scaled_gemm_b200 import synth

E2M1_MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
E4M3 = np.array([oracle.e4m3_value(b) for b in range(256)])


def unpack(codes, K):
    lo = codes & 0xF
    hi = codes >> 4
    out = np.empty((codes.shape[0], K), np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def dec_codes(c):
    v = E2M1_MAG[c & 7]
    return np.where(c & 8, -v, v)


@pytest.mark.parametrize("kind", ["normal", "moe", "uniform"])
def test_quantizer_invariants(kind):
    rows, K = 24, 256
    X = {"normal": synth.normal(rows, K, 1),
         "moe": synth.activations_with_outliers(rows, K, 2),
         "uniform": synth.uniform(rows, K, 3)}[kind]
    codes, scales, g = oracle.quantize(X)
    amax = float(np.abs(X).max())
    assert np.float32(amax / 2688.0) == np.float32(g)
    q = unpack(codes, K)
    s = E4M3[scales].astype(np.float64)                 # [rows, K/16]
    deq = dec_codes(q) * np.repeat(s, 16, axis=1) * g
    x = X.astype(np.float64)
    for r in range(rows):
        for b in range(K // 16):
            blk = slice(16 * b, 16 * b + 16)
            sb = s[r, b]
            if sb >= 2.0 ** -6:                         # normal E4M3 scale
                imax = np.argmax(np.abs(x[r, blk]))
                assert (q[r, blk][imax] & 7) in (6, 7)
            # error bound: half of the widest E2M1 gap (2) at this scale, plus
            # the saturation overshoot of the E4M3 rounding (< 1/16 relative)
            err = np.abs(deq[r, blk] - x[r, blk])
            assert (err <= 1.0 * g * sb * (1 + 2 ** -4) + 1e-30).all()
            # sign kept, order kept
            nz = x[r, blk] != 0
            assert (np.sign(deq[r, blk][nz]) * np.sign(x[r, blk][nz]) >= 0).all()
            o = np.argsort(x[r, blk], kind="stable")
            assert (np.diff(deq[r, blk][o]) >= 0).all()


def test_quantizer_packing_low_nibble_even():
    # x = +6g at k=0, -1.5g-ish at k=1: codes 0x7 (low) and a negative code (high)
    K = 16
    X = np.zeros((1, K), np.float32)
    X[0, 0] = 6.0
    X[0, 1] = -1.5
    X[0, 5] = 3.0
    codes, scales, g = oracle.quantize(X)
    assert g == np.float32(6.0 / 2688.0)
    # block amax 6 -> s = E4M3(6 / (6 g)) = E4M3(448) = 0x7E; g*s = 6/2688*448 = 1
    assert scales[0, 0] == 0x7E
    assert codes[0, 0] == (0xB << 4) | 0x7       # k=1 (-1.5) high nibble, k=0 (6.0) low nibble
    assert codes[0, 2] == (0x5 << 4) | 0x0       # k=5 (3.0) in the high nibble of byte 2


def test_quantizer_grid_values_roundtrip():
    # A block whose values are e2m1 grid points times a power-of-two scale
    # decodes exactly, as long as its amax is 6 * 448 * g.
    rng = np.random.default_rng(11)
    K = 64
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6], np.float32)
    X = rng.choice(grid, size=(3, K)).astype(np.float32)
    X[:, ::16] = 6.0                                  # every block has amax 6
    codes, scales, g = oracle.quantize(X)
    q = unpack(codes, K)
    assert (scales == 0x7E).all()                     # 6 / (6 g) = 448 exactly
    # g * 448 = 1 here (amax = 6), so codes decode to X itself
    assert np.float32(g * 448.0) == 1.0
    assert (dec_codes(q) == X).all()


def test_quantizer_zero_blocks_and_signed_zero():
    K = 32
    X = np.zeros((2, K), np.float32)
    X[0, :16] = np.linspace(-1, 1, 16, dtype=np.float32)
    X[1, 3] = -0.0
    codes, scales, g = oracle.quantize(X)
    assert (scales[:, 1] == 0).all() and scales[1, 0] == 0
    q = unpack(codes, K)
    assert (q[0, 16:] == 0).all()
    assert q[1, 3] == 0x8                              # -0 keeps its sign


def test_quantizer_all_zero_tensor():
    codes, scales, g = oracle.quantize(np.zeros((2, 32), np.float32))
    assert g == 1.0 and (codes == 0).all() and (scales == 0).all()


def test_quantizer_rejects_nonfinite():
    X = np.zeros((1, 16), np.float32)
    X[0, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(X)


def test_quantized_gemm_tracks_fp32_gemm():
    # End-to-end sanity of the pair quantize -> GEMM against the fp64 product
    # of the fp32 sources: 4-bit elements leave a relative Frobenius error of
    # roughly 10-15% on Gaussian data; a dropped scale or a swapped operand
    # index would make it O(1).
    M, N, K = 8, 12, 512
    A, B = synth.normal(M, K, 21), synth.normal(N, K, 22)
    ca, sa, ga = oracle.quantize(A)
    cb, sb, gb = oracle.quantize(B)
    alpha = np.float32(ga) * np.float32(gb)
    _, ref, _ = oracle.gemm(ca, sa, cb, sb, float(alpha), M, N, K)
    exact = A.astype(np.float64) @ B.astype(np.float64).T
    assert np.linalg.norm(ref - exact) / np.linalg.norm(exact) < 0.2
    assert np.corrcoef(ref.ravel(), exact.ravel())[0, 1] > 0.98


# ------------------------------------------------------ given global scale
# The configs' recipe after its first step (g fixed in advance).  Pinned to
# the amax-scaled quantizer above, to closed forms, and to saturation.

@pytest.mark.parametrize("kind,seed", [("normal", 3), ("moe", 4), ("uniform", 5)])
def test_given_scale_equals_amax_scale_quantizer(kind, seed):
    X = synth.source(kind, 13, 8, 96, seed)[0]
    c, s, g = oracle.quantize(X)
    c2, s2 = oracle.quantize_with_scale(X, g)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)


def test_given_scale_closed_form_block():
    # g = 1 and a block whose largest magnitude is 6: t = 6 / 6 = 1 -> E4M3 byte
    # 0x38 (1.0), and every value on the E2M1 grid keeps its code.
    vals = np.array([6, -3, 1.5, -0.5, 0, 4, -6, 2, 1, -1, 0.5, 3, -4, -2, -1.5, 0], np.float32)
    codes, scales = oracle.quantize_with_scale(vals.reshape(1, 16), 1.0)
    assert scales[0, 0] == 0x38
    mag = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    want = [(8 if v < 0 or (v == 0 and np.signbit(v)) else 0) | mag[abs(float(v))] for v in vals]
    got = [(codes[0, k // 2] >> (4 * (k & 1))) & 0xF for k in range(16)]
    assert got == want


def test_given_scale_saturates():
    # g far below amax / 2688: the block scale saturates at 448 (byte 0x7E) and
    # values beyond 6 * 448 * g saturate to the code of +-6.
    x = np.zeros((1, 16), np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 1000.0, -1000.0, 0.25
    g = 0.01
    codes, scales = oracle.quantize_with_scale(x, g)
    assert scales[0, 0] == 0x7E
    c0, c1 = codes[0, 0] & 0xF, codes[0, 0] >> 4
    assert c0 == 0x7 and c1 == 0xF            # +6 and -6
    # 0.25 / (0.01 * 448) = 0.0558 -> nearest E2M1 is 0
    assert codes[0, 1] & 0xF == 0


@pytest.mark.parametrize("g", [0.0, -1.0, float("inf"), float("nan")])
def test_given_scale_rejects_bad_scale(g):
    with pytest.raises(ValueError):
        oracle.quantize_with_scale(np.ones((1, 16), np.float32), g)
