"""GPU parity of the CUDA-core kernel for a few token rows (nvfp4_gemv_kernel),
through the C ABI, against the CPU oracle.

nvfp4_gemm hands it M = 1 always, and M <= 2 or 4 for the smaller weight
matrices; NVFP4_GEMM_GEMV=<n> sends every M <= n (up to 16) to it and
NVFP4_GEMM_GEMV_RW forces the weight rows per CTA, so every instance the
dispatcher can pick is run here.  Same bound as every GEMM parity test:
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_gemm_b200 import synth
from tests.helpers import quantized_problem, violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def bf16_bits_to_f64(d):
    return (np.asarray(d, np.uint32) << 16).view(np.float32).astype(np.float64)


def run_gemm(nv, ca, sa, cb, sb, alpha, **kw):
    D = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha, **kw)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    return D.float().cpu().numpy()


@pytest.fixture
def gemv_up_to_16(monkeypatch):
    monkeypatch.setenv("NVFP4_GEMM_GEMV", "16")


@pytest.mark.parametrize("rw", ["1", "2", "4"])
@pytest.mark.parametrize("M,N,K,kind,seed", [
    (1, 768, 6144, "normal", 1100),     # attention projection, batch 1
    (2, 256, 6144, "moe", 1211),        # MoE TP8 shape
    (3, 136, 320, "moe", 31),           # K = 10 chunks of 32: most threads idle
    (4, 768, 64, "uniform", 32),        # smallest K: two chunks per row
    (5, 520, 1024, "normal", 33),       # M between instances (8-row instance)
    (8, 264, 16448, "uniform", 34),     # 514 chunks per row: three load groups per thread
    (16, 768, 2048, "moe", 35),         # the largest instance
    (1, 2048, 8192, "moe", 36),         # MoE N = 2048
])
def test_gemv_matches_oracle(nv, monkeypatch, gemv_up_to_16, rw, M, N, K, kind, seed):
    monkeypatch.setenv("NVFP4_GEMM_GEMV_RW", rw)
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, kind, seed)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; first at {np.argwhere(bad)[:3].tolist()}"
    assert np.count_nonzero(got) >= 0.99 * np.count_nonzero(ref)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_gemv_random_codes_all_scales(nv, gemv_up_to_16, M):
    # every code value and scales over the whole non-negative E4M3 range,
    # subnormals included
    N, K = 200, 1024
    ca, cb = synth.random_codes(M, K, 61), synth.random_codes(N, K, 62)
    sa = synth.random_scales(M, K, 63, lo=0x00, hi=0x7E)
    sb = synth.random_scales(N, K, 64, lo=0x00, hi=0x7E)
    alpha = 3.0e-5
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    assert not violations(run_gemm(nv, ca, sa, cb, sb, alpha), ref, ad).any()


def test_gemv_block_sums_at_their_largest(nv, gemv_up_to_16):
    # Every code +-6 with the largest scale: each half of a block's f16x2 sum
    # reaches 8 * 36 = 288 and a block 576 * 448^2, where any rounding inside
    # a block would show.  Equal signs in row 0 (no cancellation), random
    # signs elsewhere (cancellation down to small results).
    M, N, K = 4, 136, 2048
    rng = np.random.default_rng(65)

    def codes(rows, same_sign_row0):
        sign = rng.integers(0, 2, size=(rows, K)).astype(np.uint8)
        if same_sign_row0:
            sign[0] = 0
        nib = (0x7 | (sign << 3)).astype(np.uint8)
        return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)

    ca, cb = codes(M, True), codes(N, True)
    sa = np.full((M, K // 16), 0x7E, np.uint8)
    sb = np.full((N, K // 16), 0x7E, np.uint8)
    alpha = 2.0 ** -40        # a power of two: applying it rounds nothing
    D, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    assert not violations(got, ref, ad).any()
    # row 0 x column 0: no cancellation and every partial sum exact, so the
    # result is the exact value rounded once to bf16, as the oracle rounds it
    assert got[0, 0] == bf16_bits_to_f64(D)[0, 0]


def test_gemv_one_hot_pins_layouts(nv, gemv_up_to_16):
    # Row m of A is a single 1.0 at k = km[m]: D[m, n] = alpha sA[m, km/16] B[n, km] sB[n, km/16],
    # which pins the nibble order, the scale block of every K position and the row mapping.
    M, N, K = 3, 136, 512
    rng = np.random.default_rng(66)
    km = rng.integers(0, K, M)
    A = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(km):
        A[m, k // 2] = 0x2 << (4 * (k % 2))
    sa = synth.random_scales(M, K, 67)
    cb = synth.random_codes(N, K, 68)
    sb = synth.random_scales(N, K, 69)
    D, ref, ad = oracle.gemm(A, sa, cb, sb, 1.0, M, N, K)
    got = run_gemm(nv, A, sa, cb, sb, 1.0)
    assert (got == bf16_bits_to_f64(D)).all()   # one exact product per output: bit-exact


@pytest.mark.parametrize("M,N,K", [(1, 768, 6144), (3, 256, 1024)])
def test_gemv_deterministic_and_equal_across_rows_per_cta(nv, monkeypatch, gemv_up_to_16, M, N, K):
    # The sum order depends only on the thread layout along K, not on how many
    # weight rows a CTA takes: every instance gives the same bits, every time.
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 71)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    outs = []
    for rw in ("1", "2", "4", "1"):
        monkeypatch.setenv("NVFP4_GEMM_GEMV_RW", rw)
        outs.append(nv.gemm(A, SA, B, SB, alpha).clone())
    torch.cuda.synchronize()
    for d in outs[1:]:
        assert torch.equal(outs[0].view(torch.int16), d.view(torch.int16))


def test_gemv_b_constant_after_producer_of_A(nv):
    # With the constant-B flag the kernel loads its first weight chunks before
    # the previous kernel on the stream has finished; A, written by that
    # kernel, must still be read after it.
    M, N, K = 2, 768, 2048
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 93)
    ca2, sa2, _, _, _ = quantized_problem(M, N, K, "normal", 94)
    _, ref2, ad2 = oracle.gemm(ca2, sa2, cb, sb, alpha, M, N, K)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    A2, SA2 = dev(ca2), dev(sa2)
    for _ in range(3):
        nv.gemm(A, SA, B, SB, alpha, b_constant=True)
        A.copy_(A2)
        SA.copy_(SA2)
        D = nv.gemm(A, SA, B, SB, alpha, b_constant=True)
        torch.cuda.synchronize()
        assert not violations(D.float().cpu().numpy(), ref2, ad2).any()
        A.copy_(dev(ca))
        SA.copy_(dev(sa))


def test_gemv_and_tensor_core_paths_agree_with_the_oracle(nv, monkeypatch):
    # The same decode problem through both kernels (NVFP4_GEMM_GEMV=0 sends
    # it to the tensor cores): both within the bound of the exact result.
    M, N, K = 4, 768, 6144
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 1212)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    for setting in ("4", "0"):
        monkeypatch.setenv("NVFP4_GEMM_GEMV", setting)
        assert not violations(run_gemm(nv, ca, sa, cb, sb, alpha), ref, ad).any()


def test_gemv_does_not_write_outside_D(nv, gemv_up_to_16):
    M, N, K = 5, 136, 320
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 72)
    guard = 4096
    buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
    D = buf[guard:guard + M * N].view(M, N)
    nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha, out=D)
    torch.cuda.synchronize()
    assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()
