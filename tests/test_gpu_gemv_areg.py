"""GPU parity of the one-or-two-row CUDA-core kernel (nvfp4_gemv_areg_kernel).

One or two token rows (with at most four 32-value chunks per thread and row
for one row, two for two rows: K <= 16384 and K <= 8192) run this form by
default.  Each thread's token chunks are decoded once and kept in registers,
and a weight chunk's two scales are converted in one instruction.  The
arithmetic and summation order are those of the general kernel
(nvfp4_gemv_kernel, still used with NVFP4_GEMV_AREG=0), so the two must agree
bit for bit; both are held to the oracle with the bound of every GEMM test:
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|.
NVFP4_GEMM_GEMV_RW forces the weight rows per row group (1, 2 or 4).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import quantized_problem, violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


CASES = [
    # M, N, K, forced rows per group ("" = the dispatcher's), what it covers
    (1, 768, 6144, "", "the attention decode shape: 1.5 chunks per thread"),
    (1, 2048, 6144, "", "the MoE decode shape, 4 rows per group"),
    (2, 256, 6144, "", "two token rows"),
    (1, 8192, 8192, "", "a large weight matrix: 2 chunks per thread"),
    (1, 1032, 12288, "", "3 chunks per thread (K > 8192)"),
    (1, 264, 16384, "4", "4 chunks per thread, the largest K of one row"),
    (2, 1000, 8192, "4", "two rows at their largest K; 250 groups of 4"),
    (1, 136, 256, "2", "K = 256: 8 chunks, most threads idle"),
    (2, 8, 64, "1", "the smallest shape: one chunk half used"),
    (1, 6144, 768, "4", "K = 768: 24 chunks per row"),
    (2, 2048, 6144, "1", "one row per group, two token rows"),
]


@pytest.mark.parametrize("b_constant", [False, True])
@pytest.mark.parametrize("M,N,K,rw,what", CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}-rw{c[3] or 'auto'}" for c in CASES])
def test_areg_kernel_matches_oracle_and_general_kernel(nv, monkeypatch, M, N, K, rw, what, b_constant):
    monkeypatch.delenv("NVFP4_GEMV_AREG", raising=False)
    if rw:
        monkeypatch.setenv("NVFP4_GEMM_GEMV_RW", rw)
    else:
        monkeypatch.delenv("NVFP4_GEMM_GEMV_RW", raising=False)
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 2100 + M + N + K)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    outs = [nv.gemm(A, SA, B, SB, alpha, b_constant=b_constant) for _ in range(2)]
    monkeypatch.setenv("NVFP4_GEMV_AREG", "0")
    general = nv.gemm(A, SA, B, SB, alpha, b_constant=b_constant)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert torch.equal(outs[1].view(torch.int16), outs[0].view(torch.int16))   # fixed summation order
    assert torch.equal(general.view(torch.int16), outs[0].view(torch.int16)), f"{what}: differs from the general kernel"
    bad = violations(outs[0].float().cpu().numpy(), ref, ad)
    assert not bad.any(), f"{what}: {bad.sum()} outside the bound"


def test_areg_kernel_subnormal_and_extreme_scales(nv, monkeypatch):
    # Scale bytes over the whole unsigned, non-NaN E4M3 range (0x00..0x7e,
    # the block scales a quantizer can write): subnormals (exponent field 0),
    # zero and the largest normals, on both operands, with random codes.
    monkeypatch.delenv("NVFP4_GEMV_AREG", raising=False)
    rng = np.random.default_rng(2150)
    M, N, K = 2, 264, 2048
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    pool = np.arange(0x7F, dtype=np.uint8)
    sa = rng.choice(pool, size=(M, K // 16)).astype(np.uint8)
    sb = rng.choice(pool, size=(N, K // 16)).astype(np.uint8)
    alpha = 0.75
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    D = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    monkeypatch.setenv("NVFP4_GEMV_AREG", "0")
    G = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    torch.cuda.synchronize()
    assert torch.equal(D.view(torch.int16), G.view(torch.int16))
    assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_areg_kernel_guard_bands_and_producer_of_A(nv, monkeypatch):
    # With constant weights the kernel loads B before the grid dependency
    # wait and A after it: A written by the previous kernel on the stream
    # must be the A it reads.
    monkeypatch.delenv("NVFP4_GEMV_AREG", raising=False)
    M, N, K = 2, 264, 2048
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 2160)
    ca2, sa2, _, _, _ = quantized_problem(M, N, K, "normal", 2161)
    _, ref2, ad2 = oracle.gemm(ca2, sa2, cb, sb, alpha, M, N, K)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    A2, SA2 = dev(ca2), dev(sa2)
    guard = 2048
    for _ in range(3):
        nv.gemm(A, SA, B, SB, alpha, b_constant=True)
        A.copy_(A2)
        SA.copy_(SA2)
        buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
        D = buf[guard:guard + M * N].view(M, N)
        nv.gemm(A, SA, B, SB, alpha, out=D, b_constant=True)
        torch.cuda.synchronize()
        assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()
        assert not violations(D.float().cpu().numpy(), ref2, ad2).any()
        A.copy_(dev(ca))
        SA.copy_(dev(sa))
