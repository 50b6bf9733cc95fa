"""GPU parity of the split-K kernel (nvfp4_gemm_splitk_kernel) against the oracle.

The kernel runs nvfp4_gemm for up to 16 token rows (and 64 against at most
256 weight rows) when the scales can be loaded row-major by TMA (K % 256 ==
0, 16-byte aligned scales).  NVFP4_GEMM_SK="swap:bq:splits:stages" forces its tile, K split and ring depth, so
every branch is exercised: ring reuse (stages < K tiles per CTA), the
split-K exchange by asynchronous stores counted on the owner's barrier, the
direct (unsplit) epilogues of both orientations, the swapped and the
unswapped tiles of every width, and the early weight load of the
constant-weight flag.  Every output is checked against the
oracle's exact value within
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|.
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
    # M, N, K, NVFP4_GEMM_SK ("swap:bq:splits:stages", empty: the planner's choice), what it exercises
    (16, 768, 6144, "", "default: swapped, 16-way split, K slice resident"),
    (16, 768, 6144, "1:16:4:2", "ring reuse: 6 K tiles per CTA through 2 stages"),
    (16, 768, 6144, "1:16:1:3", "no split: direct swapped epilogue through shared memory, ring reuse"),
    (16, 768, 6144, "1:64:16:2", "a 64-wide token tile for 16 rows"),
    (64, 2048, 2048, "1:64:16:1", "BQ 64, as many splits as K tiles (8)"),
    (37, 264, 1536, "1:64:2:2", "ragged M and N (last weight tile 8 rows), BQ 64"),
    (25, 136, 2560, "1:32:8:1", "BQ 32, ragged weight tile, 2 K tiles through 1 stage"),
    (200, 520, 2048, "0:64:2:10", "unswapped: 128 token rows x 64 weight rows, 2-way split"),
    (200, 520, 2048, "0:128:1:2", "unswapped 128-wide weight tile, direct epilogue, ring reuse"),
    (200, 520, 2048, "0:64:1:2", "unswapped 64-wide weight tile, direct epilogue"),
    (300, 136, 1024, "0:128:4:1", "unswapped, ragged M and N, 4-way split"),
    (130, 8, 512, "0:64:1:10", "eight weight rows, unswapped, direct epilogue"),
    (48, 1024, 8192, "1:64:8:4", "swapped BQ 64, 4 K tiles per CTA through the ring"),
    (96, 1024, 4096, "0:128:8:2", "unswapped, one token tile against eight weight tiles"),
    (512, 768, 6144, "0:64:2:6", "the largest sweep shape: 48 tiles, 2-way split, 12 K tiles through 6 stages"),
    (64, 256, 6144, "", "default for 64 token rows against 256 weight rows"),
]


@pytest.mark.parametrize("b_constant", [False, True])
@pytest.mark.parametrize("M,N,K,sk,what", CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}-{c[3] or 'auto'}" for c in CASES])
def test_splitk_matches_oracle(nv, monkeypatch, M, N, K, sk, what, b_constant):
    if sk:
        monkeypatch.setenv("NVFP4_GEMM_SK", sk)
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 700 + M + N)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    outs = [nv.gemm(A, SA, B, SB, alpha, b_constant=b_constant) for _ in range(3)]   # back to back
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    first = outs[0].view(torch.int16)
    for D in outs:
        assert torch.equal(D.view(torch.int16), first)          # deterministic split-K sums
    bad = violations(outs[0].float().cpu().numpy(), ref, ad)
    assert not bad.any(), f"{what}: {bad.sum()} outside the bound"


def test_splitk_one_token_row(nv, monkeypatch):
    # One token row on the tensor cores (the CUDA-core kernel turned off).
    monkeypatch.setenv("NVFP4_GEMM_GEMV", "0")
    M, N, K = 1, 768, 6144
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 1100)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    D = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_splitk_guard_bands(nv, monkeypatch):
    # The 16-byte stores of both epilogues stay inside D.
    for sk, (M, N, K) in (("", (37, 264, 1536)), ("1:64:1:1", (37, 264, 1536)), ("", (200, 136, 1024)),
                          ("0:64:1:1", (200, 136, 1024)), ("0:128:1:1", (200, 136, 1024))):
        monkeypatch.setenv("NVFP4_GEMM_SK", sk) if sk else monkeypatch.delenv("NVFP4_GEMM_SK", raising=False)
        ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 900 + M)
        guard = 4096
        buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
        D = buf[guard:guard + M * N].view(M, N)
        nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha, out=D)
        torch.cuda.synchronize()
        assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()
        _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
        assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_splitk_constant_weights_after_producer_of_A(nv):
    # With the constant-weight flag only B may be read before the previous
    # kernel finishes; A written right before the GEMM must be seen.
    M, N, K = 16, 768, 6144
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 931)
    ca2, sa2, _, _, _ = quantized_problem(M, N, K, "normal", 932)
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
