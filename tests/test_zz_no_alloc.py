"""nvfp4_gemm_noalloc: the GEMM entry point that allocates no device memory.

Some callers cannot let a library allocate during a call -- runtimes that own
and pool all device memory, code with a fixed memory budget, callers that
keep driver allocations off their launch path.  For them the library offers
this variant: most problems need no scratch at all there, and the rest
re-lay their scales out into a fixed static device array.  These tests call
it through the C ABI and check, on two calls in a row (the static scratch is
shared and reused between calls), that every output is within the parity
bound of the oracle's exact value and of the regular nvfp4_gemm entry
point's result.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ACC_TOL, REL_TOL, quantized_problem, violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def dev_misaligned(x):
    """A device copy of x that starts 4 bytes past a 16-byte boundary."""
    buf = torch.zeros(x.size + 4, dtype=torch.uint8, device="cuda")
    t = buf[4:].view(*x.shape)
    t.copy_(dev(x))
    return t


def sample(M, N, seed):
    if M * N <= 400_000:
        r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        return r.ravel(), c.ravel()
    rng = np.random.default_rng(seed)
    rows = np.concatenate([rng.integers(0, M, 6000), [0, M - 1, M - 1, 0]])
    cols = np.concatenate([rng.integers(0, N, 6000), [0, N - 1, 0, N - 1]])
    return rows, cols


@pytest.mark.parametrize("M,N,K,kind,seed,misaligned", [
    (1, 768, 6144, "normal", 1100, False),    # one token row: the CUDA-core kernel
    (3, 768, 6144, "normal", 1101, False),    # three token rows, also on the CUDA cores
    (8, 768, 6144, "normal", 1000, False),    # the single attention-projection GEMM: row-major scales, no scratch
    (300, 520, 1024, "uniform", 22, False),   # non-swapped tiles, ragged M and N, no scratch
    (1024, 4608, 256, "uniform", 23, False),  # a CTA-pair-sized problem: the persistent kernel here, no scratch
    (37, 136, 320, "moe", 24, False),         # K tail (320 = 5 MMA steps): scales in the static scratch
    (8, 768, 6144, "normal", 25, True),       # scales 4-byte aligned only: the static scratch, swapped tiles
    (200, 264, 512, "moe", 29, True),         # the static scratch, non-swapped, several Q tiles over atoms
])
def test_noalloc_matches_oracle_and_regular_entry_point_twice(nv, M, N, K, kind, seed, misaligned):
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, kind, seed)
    A, B = dev(ca), dev(cb)
    SA, SB = (dev_misaligned(sa), dev_misaligned(sb)) if misaligned else (dev(sa), dev(sb))
    rows, cols = sample(M, N, seed)
    _, ref, absdot = oracle.gemm_sampled(ca, sa, cb, sb, alpha, M, N, K, rows, cols)
    D_reg = nv.gemm(A, SA, B, SB, alpha)
    torch.cuda.synchronize()
    regular = D_reg.float().cpu().numpy().astype(np.float64)[rows, cols]
    assert not violations(regular, ref, absdot).any()
    for _ in range(2):                    # the second call reuses the same scratch
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        nv.gemm_noalloc(A, SA, B, SB, alpha, out=D)
        torch.cuda.synchronize()
        assert nv.get_device_error() == 0
        full = D.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(full).all()
        got = full[rows, cols]
        assert not violations(got, ref, absdot).any()
        # and within the same bound of the regular entry point's result
        assert (np.abs(got - regular) <= REL_TOL * np.abs(regular) + ACC_TOL * absdot).all()


def test_noalloc_rejects_problems_beyond_its_scratch(nv):
    # K % 256 != 0 puts the scales through the static scratch, whose 8 MiB
    # must hold (ceil(M/128) + ceil(N/128)) * (K/64) * 512 bytes.
    K = 8192 + 64
    rows = 8192 + 128          # 65 row blocks each side: 130 * 129 * 512 > 8 MiB
    A = torch.zeros((rows, K // 2), dtype=torch.uint8, device="cuda")
    sA = torch.zeros((rows, K // 16), dtype=torch.uint8, device="cuda")
    D = torch.empty((rows, rows), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error, match="UNSUPPORTED_SHAPE"):
        nv.gemm_noalloc(A, sA, A, sA, 1.0, out=D)
