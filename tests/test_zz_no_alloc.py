"""nvfp4_gemm_noalloc: the GEMM entry point that allocates no device memory.

Some callers cannot let a library allocate during a call -- runtimes that own
and pool all device memory, code with a fixed memory budget, callers that
keep driver allocations off their launch path.  For them the library offers
this variant, whose only scratch (the re-laid-out scales) is a fixed static
device array.  These tests call it through the C ABI and check it against the
regular nvfp4_gemm entry point, within the same bound the other parity tests
use, on two calls in a row (the scratch is shared and reused between calls).
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import ACC_TOL, REL_TOL, quantized_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("M,N,K,kind,seed", [
    (8, 768, 6144, "normal", 1000),    # the single attention-projection GEMM
    (300, 520, 1024, "uniform", 22),   # non-swapped tiles, ragged M and N
    (37, 136, 320, "moe", 24),         # K tail (320 = 5 MMA steps)
    (200, 264, 512, "moe", 29),        # non-swapped, several Q tiles over scale atoms
])
def test_noalloc_matches_regular_entry_point_twice(nv, M, N, K, kind, seed):
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, kind, seed)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    D_ref = nv.gemm(A, SA, B, SB, alpha)
    torch.cuda.synchronize()
    _, _, absdot = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    expect = D_ref.float().cpu().numpy().astype(np.float64)
    bound = REL_TOL * np.abs(expect) + ACC_TOL * absdot
    for _ in range(2):                    # the second call reuses the same scratch
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        nv.gemm_noalloc(A, SA, B, SB, alpha, out=D)
        torch.cuda.synchronize()
        assert nv.get_device_error() == 0
        got = D.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert (np.abs(got - expect) <= bound).all()


def test_noalloc_rejects_problems_beyond_its_scratch(nv):
    # (ceil(M/128) + ceil(N/128)) * (K/64) * 512 bytes must fit 8 MiB.
    K = 8192
    rows = 8192 + 128          # 65 row blocks each side: 130 * 128 * 512 > 8 MiB
    A = torch.zeros((rows, K // 2), dtype=torch.uint8, device="cuda")
    sA = torch.zeros((rows, K // 16), dtype=torch.uint8, device="cuda")
    D = torch.empty((rows, rows), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error, match="UNSUPPORTED_SHAPE"):
        nv.gemm_noalloc(A, sA, A, sA, 1.0, out=D)
