"""GPU parity of the 2:4-sparse GEMM (nvfp4_gemm_sparse24) against the CPU
oracle, through the C ABI.

Weights are pruned and quantized by the ORACLE (oracle.quantize_sparse24) or
drawn as random kept bytes and positions; both paths of the entry point run:
the CUDA-core kernel on the compressed weights (up to 8 token rows, or as set
by NVFP4_GEMM_SP24_GEMV) and the expansion to dense codes followed by the
dense GEMM.  Same bound as every GEMM parity test:
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_gemm_b200 import synth
from tests.helpers import violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def sparse_problem(M, N, K, kind, seed):
    A32, B32 = synth.source(kind, M, N, K, seed)
    ca, sa, ga = oracle.quantize(A32)
    bv, bm, sb, gb = oracle.quantize_sparse24(B32)
    alpha = float(np.float32(ga) * np.float32(gb))
    return ca, sa, bv, bm, sb, alpha


def run(nv, ca, sa, bv, bm, sb, alpha, **kw):
    D = nv.gemm_sparse24(dev(ca), dev(sa), dev(bv), dev(bm), dev(sb), alpha, **kw)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    return D.float().cpu().numpy()


@pytest.mark.parametrize("gemv_limit", ["8", "0"])
@pytest.mark.parametrize("M,N,K,kind,seed", [
    (1, 768, 6144, "normal", 2100),     # attention projection, batch 1
    (2, 256, 6144, "moe", 2101),        # MoE TP8 shape
    (3, 136, 320, "moe", 2102),         # K tail: 10 chunks of 32
    (8, 264, 64, "uniform", 2103),      # smallest K
    (16, 768, 2048, "normal", 2104),    # beyond the default limit: expansion + dense GEMM
    (300, 520, 1024, "uniform", 2105),  # non-swapped dense tiles after expansion
])
def test_sparse24_matches_oracle(nv, monkeypatch, gemv_limit, M, N, K, kind, seed):
    monkeypatch.setenv("NVFP4_GEMM_SP24_GEMV", gemv_limit)
    ca, sa, bv, bm, sb, alpha = sparse_problem(M, N, K, kind, seed)
    _, ref, ad = oracle.gemm_sparse24(ca, sa, bv, bm, sb, alpha, M, N, K)
    got = run(nv, ca, sa, bv, bm, sb, alpha)
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; first at {np.argwhere(bad)[:3].tolist()}"
    assert np.count_nonzero(got) >= 0.99 * np.count_nonzero(ref)


@pytest.mark.parametrize("rw", ["1", "2", "4"])
@pytest.mark.parametrize("M", [1, 2, 5, 16])
def test_sparse24_random_layout_every_instance(nv, monkeypatch, rw, M):
    # random kept bytes (every code) and every position pair, all scales
    monkeypatch.setenv("NVFP4_GEMM_SP24_GEMV", "16")
    monkeypatch.setenv("NVFP4_GEMM_GEMV_RW", rw)
    N, K = 200, 1024
    rng = np.random.default_rng(2200 + M)
    ca = synth.random_codes(M, K, 2201)
    sa = synth.random_scales(M, K, 2202, lo=0x00, hi=0x7E)
    bv = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    pairs = np.array([0 | 1 << 2, 0 | 2 << 2, 0 | 3 << 2, 1 | 2 << 2, 1 | 3 << 2, 2 | 3 << 2], np.uint8)
    nib = pairs[rng.integers(0, 6, size=(N, K // 8))]
    bm = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    sb = synth.random_scales(N, K, 2203, lo=0x00, hi=0x7E)
    alpha = 3.0e-5
    _, ref, ad = oracle.gemm_sparse24(ca, sa, bv, bm, sb, alpha, M, N, K)
    assert not violations(run(nv, ca, sa, bv, bm, sb, alpha), ref, ad).any()


@pytest.mark.parametrize("b_constant", [False, True])
@pytest.mark.parametrize("M,N,K,rw", [
    (1, 768, 6144, ""),      # 1.5 chunks per thread
    (1, 8192, 8192, ""),     # 2 chunks per thread, 4-row groups
    (1, 264, 16384, "2"),    # 4 chunks per thread
    (2, 1000, 8192, "4"),    # two rows at their largest K; 250 groups of 4
    (2, 136, 320, "1"),      # 10 chunks: most threads idle
    (1, 8, 64, "1"),         # one chunk, half used
])
def test_sparse24_register_form_equals_general_kernel(nv, monkeypatch, M, N, K, rw, b_constant):
    # One or two token rows run nvfp4_gemv_sp24_areg_kernel (token chunks held
    # in registers); NVFP4_GEMV_AREG=0 runs nvfp4_gemv_sp24_kernel.  Same
    # arithmetic and order: identical bits, and both within the oracle bound.
    monkeypatch.delenv("NVFP4_GEMM_SP24_GEMV", raising=False)
    monkeypatch.delenv("NVFP4_GEMV_AREG", raising=False)
    if rw:
        monkeypatch.setenv("NVFP4_GEMM_GEMV_RW", rw)
    else:
        monkeypatch.delenv("NVFP4_GEMM_GEMV_RW", raising=False)
    rng = np.random.default_rng(2300 + M + N)
    ca = synth.random_codes(M, K, 2301 + N)
    sa = synth.random_scales(M, K, 2302 + N, lo=0x20, hi=0x40)
    bv = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    pairs = np.array([0 | 1 << 2, 0 | 2 << 2, 0 | 3 << 2, 1 | 2 << 2, 1 | 3 << 2, 2 | 3 << 2], np.uint8)
    nib = pairs[rng.integers(0, 6, size=(N, K // 8))]
    bm = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    sb = synth.random_scales(N, K, 2303 + N, lo=0x20, hi=0x40)
    alpha = 1.5e-3
    _, ref, ad = oracle.gemm_sparse24(ca, sa, bv, bm, sb, alpha, M, N, K)
    args = (dev(ca), dev(sa), dev(bv), dev(bm), dev(sb), alpha)
    D = nv.gemm_sparse24(*args, b_constant=b_constant)
    monkeypatch.setenv("NVFP4_GEMV_AREG", "0")
    G = nv.gemm_sparse24(*args, b_constant=b_constant)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert torch.equal(D.view(torch.int16), G.view(torch.int16))
    assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_sparse24_equals_dense_gemm_on_expanded_weights(nv, monkeypatch):
    # Above the CUDA-core limit the entry point is the dense GEMM of the
    # expanded weights: the same bits as nvfp4_gemm on the oracle's expansion.
    monkeypatch.setenv("NVFP4_GEMM_SP24_GEMV", "0")
    M, N, K = 40, 768, 2048
    ca, sa, bv, bm, sb, alpha = sparse_problem(M, N, K, "moe", 2106)
    dense = oracle.sparse24_decompress(bv, bm, K)
    D1 = nv.gemm_sparse24(dev(ca), dev(sa), dev(bv), dev(bm), dev(sb), alpha)
    D2 = nv.gemm(dev(ca), dev(sa), dev(dense), dev(sb), alpha)
    torch.cuda.synchronize()
    assert torch.equal(D1.view(torch.int16), D2.view(torch.int16))


def test_sparse24_b_constant_after_producer_of_A(nv):
    M, N, K = 2, 768, 2048
    ca, sa, bv, bm, sb, alpha = sparse_problem(M, N, K, "normal", 2107)
    A32b = synth.source("normal", M, N, K, 2108)[0]
    ca2, sa2, _ = oracle.quantize(A32b)
    _, ref2, ad2 = oracle.gemm_sparse24(ca2, sa2, bv, bm, sb, alpha, M, N, K)
    A, SA, BV, BM, SB = dev(ca), dev(sa), dev(bv), dev(bm), dev(sb)
    A2, SA2 = dev(ca2), dev(sa2)
    for _ in range(3):
        nv.gemm_sparse24(A, SA, BV, BM, SB, alpha, b_constant=True)
        A.copy_(A2)
        SA.copy_(SA2)
        D = nv.gemm_sparse24(A, SA, BV, BM, SB, alpha, b_constant=True)
        torch.cuda.synchronize()
        assert not violations(D.float().cpu().numpy(), ref2, ad2).any()
        A.copy_(dev(ca))
        SA.copy_(dev(sa))


def test_sparse24_deterministic_and_guarded(nv):
    M, N, K = 3, 136, 320
    ca, sa, bv, bm, sb, alpha = sparse_problem(M, N, K, "normal", 2109)
    guard = 4096
    buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
    D = buf[guard:guard + M * N].view(M, N)
    args = (dev(ca), dev(sa), dev(bv), dev(bm), dev(sb), alpha)
    nv.gemm_sparse24(*args, out=D)
    d1 = D.clone()
    nv.gemm_sparse24(*args, out=D)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), D.view(torch.int16))
    assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()


def test_sparse24_rejects_bad_arguments(nv):
    A = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")        # K = 128
    sA = torch.zeros((4, 8), dtype=torch.uint8, device="cuda")
    Bv = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")       # K = 64: mismatch
    with pytest.raises(ValueError, match="K mismatch"):
        nv.gemm_sparse24(A, sA, Bv, torch.zeros((8, 4), dtype=torch.uint8, device="cuda"),
                         torch.zeros((8, 4), dtype=torch.uint8, device="cuda"), 1.0)
