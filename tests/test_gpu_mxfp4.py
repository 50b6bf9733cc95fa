"""GPU parity of the MXFP4 GEMM (nvfp4_gemm_mxfp4) against the oracle.

MXFP4 is the OCP microscaling sibling of NVFP4 that the same tensor-core
instruction family takes (E2M1 codes, one E8M0 scale 2^(byte - 127) per 32
values).  Inputs are quantized by the oracle (oracle_quantize_mxfp4) or drawn
as random codes and scales; expected values come from oracle_gemm_mxfp4
(an exact sum, rounded once), and every output must satisfy
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|.
Both paths run: the CUDA-core kernel for up to 4 token rows and the
tensor-core kernel (kind::mxf4) above, the latter through every tile plan
NVFP4_GEMM_PLAN can force and with both scale layouts: row-major tiles laid
out on chip (K % 512 == 0; a TMA box covers two K tiles and the kernel takes
its half) and, with NVFP4_GEMM_MX_ATOMS=1 or any other K, atoms re-laid out
in scratch first.
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


def mx_problem(M, N, K, kind, seed):
    A32, B32 = synth.source(kind, M, N, K, seed)
    ca, sa = oracle.quantize_mxfp4(A32)
    cb, sb = oracle.quantize_mxfp4(B32)
    return ca, sa, cb, sb


def check(nv, ca, sa, cb, sb, alpha, M, N, K, b_constant=False):
    _, ref, ad = oracle.gemm_mxfp4(ca, sa, cb, sb, alpha, M, N, K)
    D = nv.gemm_mxfp4(dev(ca), dev(sa), dev(cb), dev(sb), alpha, b_constant=b_constant)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    got = D.float().cpu().numpy()
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound"
    return got


@pytest.mark.parametrize("M,N,K,kind", [
    (1, 768, 6144, "normal"), (1, 2048, 6144, "moe"), (2, 256, 6144, "moe"), (3, 264, 1024, "uniform"),
    (4, 768, 320, "normal"), (1, 8, 64, "uniform")])
@pytest.mark.parametrize("b_constant", [False, True])
def test_mxfp4_decode_kernel(nv, M, N, K, kind, b_constant):
    ca, sa, cb, sb = mx_problem(M, N, K, kind, 800 + M + N + K)
    check(nv, ca, sa, cb, sb, 0.75, M, N, K, b_constant)


@pytest.fixture(params=["rowmajor", "atoms"])
def layout(request, monkeypatch):
    if request.param == "atoms":
        monkeypatch.setenv("NVFP4_GEMM_MX_ATOMS", "1")
    else:
        monkeypatch.delenv("NVFP4_GEMM_MX_ATOMS", raising=False)
    return request.param


@pytest.mark.parametrize("M,N,K,kind", [
    (5, 768, 6144, "normal"), (16, 2048, 2048, "moe"), (37, 264, 1024, "uniform"), (100, 520, 1024, "normal"),
    (300, 136, 2048, "moe"), (200, 264, 320, "uniform"), (129, 8, 192, "normal"), (700, 1024, 512, "uniform"),
    (512, 768, 6144, "normal"), (64, 2048, 1536, "moe")])
@pytest.mark.parametrize("b_constant", [False, True])
def test_mxfp4_tensor_cores(nv, layout, M, N, K, kind, b_constant):
    ca, sa, cb, sb = mx_problem(M, N, K, kind, 900 + M + N + K)
    check(nv, ca, sa, cb, sb, 1.0, M, N, K, b_constant)


@pytest.mark.parametrize("plan,M,N,K", [
    ("1:16:8", 8, 768, 6144),     # swapped, 8-way split-K cluster
    ("1:64:4", 100, 256, 2048),   # swapped, two token tiles
    ("0:128:2", 300, 520, 1024),  # unswapped, split
    ("0:256:1", 512, 512, 2048),  # 256-wide tiles: two 128-row scale blocks per Q tile
    ("1:16:1", 40, 264, 448),     # K % 128 == 64: the last atom holds one K step
    ("1:32:8", 24, 256, 6144),    # 8-way split of 24 K tiles: slices start on odd K tiles too
    ("0:64:8", 256, 512, 4096),   # unswapped 8-way split, row-major scales
])
def test_mxfp4_forced_plans(nv, monkeypatch, layout, plan, M, N, K):
    monkeypatch.setenv("NVFP4_GEMM_PLAN", plan)
    monkeypatch.setenv("NVFP4_GEMM_GEMV", "0")
    ca, sa, cb, sb = mx_problem(M, N, K, "uniform", 1000 + M)
    check(nv, ca, sa, cb, sb, 0.5, M, N, K)


@pytest.mark.parametrize("M", [1, 3, 24])
def test_mxfp4_random_codes_and_scales(nv, M):
    # Every code and a spread of E8M0 scales (2^-20 .. 2^12), per 32-value
    # block, on both paths.
    N, K = 264, 1024
    rng = np.random.default_rng(M)
    ca, cb = synth.random_codes(M, K, 11 + M), synth.random_codes(N, K, 12 + M)
    sa = rng.integers(107, 140, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(107, 140, size=(N, K // 32), dtype=np.uint8)
    check(nv, ca, sa, cb, sb, 1.0 / 3.0, M, N, K)


@pytest.mark.parametrize("M,K", [(1, 256), (24, 256), (24, 1024), (40, 2048)])
def test_mxfp4_one_hot_pins_layout(nv, M, K):
    # A row of one-hot codes against scaled one-hot columns: each output is a
    # single exact product, which pins the nibble order and which E8M0 byte
    # (block k / 32) scales element k, on both paths; K = 1024 and 2048 run
    # the row-major-scale form, whose odd K tiles read the upper half of a box.
    N = 64
    rng = np.random.default_rng(5 + M)
    ka = rng.integers(0, K, M)
    kb = rng.integers(0, K, N)
    kb[: min(N, M)] = ka[: min(N, M)]            # some outputs hit
    ca = np.zeros((M, K // 2), np.uint8)
    cb = np.zeros((N, K // 2), np.uint8)
    for m, k in enumerate(ka):
        ca[m, k // 2] |= np.uint8(0x6 << (4 * (k % 2)))          # 4.0
    for n, k in enumerate(kb):
        cb[n, k // 2] |= np.uint8(0xB << (4 * (k % 2)))          # -1.5
    sa = rng.integers(120, 134, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 134, size=(N, K // 32), dtype=np.uint8)
    got = check(nv, ca, sa, cb, sb, 1.0, M, N, K)
    D, _, _ = oracle.gemm_mxfp4(ca, sa, cb, sb, 1.0, M, N, K)
    assert np.array_equal(got, oracle.bf16_bits_to_float(D))     # one exact product per output: bit-exact


@pytest.mark.parametrize("M,N,K,scales", [
    (1, 768, 6144, "moderate"), (2, 256, 6144, "moderate"), (1, 1032, 12288, "moderate"),
    (2, 264, 8192, "moderate"), (1, 264, 2048, "tiny"), (2, 136, 1024, "tiny"), (1, 8, 64, "moderate")])
@pytest.mark.parametrize("b_constant", [False, True])
def test_mxfp4_register_form_equals_general_kernel(nv, monkeypatch, M, N, K, scales, b_constant):
    # One or two token rows run nvfp4_gemv_mx_areg_kernel; NVFP4_GEMV_AREG=0
    # runs nvfp4_gemv_mx_kernel.  Identical bits, both within the bound.
    # "tiny": exponent sums ea + eb - 254 from -174 to -94, so chunks take both
    # the multiply (a normal power of two) and the ldexpf branch.
    monkeypatch.delenv("NVFP4_GEMV_AREG", raising=False)
    rng = np.random.default_rng(3000 + M + N + K)
    ca, cb = synth.random_codes(M, K, 3001 + N), synth.random_codes(N, K, 3002 + N)
    lo, hi = (107, 140) if scales == "moderate" else (40, 81)
    sa = rng.integers(lo, hi, size=(M, K // 32), dtype=np.uint8)
    sb = rng.integers(lo, hi, size=(N, K // 32), dtype=np.uint8)
    alpha = 0.375
    _, ref, ad = oracle.gemm_mxfp4(ca, sa, cb, sb, alpha, M, N, K)
    args = (dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    D = nv.gemm_mxfp4(*args, b_constant=b_constant)
    monkeypatch.setenv("NVFP4_GEMV_AREG", "0")
    G = nv.gemm_mxfp4(*args, b_constant=b_constant)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert torch.equal(D.view(torch.int16), G.view(torch.int16))
    assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_mxfp4_deterministic_and_guarded(nv):
    M, N, K = 64, 768, 2048
    ca, sa, cb, sb = mx_problem(M, N, K, "moe", 1234)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    guard = 4096
    outs = []
    for _ in range(3):
        buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
        D = buf[guard:guard + M * N].view(M, N)
        nv.gemm_mxfp4(A, SA, B, SB, 1.0, out=D)
        torch.cuda.synchronize()
        assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()
        outs.append(D.clone())
    assert all(torch.equal(o.view(torch.int16), outs[0].view(torch.int16)) for o in outs)
    _, ref, ad = oracle.gemm_mxfp4(ca, sa, cb, sb, 1.0, M, N, K)
    assert not violations(outs[0].float().cpu().numpy(), ref, ad).any()


def test_mxfp4_rejects_bad_shapes(nv):
    A = torch.zeros((4, 48), dtype=torch.uint8, device="cuda")    # K = 96: not a multiple of 64
    s = torch.zeros((4, 3), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.Nvfp4Error, match="UNSUPPORTED_SHAPE"):
        nv.gemm_mxfp4(A, s, torch.zeros((8, 48), dtype=torch.uint8, device="cuda"),
                      torch.zeros((8, 3), dtype=torch.uint8, device="cuda"), 1.0)
