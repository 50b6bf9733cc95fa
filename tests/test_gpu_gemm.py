"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Inputs come from the shared generator and are quantised by the ORACLE; the
GPU GEMM result must satisfy, element by element,
    |gpu - ref| <= 2^-8 |ref| + 2^-20 |alpha| sum_k |a_k b_k|
(ref = the exact value).  The quantiser and the scale re-layout are integer
work and must be bit-exact.
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


def run_gemm(nv, ca, sa, cb, sb, alpha):
    D = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    return D.float().cpu().numpy()


# ------------------------------------------------------------------ quantize
@pytest.mark.parametrize("rows,K,kind,seed", [
    (8, 6144, "normal", 1000), (33, 512, "moe", 7), (17, 256, "uniform", 3), (1, 16, "normal", 5),
    (64, 2048, "moe", 11), (3, 8192, "uniform", 13)])
def test_quantize_bitexact(nv, rows, K, kind, seed):
    X = synth.source(kind, rows, 8, K, seed)[0]
    c, s, g = oracle.quantize(X)
    gc, gs, gg = nv.quantize(dev(X))
    torch.cuda.synchronize()
    assert np.float32(gg.item()) == np.float32(g)
    assert (gs.cpu().numpy() == s).all()
    assert (gc.cpu().numpy() == c).all()


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("rows,K,kind,seed,gmul", [
    (8, 6144, "normal", 1000, 1.0),      # g from the tensor's own amax
    (33, 512, "moe", 7, 0.37),           # smaller g: scales and codes saturate on outlier blocks
    (17, 256, "uniform", 3, 5.0),        # larger g: small block scales, subnormal E4M3 bytes
    (3, 8192, "normal", 13, 1.0)])
def test_quantize_scaled_bitexact(nv, bf16, rows, K, kind, seed, gmul):
    # One-launch quantizer with the global scale given, fp32 and BF16 input;
    # BF16 values widen to fp32 exactly, so the oracle sees the same numbers.
    X = synth.source(kind, rows, 8, K, seed)[0]
    Xt = dev(X)
    if bf16:
        Xt = Xt.to(torch.bfloat16)
        X = Xt.float().cpu().numpy()
    g = float(np.float32(oracle.quantize(X)[2] * gmul))
    c, s = oracle.quantize_with_scale(X, g)
    gc, gs = nv.quantize_scaled(Xt, g)
    torch.cuda.synchronize()
    assert (gs.cpu().numpy() == s).all()
    assert (gc.cpu().numpy() == c).all()


def test_quantize_scaled_then_gemm_chain(nv):
    # Activations quantized by nvfp4_quantize_scaled and consumed by the GEMM
    # that follows on the stream (programmatic dependent launch between them),
    # three times back to back with new activations each time.
    M, N, K = 16, 768, 2048
    W = synth.source("moe", M, N, K, 1201)[1]
    cb, sb, gb = oracle.quantize(W)
    B, SB = dev(cb), dev(sb)
    for rep in range(3):
        X = synth.activations_with_outliers(M, K, 300 + rep)
        ga = float(np.float32(oracle.quantize(X)[2]))
        ca, sa = oracle.quantize_with_scale(X, ga)
        alpha = float(np.float32(ga) * np.float32(gb))
        _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
        qa, qs = nv.quantize_scaled(dev(X), ga)
        D = nv.gemm(qa, qs, B, SB, alpha)
        torch.cuda.synchronize()
        assert nv.get_device_error() == 0
        assert not violations(D.float().cpu().numpy(), ref, ad).any()


@pytest.mark.parametrize("M,N,K", [
    (1, 768, 6144), (8, 768, 6144), (16, 2048, 1024),   # one 16-row activation tile (fused)
    (33, 768, 2048), (64, 256, 6144),                   # 32-row tiles, two of them at M=64 (fused)
    (100, 520, 1024),                                    # beyond the swapped plans: quantize, then GEMM
    (7, 264, 320)])                                      # K % 256 != 0: quantize, then GEMM
@pytest.mark.parametrize("fuse", ["0", "1"])
def test_gemm_bf16a_matches_quantize_then_gemm(nv, monkeypatch, fuse, M, N, K):
    # BF16 activations quantized inside nvfp4_gemm_bf16a (by the separate
    # quantizer, or with NVFP4_GEMM_FUSE_QUANT=1 by the GEMM kernel where the
    # shape allows) give the same bits as nvfp4_quantize_scaled followed by
    # nvfp4_gemm, and the oracle's result within the bound.
    monkeypatch.setenv("NVFP4_GEMM_FUSE_QUANT", fuse)
    X = synth.activations_with_outliers(M, K, 500 + M)
    A = dev(X).to(torch.bfloat16)
    Xb = A.float().cpu().numpy()
    ga = float(np.float32(oracle.quantize(Xb)[2]))
    W = synth.normal(N, K, 600 + N, std=0.02)
    cb, sb, gb = oracle.quantize(W)
    B, SB = dev(cb), dev(sb)
    alpha = float(np.float32(ga) * np.float32(gb))
    ca, sa = oracle.quantize_with_scale(Xb, ga)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    D1 = nv.gemm_bf16a(A, ga, B, SB, alpha)
    qa, qs = nv.quantize_scaled(A, ga)
    D2 = nv.gemm(qa, qs, B, SB, alpha)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert torch.equal(D1.view(torch.int16), D2.view(torch.int16))
    assert not violations(D1.float().cpu().numpy(), ref, ad).any()


def test_quantize_scaled_rejects_bad_arguments(nv):
    X = torch.ones((4, 32), device="cuda")
    for g in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(nv.Nvfp4Error):
            nv.quantize_scaled(X, g)
    with pytest.raises(TypeError):
        nv.quantize_scaled(X.half(), 1.0)


def test_quantize_rounding_edges_bitexact(nv):
    # Values placed on E2M1 midpoints, E4M3 midpoints, zeros of both signs,
    # tiny magnitudes and saturating blocks, to pin the hardware conversions
    # against the oracle's nearest-even definition.
    K = 256
    rng = np.random.default_rng(99)
    X = np.zeros((6, K), np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 6.0, 0.1], np.float32)
    X[0, :] = np.resize(np.concatenate([mids, -mids]), K)
    X[0, ::16] = 6.0                                   # g*s == 1 in every block: exact midpoints
    X[1, :] = -0.0
    X[1, 5] = 1e-30
    X[2, :] = rng.standard_normal(K).astype(np.float32) * np.float32(1e-6)
    X[2, 0] = 6.0
    X[3, :] = np.resize(np.array([1.0, -1.0, 0.0, 3e-3], np.float32), K)
    X[4, :] = rng.uniform(-6, 6, K).astype(np.float32)
    X[5, :] = rng.standard_normal(K).astype(np.float32) * np.exp(rng.uniform(-12, 3, K)).astype(np.float32)
    c, s, g = oracle.quantize(X)
    gc, gs, gg = nv.quantize(dev(X))
    torch.cuda.synchronize()
    assert np.float32(gg.item()) == np.float32(g)
    assert (gs.cpu().numpy() == s).all()
    assert (gc.cpu().numpy() == c).all()


# ------------------------------------------------------------------ swizzle
@pytest.mark.parametrize("rows,K", [(1, 64), (128, 256), (200, 6144), (257, 512)])
def test_swizzle_bitexact(nv, rows, K):
    s = synth.random_scales(rows, K, rows + K)
    ref = oracle.swizzle_scales(s, rows, K)
    got = nv.swizzle_scales(dev(s), K)
    torch.cuda.synchronize()
    assert (got.cpu().numpy() == ref).all()


# ------------------------------------------------------------------ GEMM
SHAPES = [
    # (M, N, K, kind, seed): the pages' shapes at small M, plus ragged tails
    (8, 768, 6144, "normal", 1000),      # single GEMM M=8 (attention projection)
    (1, 768, 6144, "normal", 1100),
    (16, 256, 6144, "moe", 1201),
    (64, 2048, 1024, "moe", 1202),
    (128, 768, 512, "normal", 1103),
    (129, 264, 512, "uniform", 21),      # first non-swapped size, ragged tiles
    (300, 520, 1024, "uniform", 22),
    (5, 40, 64, "normal", 23),           # one K step
    (37, 136, 320, "moe", 24),           # K tail: 5 steps = 1 stage + 1 step
    (256, 256, 2048, "uniform", 25),
    (512, 768, 768, "normal", 26),
    (200, 264, 320, "moe", 27),          # K tail, non-swapped: scale atoms, several Q tiles
    (700, 256, 1024, "uniform", 28),     # few weight columns: narrow non-swapped tiles
]


@pytest.mark.parametrize("M,N,K,kind,seed", SHAPES)
def test_gemm_matches_oracle(nv, M, N, K, kind, seed):
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, kind, seed)
    D, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; first at {np.argwhere(bad)[:3].tolist()}"
    # the output is non-zero where the exact value is (the "silently zero" failure)
    assert np.count_nonzero(got) >= 0.99 * np.count_nonzero(ref)


def test_gemm_random_codes_all_scales(nv):
    # every code value and a wide spread of scales, including E4M3 subnormals
    M, N, K = 96, 200, 1024
    ca, cb = synth.random_codes(M, K, 1), synth.random_codes(N, K, 2)
    sa = synth.random_scales(M, K, 3, lo=0x00, hi=0x7E)
    sb = synth.random_scales(N, K, 4, lo=0x00, hi=0x7E)
    alpha = 3.0e-5
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    assert not violations(got, ref, ad).any()


@pytest.mark.parametrize("M", [3, 200])
def test_gemm_one_hot_pins_layouts(nv, M):
    # Row m of A is a single 1.0 at k = km[m]: D[m, n] = alpha sA[m, km/16] B[n, km] sB[n, km/16],
    # which pins the nibble order, the K position of every scale block and the row mapping.
    N, K = 136, 512
    rng = np.random.default_rng(M)
    km = rng.integers(0, K, M)
    A = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(km):
        A[m, k // 2] = 0x2 << (4 * (k % 2))
    sa = synth.random_scales(M, K, 5)
    cb = synth.random_codes(N, K, 6)
    sb = synth.random_scales(N, K, 7)
    _, ref, ad = oracle.gemm(A, sa, cb, sb, 1.0, M, N, K)
    got = run_gemm(nv, A, sa, cb, sb, 1.0)
    assert not violations(got, ref, ad).any()
    assert np.count_nonzero(ref) > 0


def test_gemm_alpha_is_applied(nv):
    ca, sa, cb, sb, alpha = quantized_problem(16, 128, 256, "normal", 31)
    g1 = run_gemm(nv, ca, sa, cb, sb, 1.0)
    g2 = run_gemm(nv, ca, sa, cb, sb, 0.5)
    assert np.abs(g1).max() > 0
    assert (g2 == (g1 * 0.5)).all()      # scaling by a power of two is exact in bf16 here


@pytest.mark.parametrize("M,N,K", [(1, 768, 6144), (256, 768, 6144), (2048, 2048, 512), (2048, 2048, 6144)])
def test_gemm_deterministic(nv, M, N, K):
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 41)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    d1 = nv.gemm(A, SA, B, SB, alpha).clone()
    d2 = nv.gemm(A, SA, B, SB, alpha)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


def test_gemm_does_not_write_outside_D(nv):
    M, N, K = 37, 136, 320
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 51)
    guard = 4096
    buf = torch.full((M * N + 2 * guard,), 12345.0, dtype=torch.bfloat16, device="cuda")
    D = buf[guard:guard + M * N].view(M, N)
    nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha, out=D)
    torch.cuda.synchronize()
    assert (buf[:guard] == 12345.0).all() and (buf[guard + M * N:] == 12345.0).all()


def test_shape_mismatch_raises(nv):
    A = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")      # K = 128
    B = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")     # K = 256
    with pytest.raises(ValueError, match="K mismatch"):
        nv.gemm(A, torch.zeros((4, 8), dtype=torch.uint8, device="cuda"), B,
                torch.zeros((8, 16), dtype=torch.uint8, device="cuda"), 1.0)


# ------------------------------------------------------------------ full-size sampled parity
# Every configured shape at full size, on the configs' own inputs (seeded fp32
# sources quantized by the oracle): the single 8 x 768 x 6144 GEMM, the
# attention sweep, the MoE sweep (N = 2048 and 256) and the saturation sweep
# ("Peeling the Kernel Onion", sections "The Chain of Reasoning", "The
# Benchmark Design" and "The Results").  Outputs are sampled: random
# positions plus every tile-edge row and column (boundary_samples).
CONFIG_SHAPES = ([("single_8x768x6144", 8, 768, 6144, "normal", 1000)] + synth.attention_sweep() +
                 synth.moe_sweep() + synth.saturation_sweep())


_problems = {}


def config_problem(M, N, K, kind, seed):
    key = (M, N, K, kind, seed)
    if key not in _problems:
        _problems.clear()            # keep at most one large problem in host memory
        _problems[key] = quantized_problem(M, N, K, kind, seed)
    return _problems[key]


def run_gemm_sampled(nv, ca, sa, cb, sb, alpha, rows, cols):
    M, N = ca.shape[0], cb.shape[0]
    assert rows.min() >= 0 and rows.max() < M and cols.min() >= 0 and cols.max() < N   # checked before any gather
    D = nv.gemm(dev(ca), dev(sa), dev(cb), dev(sb), alpha)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    r = torch.from_numpy(rows.astype(np.int64)).cuda()
    c = torch.from_numpy(cols.astype(np.int64)).cuda()
    return D[r, c].float().cpu().numpy()


# The saturation shapes run twice in a row: on the CTA-pair kernel (the
# default) and with NVFP4_GEMM_PAIR=0 on the single-CTA persistent kernel.
CONFIG_CASES = []
for _c in CONFIG_SHAPES:
    if _c[0].startswith("sat_"):
        CONFIG_CASES += [_c + ("pair",), _c + ("single_cta",)]
    else:
        CONFIG_CASES.append(_c + ("default",))


@pytest.mark.parametrize("name,M,N,K,kind,seed,kernel", CONFIG_CASES,
                         ids=[f"{c[0]}-{c[6]}" for c in CONFIG_CASES])
def test_config_shape_sampled(nv, monkeypatch, name, M, N, K, kind, seed, kernel):
    if kernel == "single_cta":
        monkeypatch.setenv("NVFP4_GEMM_PAIR", "0")
    ca, sa, cb, sb, alpha = config_problem(M, N, K, kind, seed)
    rows, cols = boundary_samples(M, N, seed + (kernel == "single_cta"), n_random=3000)
    got = run_gemm_sampled(nv, ca, sa, cb, sb, alpha, rows, cols)
    _, ref, ad = oracle.gemm_sampled(ca, sa, cb, sb, alpha, M, N, K, rows, cols)
    assert not violations(got, ref, ad).any()


# 128 < M <= 256 with N >= 2048 takes 128-wide tiles, which have the second
# producer warp: full, ragged and short-K shapes on the default plan, sampled.
@pytest.mark.parametrize("M,N,K", [(256, 8192, 8192), (256, 6144, 768), (200, 2048, 2048), (129, 4096, 1024)])
def test_mid_m_wide_n_sampled(nv, M, N, K):
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 71)
    rows, cols = boundary_samples(M, N, 71, n_random=2000)
    got = run_gemm_sampled(nv, ca, sa, cb, sb, alpha, rows, cols)
    _, ref, ad = oracle.gemm_sampled(ca, sa, cb, sb, alpha, M, N, K, rows, cols)
    assert not violations(got, ref, ad).any()


# ------------------------------------------------------------------ bounded waits
def test_wait_timeout_reports_and_context_survives(nv):
    assert nv.get_device_error() == 0
    nv.debug_wait_timeout(20_000_000)            # 20 ms on a barrier nothing arrives on
    assert nv.get_device_error() == 5            # NVFP4_ERR_TIMEOUT
    assert nv.get_device_error() == 0            # cleared
    ca, sa, cb, sb, alpha = quantized_problem(8, 128, 256, "normal", 61)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, 8, 128, 256)
    assert not violations(run_gemm(nv, ca, sa, cb, sb, alpha), ref, ad).any()


def test_gemm_unaligned_scales_take_the_relayout_path(nv):
    # sA 4-byte aligned but not 16-byte aligned: the library re-lays the scales
    # out in global scratch instead of loading row-major tiles with TMA.
    M, N, K = 24, 256, 1024
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 71)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    buf = torch.zeros(sa.size + 4, dtype=torch.uint8, device="cuda")
    sA = buf[4:].view(M, K // 16)
    sA.copy_(dev(sa))
    D = nv.gemm(dev(ca), sA, dev(cb), dev(sb), alpha)
    torch.cuda.synchronize()
    assert not violations(D.float().cpu().numpy(), ref, ad).any()


def test_gemm_pair_path_unaligned_scales(nv):
    # The CTA-pair kernel re-lays both scale tensors out into atoms on the
    # device; with sA and sB only 4-byte aligned the re-layout reads them a
    # word at a time.
    M, N, K = 2304, 4352, 512
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 73)
    bufa = torch.zeros(sa.size + 4, dtype=torch.uint8, device="cuda")
    bufb = torch.zeros(sb.size + 4, dtype=torch.uint8, device="cuda")
    sA = bufa[4:].view(M, K // 16)
    sB = bufb[4:].view(N, K // 16)
    sA.copy_(dev(sa))
    sB.copy_(dev(sb))
    D = nv.gemm(dev(ca), sA, dev(cb), sB, alpha)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    rows, cols = boundary_samples(M, N, 77)
    _, ref, ad = oracle.gemm_sampled(ca, sa, cb, sb, alpha, M, N, K, rows, cols)
    assert not violations(D.float().cpu().numpy()[rows, cols], ref, ad).any()


@pytest.mark.parametrize("M,N,K", [(1, 768, 6144), (16, 256, 1024), (200, 264, 512), (512, 768, 2048)])
def test_gemm_b_constant_prefetch_matches_oracle(nv, M, N, K):
    # nvfp4_gemm_ex with the constant-B flag starts loading B before the
    # previous kernel on the stream has finished; results must not change.
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "moe", 81 + M)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    A, SA, B, SB = dev(ca), dev(sa), dev(cb), dev(sb)
    outs = []
    for _ in range(3):      # back-to-back launches exercise the early start
        outs.append(nv.gemm(A, SA, B, SB, alpha, b_constant=True))
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    for D in outs:
        assert not violations(D.float().cpu().numpy(), ref, ad).any()


@pytest.mark.parametrize("M,N,K", [(8, 768, 2048), (16, 256, 1024), (512, 768, 2048)])
def test_gemm_b_constant_after_producer_of_A(nv, M, N, K):
    # A is written by the kernel right before the GEMM; with the flag only B
    # may be read early, so D must reflect the new A.  The shapes take the
    # split-K kernel, the swapped 16-row tiles and the 128-wide unswapped
    # tiles (the last two with A and B on separate producer warps).
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "normal", 91)
    ca2, sa2, _, _, _ = quantized_problem(M, N, K, "normal", 92)
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


@pytest.mark.parametrize("plan,M,N,K", [
    ("1:16:16", 8, 768, 6144),     # 16-CTA split-K cluster (non-portable size)
    ("0:256:8", 512, 512, 4096),   # 256-wide tiles, split-K slots in the ring
    ("1:64:4", 100, 256, 2048),    # swapped, two token tiles
    ("0:32:2", 300, 136, 1024),    # narrow tiles, ragged N
    ("1:16:1", 40, 264, 512),      # swapped, three token tiles, no split
])
def test_gemm_forced_plans_match_oracle(nv, monkeypatch, plan, M, N, K):
    # Every tile plan the dispatcher can take must give the same results.
    monkeypatch.setenv("NVFP4_GEMM_PLAN", plan)
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "uniform", 101 + M)
    _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} outside the bound"


def boundary_samples(M, N, seed, n_random=4000, edge=256):
    """Random (row, col) pairs plus every element of the rows and columns
    that sit on either side of a 128/256 tile edge and at the ragged end."""
    rng = np.random.default_rng(seed)
    rows = [rng.integers(0, M, n_random)]
    cols = [rng.integers(0, N, n_random)]
    for r in sorted({x for x in (0, 127, 128, 255, 256, M - 1) if x < M}):
        c = np.arange(0, N, max(1, N // edge))
        rows.append(np.full(c.size, r))
        cols.append(c)
    for c in sorted({x for x in (0, 127, 128, 255, 256, N - 1) if x < N}):
        r = np.arange(0, M, max(1, M // edge))
        rows.append(r)
        cols.append(np.full(r.size, c))
    rows.append(np.array([M - 1, M - 1, 0]))
    cols.append(np.array([N - 1, 0, N - 1]))
    return np.concatenate(rows), np.concatenate(cols)


@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("M,N,K,full", [
    (1024, 2432, 256, True),      # 8 x 19 = 152 tiles of 128x128: persistent, BQ 128
    (1100, 4104, 512, False),     # 153 tiles of 128x256, ragged M and N: CTA-pair tiles of 256x256
                                  # whose second half lies wholly past M (rows) and N (columns)
    (4096, 4096, 1024, False),    # 32 x 16 = 512 tiles, several tiles per CTA (pair)
    (2304, 4352, 2048, False),    # 9 x 17 pair tiles, long K
    (1025, 4352, 256, False),     # one K tile per tile; the last tile row holds a single row of A
    (1280, 9000, 768, False),     # last tile column holds 40 columns: the second CTA's B rows all past N
    (2048, 2048, 6144, False),    # 64 pair tiles on 74 pairs, long K
    (1800, 1544, 2048, False),    # ragged M and N (8 valid columns in the last tile column)
    (520, 6144, 512, False),      # a mid-size M on pair tiles: the last tile row holds 8 rows
])
def test_gemm_persistent_path_matches_oracle(nv, monkeypatch, pair, M, N, K, full):
    # NVFP4_GEMM_PAIR=0 selects the single-CTA persistent kernel where the
    # CTA-pair kernel would run; both must give the oracle's results.
    monkeypatch.setenv("NVFP4_GEMM_PAIR", pair)
    ca, sa, cb, sb, alpha = quantized_problem(M, N, K, "uniform", 131 + M)
    got = run_gemm(nv, ca, sa, cb, sb, alpha)
    if full:
        _, ref, ad = oracle.gemm(ca, sa, cb, sb, alpha, M, N, K)
        assert not violations(got, ref, ad).any()
    else:
        rows, cols = boundary_samples(M, N, M + N)
        _, ref, ad = oracle.gemm_sampled(ca, sa, cb, sb, alpha, M, N, K, rows, cols)
        assert not violations(got[rows, cols], ref, ad).any()
