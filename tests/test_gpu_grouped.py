"""GPU parity of the grouped (MoE) NVFP4 GEMM against the oracle.

Routing follows the workload recipe: 512 tokens, top-8 of 256 experts with a
Zipf(1.1) expert popularity, pairs sorted by expert; alpha[g] = gA * gB_g.
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


def run(nv, A, sA, B, sB, alpha, off):
    D = nv.grouped_gemm(dev(A), dev(sA), dev(B), dev(sB), dev(alpha.astype(np.float32)), dev(off.astype(np.int32)))
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    return D.float().cpu().numpy()


def test_grouped_small_with_empty_and_large_groups(nv):
    rng = np.random.default_rng(3)
    G, N, K = 6, 264, 512
    counts = [3, 0, 150, 1, 0, 37]          # empty groups and one over a 128-row pass
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    Mt = int(off[-1])
    A = synth.random_codes(Mt, K, 1)
    sA = synth.random_scales(Mt, K, 2)
    B = np.stack([synth.random_codes(N, K, 10 + g) for g in range(G)])
    sB = np.stack([synth.random_scales(N, K, 20 + g) for g in range(G)])
    alpha = rng.uniform(0.5, 2.0, G).astype(np.float32)
    _, ref, ad = oracle.grouped_gemm(A, sA, B, sB, alpha, off, G, Mt, N, K)
    got = run(nv, A, sA, B, sB, alpha, off)
    assert not violations(got, ref, ad).any()


@pytest.mark.parametrize("K,N", [(1280, 384), (2304, 200)])
def test_grouped_every_box_count_and_ragged_k_tiles(nv, K, N):
    # Passes of 1..8 sixteen-row boxes (MMA N = 16..128, row counts off a box
    # edge too), two passes for one expert, K = 5 and 9 K tiles (not a
    # multiple of the ring depth), and N = 384 weight rows (three units per
    # expert), so the ring stages wrap around many times within one launch.
    # N = 200 ends in a 72-column weight tile: the epilogue's 16-byte pieces
    # stop inside the third lane quadrant.
    rng = np.random.default_rng(11)
    counts = [16 * b - (b % 3) for b in range(1, 9)] + [0, 200, 1, 33]
    G = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    Mt = int(off[-1])
    A = synth.random_codes(Mt, K, 31)
    sA = synth.random_scales(Mt, K, 32)
    B = np.stack([synth.random_codes(N, K, 40 + g) for g in range(G)])
    sB = np.stack([synth.random_scales(N, K, 60 + g) for g in range(G)])
    alpha = rng.uniform(0.5, 2.0, G).astype(np.float32)
    _, ref, ad = oracle.grouped_gemm(A, sA, B, sB, alpha, off, G, Mt, N, K)
    got = run(nv, A, sA, B, sB, alpha, off)
    assert not violations(got, ref, ad).any()


def test_grouped_moe_recipe_reduced(nv):
    # The MoE recipe (Zipf routing, N(0,0.02) experts, N(0,1) tokens with 1%
    # x20 outliers, per-expert global scales) at N=256, K=1024, quantised by
    # the oracle.
    N, K = 256, 1024
    r = synth.moe_routing()
    G = synth.MOE_EXPERTS
    X = synth.activations_with_outliers(synth.MOE_TOKENS, K, 1400)
    ct, st_, ga = oracle.quantize(X)
    A = ct[r.token_of_row]
    sA = st_[r.token_of_row]
    B = np.empty((G, N, K // 2), np.uint8)
    sB = np.empty((G, N, K // 16), np.uint8)
    alpha = np.empty(G, np.float32)
    for g in range(G):
        cb, sb, gb = oracle.quantize(synth.normal(N, K, 5000 + g, std=0.02))
        B[g], sB[g] = cb, sb
        alpha[g] = np.float32(ga) * np.float32(gb)
    Mt = int(r.row_offsets[-1])
    _, ref, ad = oracle.grouped_gemm(A, sA, B, sB, alpha, r.row_offsets, G, Mt, N, K)
    got = run(nv, A, sA, B, sB, alpha, r.row_offsets)
    bad = violations(got, ref, ad)
    assert not bad.any(), f"{bad.sum()} outside the bound"


def test_grouped_full_size_sampled(nv):
    # 256 experts x [2048 x 6144], 4096 routed rows: random codes and scales at
    # full size (the quantiser is pinned separately), sampled outputs checked.
    G, N, K = synth.MOE_EXPERTS, synth.MOE_N, synth.HIDDEN_K
    r = synth.moe_routing()
    Mt = int(r.row_offsets[-1])
    A = synth.random_codes(Mt, K, 7)
    sA = synth.random_scales(Mt, K, 8, lo=0x30, hi=0x40)
    B = synth.random_codes(G * N, K, 9).reshape(G, N, K // 2)
    sB = synth.random_scales(G * N, K, 10, lo=0x28, hi=0x38).reshape(G, N, K // 16)
    alpha = np.full(G, 1.0e-3, np.float32) * np.arange(1, G + 1, dtype=np.float32)
    got = run(nv, A, sA, B, sB, alpha, r.row_offsets)
    rng = np.random.default_rng(11)
    rows = np.concatenate([rng.integers(0, Mt, 1500), [0, Mt - 1]])
    cols = np.concatenate([rng.integers(0, N, 1500), [N - 1, 0]])
    group = np.searchsorted(r.row_offsets, rows, side="right") - 1
    for g in np.unique(group):
        sel = group == g
        _, ref, ad = oracle.gemm_sampled(A, sA, B[g], sB[g], float(alpha[g]), Mt, N, K, rows[sel], cols[sel])
        assert not violations(got[rows[sel], cols[sel]], ref, ad).any(), f"expert {g}"


def test_grouped_repeated_launches_on_two_streams(nv):
    # Work units are handed out at run time from a per-stream counter that the
    # last CTA of each launch zeroes: back-to-back launches on one stream and
    # launches on a second stream must each cover every unit exactly once.
    rng = np.random.default_rng(5)
    G, N, K = 9, 392, 768
    counts = [0, 260, 5, 0, 129, 1, 0, 77, 16]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    Mt = int(off[-1])
    A = synth.random_codes(Mt, K, 31)
    sA = synth.random_scales(Mt, K, 32)
    B = np.stack([synth.random_codes(N, K, 40 + g) for g in range(G)])
    sB = np.stack([synth.random_scales(N, K, 50 + g) for g in range(G)])
    alpha = rng.uniform(0.5, 2.0, G).astype(np.float32)
    _, ref, ad = oracle.grouped_gemm(A, sA, B, sB, alpha, off, G, Mt, N, K)
    args = [dev(A), dev(sA), dev(B), dev(sB), dev(alpha), dev(off)]
    other = torch.cuda.Stream()
    outs = []
    for s in (None, None, None, other, other):
        D = torch.full((Mt, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        if s is other:
            other.wait_stream(torch.cuda.current_stream())   # inputs and the NaN fill come first
            with torch.cuda.stream(other):
                nv.grouped_gemm(*args, out=D, stream=other)
        else:
            nv.grouped_gemm(*args, out=D)
        outs.append(D)
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    first = outs[0].view(torch.int16)
    for D in outs:
        assert torch.equal(D.view(torch.int16), first)     # one CTA computes each unit: bit-identical
    assert not violations(outs[0].float().cpu().numpy(), ref, ad).any()


def test_grouped_more_experts_than_the_order_table(nv):
    # More than 2048 experts: units are handed out in expert order instead of
    # heavy experts first, skipping the empty ones at run time.
    rng = np.random.default_rng(6)
    G, N, K = 2100, 128, 256
    counts = np.zeros(G, np.int64)
    hot = rng.choice(G, 40, replace=False)
    counts[hot] = rng.integers(1, 40, 40)
    counts[hot[0]] = 200                     # one expert over a 128-row pass
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    Mt = int(off[-1])
    A = synth.random_codes(Mt, K, 61)
    sA = synth.random_scales(Mt, K, 62)
    B = synth.random_codes(G * N, K, 63).reshape(G, N, K // 2)
    sB = synth.random_scales(G * N, K, 64).reshape(G, N, K // 16)
    alpha = rng.uniform(0.5, 2.0, G).astype(np.float32)
    _, ref, ad = oracle.grouped_gemm(A, sA, B, sB, alpha, off, G, Mt, N, K)
    got = run(nv, A, sA, B, sB, alpha, off)
    assert not violations(got, ref, ad).any()


def test_grouped_full_size_recipe_sampled_experts(nv):
    # The grouped configuration itself: 256 experts x [2048 x 6144], 512
    # tokens top-8 with Zipf(1.1) routing, tokens N(0,1) with 1% x20 outliers
    # (one global scale), and for the checked experts weights N(0, 0.02)
    # quantized by the oracle with one global scale per expert (alpha[e] =
    # gA * gB_e).  Quantizing all 256 experts on the host would take minutes,
    # so ten experts follow the recipe -- the busiest, the least busy active
    # ones and a random draw -- and the rest hold random codes (their rows are
    # computed but not checked).  Every row of a checked expert is checked at
    # sampled columns and at the first and last column.
    G, N, K = synth.MOE_EXPERTS, synth.MOE_N, synth.HIDDEN_K
    r = synth.moe_routing()
    Mt = int(r.row_offsets[-1])
    counts = np.diff(r.row_offsets)
    X = synth.activations_with_outliers(synth.MOE_TOKENS, K, 1400)
    ct, st_, ga = oracle.quantize(X)
    A, sA = ct[r.token_of_row], st_[r.token_of_row]
    rng = np.random.default_rng(1401)
    active = np.flatnonzero(counts)
    by_load = active[np.argsort(counts[active], kind="stable")]
    checked = sorted(set(by_load[-3:].tolist()) | set(by_load[:3].tolist()) |
                     set(rng.choice(active, 4, replace=False).tolist()))
    B = synth.random_codes(G * N, K, 1402).reshape(G, N, K // 2)
    sB = synth.random_scales(G * N, K, 1403, lo=0x28, hi=0x38).reshape(G, N, K // 16)
    alpha = np.full(G, 1.0e-3, np.float32)
    for e in checked:
        cb, sb, gb = oracle.quantize(synth.normal(N, K, 1500 + e, std=0.02))
        B[e], sB[e] = cb, sb
        alpha[e] = np.float32(ga) * np.float32(gb)
    D = nv.grouped_gemm(dev(A), dev(sA), dev(B), dev(sB), dev(alpha), dev(r.row_offsets.astype(np.int32)))
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    for e in checked:
        r0, r1 = int(r.row_offsets[e]), int(r.row_offsets[e + 1])
        rows = np.repeat(np.arange(r0, r1), 34)
        cols = np.concatenate([np.concatenate([[0, N - 1], rng.integers(0, N, 32)]) for _ in range(r1 - r0)])
        assert rows.min() >= 0 and rows.max() < Mt and cols.min() >= 0 and cols.max() < N   # before the gather
        got = D[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()].float().cpu().numpy()
        _, ref, ad = oracle.gemm_sampled(A, sA, B[e], sB[e], float(alpha[e]), Mt, N, K, rows, cols)
        assert not violations(got, ref, ad).any(), f"expert {e}"
