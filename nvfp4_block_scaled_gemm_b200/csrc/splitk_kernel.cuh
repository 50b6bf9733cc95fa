// Split-K NVFP4 GEMM for few to a few hundred token rows, built for chains of
// dependent launches.
//
// With few token rows the GEMM streams the weight matrix once and does little
// else: "Peeling the Kernel Onion", section "The Critical Connection to Real
// Inference" (about 16 rows per expert), and "The SM120 FP4 Kernel Disaster",
// section "Finding 4: Memory Bandwidth Is the Real Wall".  A 3 MB weight
// matrix is half a microsecond of HBM time, so what bounds such a GEMM inside
// a layer chain is the latency of its serial steps, not bandwidth.  This
// kernel arranges the work so that as little as possible sits after the
// point where it must wait for the previous kernel in the stream:
//
//   * The weight matrix is cut into 128-row tiles and K into slices, one
//     (tile, slice) per CTA, the slices of a tile forming one thread-block
//     cluster of up to 16 CTAs; a launch has about one to two CTAs per SM, each
//     streaming a disjoint part of the weights.
//   * Every CTA is small enough (at most ~110 KB of shared memory and 256 TMEM
//     columns) that the CTAs of the next launch in the stream fit on the SMs
//     beside it, so with programmatic dependent launch they start while this
//     one still runs.
//   * When the caller declares the weights constant, the CTA's weight tiles
//     and weight scales are requested before the wait on the previous grid,
//     and the weight scales are moved into TMEM before it as well.  After the
//     wait only the activation tiles (a few KB), their scales, the MMAs and
//     the split-K reduction remain.
//   * The split-K partials meet in L2: each CTA writes its fp32 128 x BQ
//     partial to a global workspace with coalesced 16-byte stores, one
//     cluster barrier (release/acquire at cluster scope) makes them visible,
//     and each rank sums its 128 / splits rows over the ranks in rank order
//     (deterministic) and writes them with 16-byte stores.
//
// Orientation.  SWAP (token rows <= 64): the weights are the 128-row MMA
// operand P and the token rows the BQ-wide operand Q (BQ = 16, 32, 64); the
// output tile is the transpose, D[m][n] with n along P.  Otherwise the token
// rows are P (128-row tiles) and the weights Q (BQ = 64 or 128 rows).
//
// Warp roles (192 threads): warp 0 TMA producer; warp 1 TMEM allocator and
// MMA warp: per K tile its 32 lanes turn each operand's row-major scale tile
// (row r's 16 bytes = the 4 K steps' words) in place into four 512-byte
// atoms (atom j, line L = the step-j words of rows L, L+32, L+64, L+96), and
// its lane 0 copies them into TMEM with tcgen05.cp and issues the four
// tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 (K = 64 each,
// fp32 accumulation in TMEM) right behind them, in order on the tensor pipe,
// so no other warp sits between a K tile's arrival and its MMAs; warps 2..5
// the epilogue.
//
// Ring.  `stages` stage buffers, each holding one 256-element K tile of both
// operands and their scales, with its own TMEM scale buffer.  For the shapes
// this kernel is chosen for, a CTA's whole K slice usually fits, so nothing
// is reused.  Barriers per stage: wfull (weight tile and scales landed),
// tfull (token tile and scales landed), empty (the MMA commit: stage and
// TMEM scale buffer free); plus accum (all MMAs done).  Every wait is
// bounded.
#pragma once

#include "gemm_kernel.cuh"

namespace nvfp4 {

constexpr int kSkThreads = 192;
constexpr int kSkMaxStages = 10;

template <int BQ>
struct SkConfig {
    static_assert(BQ == 16 || BQ == 32 || BQ == 64 || BQ == 128, "BQ");
    static constexpr int P_BYTES = kBM * kStageKBytes;      // 16 KB: 128 rows x 256 values
    static constexpr int Q_BYTES = BQ * kStageKBytes;
    static constexpr int SFP_BYTES = 2048;                   // 128 rows x 16 scale bytes
    static constexpr int SFQ_BYTES = 2048;                   // BQ <= 128 rows x 16 scale bytes
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;
    static constexpr int ACC_COLS = BQ < 32 ? 32 : BQ;       // fp32 accumulator columns in TMEM
    static constexpr int SF_STRIDE = 32;                     // TMEM scale columns per stage: P 16, Q 16
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the 128-byte swizzle");
};

struct SkParams {
    __nv_bfloat16* D;
    float alpha;
    int rows_p, rows_q;    // valid rows of P and Q
    int ldd;               // row stride of D in elements (= N)
    int k_tiles;           // K / 256
    int tiles_q;           // blockIdx.y = tq + tiles_q * tp
    int stages;            // ring depth, 1 .. kSkMaxStages
    int prefetch_w;        // the weights are constant: load them before waiting on the previous grid
    uint32_t tmem_cols;    // power of two >= 32
    float4* ws;            // split-K partials: [tile][rank][BQ/4][128 rows] float4 (global workspace)
};

// Bytes of dynamic shared memory a launch needs: [ring][barriers][TMEM
// address, abort flag], 1024-byte aligned (the split-K partials meet in
// global memory, so a split needs no more).
template <int BQ>
__host__ __device__ constexpr int sk_smem_bytes(int stages, [[maybe_unused]] bool split) {
    return 1024 + stages * SkConfig<BQ>::STAGE_BYTES + 8 * (4 * kSkMaxStages + 2) + 16;
}

template <int BQ, bool SWAP>
__global__ void __launch_bounds__(kSkThreads, 2)
    nvfp4_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                             const __grid_constant__ CUtensorMap tmSP, const __grid_constant__ CUtensorMap tmSQ,
                             const SkParams prm) {
    using C = SkConfig<BQ>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = prm.stages;
    const int splits = gridDim.x;
    // [ring][barriers][tmem slot, abort flag]
    const int ring_bytes = S * C::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ring_bytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * kSkMaxStages + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int tq = blockIdx.y % prm.tiles_q, tp = blockIdx.y / prm.tiles_q;
    const int kt_begin = (int)((long long)split * prm.k_tiles / splits);
    const int kt_end = (int)((long long)(split + 1) * prm.k_tiles / splits);
    const int nkt = kt_end - kt_begin;
    const int q_row0 = tq * BQ;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto wfull_bar = [&](int s) { return bar_base + 8u * s; };
    auto tfull_bar = [&](int s) { return bar_base + 8u * (kSkMaxStages + s); };
    auto empty_bar = [&](int s) { return bar_base + 8u * (2 * kSkMaxStages + s); };
    const uint32_t accum_bar = bar_base + 8u * (4 * kSkMaxStages);
    auto stage_addr = [&](int s) { return smem_base + (uint32_t)(s * C::STAGE_BYTES); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(wfull_bar(s), 1);
            mbar_init(tfull_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(accum_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), prm.tmem_cols);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        prefetch_tensor_map(&tmP);
        prefetch_tensor_map(&tmQ);
        prefetch_tensor_map(&tmSP);
        prefetch_tensor_map(&tmSQ);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_launch_dependents();

    // Which operand holds the weights: P when swapped, Q otherwise.  Byte
    // offsets inside a stage and TMEM column offsets inside a scale buffer.
    constexpr uint32_t kOffQ = C::P_BYTES, kOffSP = C::P_BYTES + C::Q_BYTES, kOffSQ = kOffSP + C::SFP_BYTES;
    constexpr uint32_t kWScaleOff = SWAP ? kOffSP : kOffSQ, kTScaleOff = SWAP ? kOffSQ : kOffSP;
    constexpr uint32_t kWCol = SWAP ? 0 : 16, kTCol = SWAP ? 16 : 0;
    constexpr uint32_t kWTx = SWAP ? C::P_BYTES + 16 * kBM : C::Q_BYTES + 16 * BQ;   // weight tile + scale tile bytes
    constexpr uint32_t kTTx = SWAP ? C::Q_BYTES + 16 * BQ : C::P_BYTES + 16 * kBM;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();   // weights: read by this CTA only
            const uint64_t pol_t = policy_evict_last();    // token rows: shared by every weight tile
            auto load_w = [&](int s, int kt) {
                const uint32_t st = stage_addr(s);
                mbar_arrive_expect_tx(wfull_bar(s), kWTx);
                if (SWAP) {
                    tma_load_2d(st, &tmP, wfull_bar(s), kt * kStageKBytes, tp * kBM, pol_w);
                    tma_load_2d(st + kOffSP, &tmSP, wfull_bar(s), kt * 16, tp * kBM, pol_w);
                } else {
                    tma_load_2d(st + kOffQ, &tmQ, wfull_bar(s), kt * kStageKBytes, q_row0, pol_w);
                    tma_load_2d(st + kOffSQ, &tmSQ, wfull_bar(s), kt * 16, q_row0, pol_w);
                }
            };
            auto load_t = [&](int s, int kt) {
                const uint32_t st = stage_addr(s);
                mbar_arrive_expect_tx(tfull_bar(s), kTTx);
                if (SWAP) {
                    tma_load_2d(st + kOffQ, &tmQ, tfull_bar(s), kt * kStageKBytes, q_row0, pol_t);
                    tma_load_2d(st + kOffSQ, &tmSQ, tfull_bar(s), kt * 16, q_row0, pol_t);
                } else {
                    tma_load_2d(st, &tmP, tfull_bar(s), kt * kStageKBytes, tp * kBM, pol_t);
                    tma_load_2d(st + kOffSP, &tmSP, tfull_bar(s), kt * 16, tp * kBM, pol_t);
                }
            };
            const int pre = prm.prefetch_w ? min(nkt, S) : 0;
            for (int i = 0; i < pre; ++i) load_w(i, kt_begin + i);
            grid_dependency_wait();
            for (int i = 0; i < nkt; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(empty_bar(s), (uint32_t)((i / S) - 1) & 1u, abort_flag)) break;
                if (i >= pre) load_w(s, kt_begin + i);
                load_t(s, kt_begin + i);
            }
        }
    } else if (warp == 1) {
        // ---- MMA warp: scale atoms, tcgen05.cp, MMAs
        // Wait (lane 0, bounded) for a barrier phase; the warp follows.
        auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
            int ok = 1;
            if (lane == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
            return __shfl_sync(0xffffffffu, ok, 0) != 0;
        };
        auto sf_col = [&](int s) { return tmem + (uint32_t)(C::ACC_COLS + s * C::SF_STRIDE); };
        // Row-major scale tile at `base` -> four atoms in place (the warp's
        // loads first, then its stores), not yet fenced for the tensor core.
        auto build_atoms = [&](uint32_t base) {
            uint32_t w[16];
            gather_scale_words<true>(base, lane, w);   // w[4j + r1] = step j of row lane + 32 r1
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + 512u * j + 16u * lane),
                             "r"(w[4 * j]), "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                             : "memory");
        };
        auto copy_atoms = [&](uint32_t base, uint32_t col) {   // lane 0, after the fence
#pragma unroll
            for (int j = 0; j < 4; ++j) tc_copy_32x128b_x4(col + 4 * j, desc_scale_atom(base + 512u * j));
        };
        auto issue_mmas = [&](int i, int s) {   // lane 0
            const uint32_t st = stage_addr(s);
            const uint32_t sf = sf_col(s);
            constexpr uint32_t idesc = idesc_nvf4(kBM, BQ);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                tc_mma_nvf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + kOffQ + 32 * j), idesc,
                            sf + 4 * j, sf + 16 + 4 * j, (i > 0 || j > 0) ? 1u : 0u);
            tc_commit(empty_bar(s));   // frees the stage and its TMEM scale buffer
        };
        auto fence_and_sync = [&]() {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        };
        const int first = min(nkt, S);
        bool ok = true;
        if (!prm.prefetch_w) grid_dependency_wait();
        // The weights' scales of the first ring pass (before the grid
        // dependency when the weights were requested early).
        for (int i = 0; i < first && ok; ++i) {
            ok = warp_wait(wfull_bar(i), 0);
            if (ok) build_atoms(stage_addr(i) + kWScaleOff);
        }
        if (ok) {
            fence_and_sync();
            if (lane == 0) {
                tc_fence_after();
                for (int i = 0; i < first; ++i) copy_atoms(stage_addr(i) + kWScaleOff, sf_col(i) + kWCol);
            }
        }
        if (prm.prefetch_w) grid_dependency_wait();
        // First pass: every resident K tile's token scales once they have
        // all landed, one fence, then all copies and MMAs back to back.
        for (int i = 0; i < first && ok; ++i) {
            ok = warp_wait(tfull_bar(i), 0);
            if (ok) build_atoms(stage_addr(i) + kTScaleOff);
        }
        if (ok) {
            fence_and_sync();
            if (lane == 0) {
                tc_fence_after();
                for (int i = 0; i < first; ++i) {
                    copy_atoms(stage_addr(i) + kTScaleOff, sf_col(i) + kTCol);
                    issue_mmas(i, i);
                }
            }
            __syncwarp();
        }
        // Later K tiles (ring reuse): one at a time.
        for (int i = first; i < nkt && ok; ++i) {
            const int s = i % S;
            const uint32_t ph = (uint32_t)(i / S) & 1u;
            ok = warp_wait(wfull_bar(s), ph);
            if (!ok) break;
            build_atoms(stage_addr(s) + kWScaleOff);
            ok = warp_wait(tfull_bar(s), ph);
            if (!ok) break;
            build_atoms(stage_addr(s) + kTScaleOff);
            fence_and_sync();
            if (lane == 0) {
                tc_fence_after();
                copy_atoms(stage_addr(s) + kWScaleOff, sf_col(s) + kWCol);
                copy_atoms(stage_addr(s) + kTScaleOff, sf_col(s) + kTCol);
                issue_mmas(i, s);
            }
            __syncwarp();
        }
        if (lane == 0) tc_commit(accum_bar);   // always (also after an abort), once every MMA above is done
        __syncwarp();
    } else {
        const int quad = warp & 3;   // TMEM lane quadrant of this warp
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        grid_dependency_wait();   // before the D stores and the split-K partials
        int acc_ok = 1;
        if (lane == 0) acc_ok = mbar_wait(accum_bar, 0, abort_flag) ? 1 : 0;
        acc_ok = __shfl_sync(0xffffffffu, acc_ok, 0);
        tc_fence_after();
        if (splits == 1 && acc_ok && !*abort_flag) {
            // ---- direct epilogue: TMEM -> registers -> alpha, BF16 -> global
            const int p = tp * kBM + quad * 32 + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < BQ; c0 += 16) {
                uint32_t r[16];
                tmem_load_16(t_quad + c0, r);
                tmem_wait_load();
                float v[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]) * prm.alpha;
                if (!SWAP) {
                    // D[p][q0 .. q0+15]: two 16-byte stores
                    const int q0 = q_row0 + c0;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (p < prm.rows_p && q0 + 8 * h < prm.rows_q) {   // rows_q (= N) is a multiple of 8
                            uint4 w;
                            w.x = pack_bf16x2(v[8 * h + 0], v[8 * h + 1]);
                            w.y = pack_bf16x2(v[8 * h + 2], v[8 * h + 3]);
                            w.z = pack_bf16x2(v[8 * h + 4], v[8 * h + 5]);
                            w.w = pack_bf16x2(v[8 * h + 6], v[8 * h + 7]);
                            *reinterpret_cast<uint4*>(prm.D + (size_t)p * prm.ldd + q0 + 8 * h) = w;
                        }
                    }
                } else {
                    // D[m][n]: the warp's 32 rows n x 16 columns m go through
                    // shared memory (the ring, free once every MMA is done)
                    // and leave as 16-byte pieces of 8 consecutive n.
                    const uint32_t tb = smem_base + (uint32_t)(quad * 1024);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const __nv_bfloat16 h = __float2bfloat16_rn(v[c]);
                        asm volatile("st.shared.b16 [%0], %1;" ::"r"(tb + (uint32_t)(c * 64 + lane * 2)),
                                     "h"(*reinterpret_cast<const uint16_t*>(&h))
                                     : "memory");
                    }
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int idx = lane + 32 * h, c = idx >> 2, part = idx & 3;
                        const int m = q_row0 + c0 + c, n = tp * kBM + quad * 32 + part * 8;
                        const uint4 val = ld_shared_v4(tb + (uint32_t)(c * 64 + part * 16));
                        if (m < prm.rows_q && n < prm.rows_p)   // rows_p (= N) is a multiple of 8
                            *reinterpret_cast<uint4*>(prm.D + (size_t)m * prm.ldd + n) = val;
                    }
                    __syncwarp();
                }
            }
        }
    }

    if (splits > 1) {
        // ---- split-K through L2: this CTA's fp32 partial tile -> the workspace
        // (coalesced 16-byte stores), one cluster barrier (release/acquire at
        // cluster scope orders them), then each rank sums its 128 / splits rows
        // of every rank's partial in rank order -- the tiled kernel's exchange.
        if (warp >= 2 && !*abort_flag) {
            const int quad = warp & 3;
            const int row = quad * 32 + lane;
            float4* dst = prm.ws + ((size_t)blockIdx.y * gridDim.x + split) * (size_t)(BQ / 4) * kBM;
            const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
            constexpr int CW = BQ < 32 ? 16 : 32;   // columns per TMEM load (one wait each)
#pragma unroll 1
            for (int c0 = 0; c0 < BQ; c0 += CW) {
                uint32_t r[32];
                if (CW == 32) {
                    tmem_load_32(t_quad + c0, r);
                } else {
                    uint32_t h[16];
                    tmem_load_16(t_quad + c0, h);
#pragma unroll
                    for (int c = 0; c < 16; ++c) r[c] = h[c];
                }
                tmem_wait_load();
#pragma unroll
                for (int c = 0; c < CW / 4; ++c)
                    dst[(c0 / 4 + c) * kBM + row] = make_float4(__uint_as_float(r[4 * c]), __uint_as_float(r[4 * c + 1]),
                                                                __uint_as_float(r[4 * c + 2]), __uint_as_float(r[4 * c + 3]));
            }
        }
        cluster_sync();   // every rank's partial is in the workspace and visible to the cluster
        if (warp >= 2 && !*abort_flag) {
            GemmParams gp{};
            gp.ws = prm.ws;
            gp.D = prm.D;
            gp.alpha = prm.alpha;
            gp.rows_p = prm.rows_p;
            gp.rows_q = prm.rows_q;
            gp.ldd = prm.ldd;
            const int t = threadIdx.x - 64;
            switch (splits) {
                case 2: reduce_from_workspace<BQ, SWAP, 2>(gp, tp, q_row0, t); break;
                case 4: reduce_from_workspace<BQ, SWAP, 4>(gp, tp, q_row0, t); break;
                case 8: reduce_from_workspace<BQ, SWAP, 8>(gp, tp, q_row0, t); break;
                default: reduce_from_workspace<BQ, SWAP, 16>(gp, tp, q_row0, t); break;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, prm.tmem_cols);
    }
}

}  // namespace nvfp4
