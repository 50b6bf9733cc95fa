// Persistent NVFP4 GEMM for large problems (many 128 x BQ output tiles).
//
// Same arithmetic and data path as nvfp4_gemm_kernel (TMA ring, scale tiles
// written into TMEM by four writer warps, tcgen05.mma.kind::mxf4nvf4.block16
// with fp32 accumulation in TMEM, alpha + BF16 epilogue), but one CTA per SM
// walks a list of tiles, so the ring keeps streaming the next tile's operands
// while the current tile's epilogue drains the accumulator.  The saturation
// shapes of "Peeling the Kernel Onion" (section "The Benchmark Design") are
// the intended use: 512 to 8192 tiles per launch.
//
// Tile order: groups of kGroupM row blocks; inside a group the row block
// varies fastest, so the CTAs running at one time share a few row blocks of A
// and a band of column blocks of B in L2.
//
// Warp roles (320 threads): warp 0 TMA producer; warp 1 TMEM allocator and
// MMA issuer; warps 2..5 epilogue (TMEM lane quadrant w % 4); warps 6..9
// scale writers (TMEM lane quadrant w % 4).
// Barriers: full[s], empty[s] (ring; an MMA commit on empty also frees the
// TMEM scale buffer of that K tile), sf_ready[b] (4 writer arrivals),
// acc_full (MMA commit after a tile's last K tile), acc_empty (4 epilogue
// arrivals once the accumulator has been read).  Every wait is bounded.
#pragma once

#include "gemm_kernel.cuh"

namespace nvfp4 {

constexpr int kPersistThreads = 320;
constexpr int kGroupM = 8;

struct PersistParams {
    __nv_bfloat16* D;
    float alpha;
    int M, N, K;           // D is M x N
    int k_tiles;           // K / 256
    int tiles_m, tiles_n;  // 128-row and BQ-column tiles
};

template <int BQ>
struct PersistConfig {
    static constexpr int P_BYTES = kBM * kStageKBytes;
    static constexpr int Q_BYTES = BQ * kStageKBytes;
    static constexpr int Q_BLOCKS = BQ > 128 ? BQ / 128 : 1;
    static constexpr int SFP_BYTES = 4 * kAtomBytes;
    static constexpr int SFQ_BYTES = 4 * kAtomBytes * Q_BLOCKS;
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;
    static constexpr int STAGES_FIT = (kSmemLimit - 2048) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 1024;
    static constexpr int SF_BASE = BQ;
    static constexpr int SF_STRIDE = 16 + 16 * Q_BLOCKS;
    static constexpr int TMEM_COLS = 512;
    static_assert(SF_BASE + kScaleBuffers * SF_STRIDE <= TMEM_COLS, "TMEM columns");
    static_assert(STAGES >= kScaleBuffers, "scale buffers are released through the ring barriers");
};

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
    const int per_group = kGroupM * tiles_n;
    const int group = t / per_group;
    const int first_m = group * kGroupM;
    const int rows_in_group = min(kGroupM, tiles_m - first_m);
    const int r = t - group * per_group;
    tm = first_m + r % rows_in_group;
    tn = r / rows_in_group;
}

template <int BQ>
__global__ void __launch_bounds__(kPersistThreads, 1)
    nvfp4_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                 const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                                 const PersistParams prm) {
    using C = PersistConfig<BQ>;
    constexpr int S = C::STAGES;
    constexpr int NB = kScaleBuffers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
    // bars: [0,S) full, [S,2S) empty, [2S,2S+NB) sf_ready, [2S+NB] acc_full, [2S+NB+1] acc_empty
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + NB + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
    auto sf_ready_bar = [&](int b) { return bar_base + 8u * (2 * S + b); };
    const uint32_t acc_full_bar = bar_base + 8u * (2 * S + NB);
    const uint32_t acc_empty_bar = bar_base + 8u * (2 * S + NB + 1);
    const int tiles = prm.tiles_m * prm.tiles_n;
    const int KT = prm.k_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < NB; ++b) mbar_init(sf_ready_bar(b), 4);
        mbar_init(acc_full_bar, 1);
        mbar_init(acc_empty_bar, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        prefetch_tensor_map(&tmA);
        prefetch_tensor_map(&tmB);
        prefetch_tensor_map(&tmSA);
        prefetch_tensor_map(&tmSB);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_launch_dependents();
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            int it = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, prm.tiles_m, prm.tiles_n, tm, tn);
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(empty_bar(s), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) goto producer_done;
                    const uint32_t st = smem_base + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(full_bar(s), C::P_BYTES + C::Q_BYTES + 16 * kBM + 16 * BQ);
                    tma_load_2d(st, &tmA, full_bar(s), kt * kStageKBytes, tm * kBM, pol_a);
                    tma_load_2d(st + C::P_BYTES, &tmB, full_bar(s), kt * kStageKBytes, tn * BQ, pol_b);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSA, full_bar(s), kt * 16, tm * kBM, pol_a);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSB, full_bar(s), kt * 16, tn * BQ,
                                pol_b);
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(kBM, BQ);
            int it = 0, tt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tt) {
                // the epilogue must have read the previous tile's accumulator
                if (!mbar_wait(acc_empty_bar, ((uint32_t)tt & 1u) ^ 1u, abort_flag)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S, b = it % NB;
                    if (!mbar_wait(sf_ready_bar(b), (uint32_t)(it / NB) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_base + s * C::STAGE_BYTES;
                    const uint32_t sf = tmem + C::SF_BASE + b * C::SF_STRIDE;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_nvf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::P_BYTES + 32 * j),
                                    idesc, sf + 4 * j, sf + 16 + 4 * C::Q_BLOCKS * j, (kt > 0 || j > 0) ? 1u : 0u);
                    tc_commit(empty_bar(s));
                }
                tc_commit(acc_full_bar);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---- scale writers (TMEM lane quadrant warp % 4)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        const int total = ((tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * KT;
        for (int it = 0; it < total;) {
            int got = 1, cnt = 1;
            if (lane == 0) {
                const int s0 = it % S, j0 = it - NB;
                got = mbar_wait(full_bar(s0), (uint32_t)(it / S) & 1u, abort_flag) &&
                      (j0 < 0 || mbar_wait(empty_bar(j0 % S), (uint32_t)(j0 / S) & 1u, abort_flag));
                while (got && cnt < NB / 2 && it + cnt < total) {
                    const int i1 = it + cnt, s1 = i1 % S, j1 = i1 - NB;
                    if (!mbar_test(full_bar(s1), (uint32_t)(i1 / S) & 1u) ||
                        (j1 >= 0 && !mbar_test(empty_bar(j1 % S), (uint32_t)(j1 / S) & 1u)))
                        break;
                    ++cnt;
                }
            }
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            cnt = __shfl_sync(0xffffffffu, cnt, 0);
            for (int u = 0; u < cnt; ++u) {
                const int iu = it + u;
                const uint32_t st = smem_base + (iu % S) * C::STAGE_BYTES;
                const uint32_t sf = t_quad + C::SF_BASE + (iu % NB) * C::SF_STRIDE;
                uint32_t wp[16];
                gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES, lane, wp);
                tmem_store_16(sf, wp);
                if (C::Q_BLOCKS == 1) {
                    uint32_t wq[16];
                    gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq);
                    tmem_store_16(sf + 16, wq);
                } else {
                    uint32_t wq0[16], wq1[16], wq[32];
                    gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq0);
                    gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + 4 * kAtomBytes, lane, wq1);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int r1 = 0; r1 < 4; ++r1) {
                            wq[8 * j + r1] = wq0[4 * j + r1];
                            wq[8 * j + 4 + r1] = wq1[4 * j + r1];
                        }
                    tmem_store_32(sf + 16, wq);
                }
            }
            tmem_wait_store();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int u = 0; u < cnt; ++u) mbar_arrive(sf_ready_bar((it + u) % NB));
            it += cnt;
        }
    } else {
        // ---- epilogue (warps 2..5, TMEM lane quadrant warp % 4 = tile row)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        int tt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tt) {
            int tm, tn;
            tile_coords(t, prm.tiles_m, prm.tiles_n, tm, tn);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(acc_full_bar, (uint32_t)tt & 1u, abort_flag) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0) || *abort_flag) break;
            tc_fence_after();
            const int p = tm * kBM + quad * 32 + lane;
            const int q_base = tn * BQ;
            __nv_bfloat16* drow = prm.D + (size_t)p * prm.N;
#pragma unroll 1
            for (int c0 = 0; c0 < BQ; c0 += 32) {
                uint32_t r0[16], r1[16];
                tmem_load_16(t_quad + c0, r0);
                tmem_load_16(t_quad + c0 + 16, r1);
                tmem_wait_load();
                if (c0 + 32 >= BQ) {
                    // last chunk read: hand the accumulator back to the MMA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty_bar);
                }
                if (p < prm.M) {
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int q = q_base + c0 + 8 * h;
                        if (q < prm.N) {   // N is a multiple of 8
                            const uint32_t* r = h < 2 ? r0 + 8 * h : r1 + 8 * (h - 2);
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(r[0]) * prm.alpha, __uint_as_float(r[1]) * prm.alpha);
                            w.y = pack_bf16x2(__uint_as_float(r[2]) * prm.alpha, __uint_as_float(r[3]) * prm.alpha);
                            w.z = pack_bf16x2(__uint_as_float(r[4]) * prm.alpha, __uint_as_float(r[5]) * prm.alpha);
                            w.w = pack_bf16x2(__uint_as_float(r[6]) * prm.alpha, __uint_as_float(r[7]) * prm.alpha);
                            *reinterpret_cast<uint4*>(drow + q) = w;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace nvfp4
