// Persistent NVFP4 GEMM on CTA pairs: one tcgen05.mma.cta_group::2 per K step
// computes a 256 x 256 block of D on two SMs.
//
// The arithmetic is that of the other GEMM kernels (E2M1 products scaled by
// one UE4M3 factor per 16 elements of K on each side, fp32 accumulation in
// TMEM, alpha and BF16 rounding in the epilogue); what changes is how the
// tensor cores are fed.  A thread-block cluster of two CTAs shares each MMA:
//   * CTA r (r = 0, 1) holds rows 128r..128r+127 of the A tile and rows
//     128r..128r+127 of the B tile in its shared memory;
//   * each CTA's TMEM holds the scales of its own 128 A rows and of all 256
//     B rows (the layout of the single-CTA kernel with a 256-row B tile);
//   * CTA 0 issues the MMA (M = 256, N = 256); D rows 128r.. land in CTA r's
//     TMEM, so each CTA runs the epilogue of its own half.
// Per SM this halves the B tile each K tile moves through shared memory and
// L2 against the single-CTA 128 x 256 tile, for the same MMA work.
//
// Every TMA load is a plain load of this CTA's own operand rows into its own
// shared memory, completing on its own barrier.  The pair synchronises
// through mbarriers only:
//   full[s]        local: TMA bytes of stage s landed (expect_tx);
//   empty[s]       both CTAs: arrived by CTA 0's MMA commit (multicast to the
//                  pair) when the MMAs reading stage s (and the TMEM scale
//                  buffer of that K tile) have completed;
//   sf_ready[b]    CTA 0 only: 8 arrivals, the four scale-writer warps of
//                  each CTA, after their stage's data landed and its scales
//                  reached TMEM (so CTA 0 learns that CTA 1's stage is full
//                  through these arrivals);
//   acc_full       both CTAs: MMA commit after the last K tile of a tile;
//   acc_empty      CTA 0 only: 8 arrivals, the epilogue warps of both CTAs,
//                  once the accumulator has been read.
// All waits are bounded (a timeout sets the device error word and the CTA's
// abort flag).  Warp roles are those of the single-CTA persistent kernel:
// warp 0 TMA producer, warp 1 TMEM allocator (both CTAs) and MMA issuer
// (CTA 0), warps 2..5 epilogue, warps 6..9 scale writers.
//
// Used for the compute-bound shapes of "Peeling the Kernel Onion" (section
// "The Benchmark Design"): K a multiple of 256, scales in row-major
// [rows, K/16] order with 16-byte aligned rows.
#pragma once

#include "persistent_kernel.cuh"

namespace nvfp4 {

constexpr int kPairBM = 256;  // D rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;  // D columns per pair tile

struct PairConfig {
    static constexpr int A_BYTES = 128 * kStageKBytes;   // this CTA's 128 A rows
    static constexpr int B_BYTES = 128 * kStageKBytes;   // this CTA's 128 B rows
    static constexpr int SFA_BYTES = 128 * 16;           // scales of the 128 A rows
    static constexpr int SFB_BYTES = kPairBN * 16;       // scales of all 256 B rows
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES_FIT = (kSmemLimit - 2048) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 1024;
    static constexpr int SF_BASE = kPairBN;   // accumulator: columns [0, 256)
    static constexpr int SF_STRIDE = 16 + 32; // SFA 4 columns x 4 steps, SFB 8 x 4
    static constexpr int TMEM_COLS = 512;
    static_assert(SF_BASE + kScaleBuffers * SF_STRIDE <= TMEM_COLS, "TMEM columns");
    static_assert(STAGES >= kScaleBuffers, "scale buffers are released through the ring barriers");
};

__device__ __forceinline__ uint32_t cluster_cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// prm.tiles_m / tiles_n count 256 x 256 pair tiles.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPersistThreads, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                           const PersistParams prm) {
    using C = PairConfig;
    constexpr int S = C::STAGES;
    constexpr int NB = kScaleBuffers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
    // bars: [0,S) full, [S,2S) empty, [2S,2S+NB) sf_ready, [2S+NB] acc_full, [2S+NB+1] acc_empty
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + NB + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_cta_rank();
    const int pair = (int)cluster_id_x(), pairs = (int)cluster_count_x();
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
        for (int b = 0; b < NB; ++b) mbar_init(sf_ready_bar(b), 8);
        mbar_init(acc_full_bar, 1);
        mbar_init(acc_empty_bar, 8);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tensor_map(&tmA);
        prefetch_tensor_map(&tmB);
        prefetch_tensor_map(&tmSA);
        prefetch_tensor_map(&tmSB);
    }
    // both CTAs' barriers are initialised before either CTA arrives remotely
    cluster_sync();
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish_pair();
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
            for (int t = pair; t < tiles; t += pairs) {
                int tm, tn;
                tile_coords(t, prm.tiles_m, prm.tiles_n, tm, tn);
                const int a_row = tm * kPairBM + (int)rank * 128;
                const int b_row = tn * kPairBN + (int)rank * 128;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(empty_bar(s), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) goto producer_done;
                    const uint32_t st = smem_base + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
                    tma_load_2d(st, &tmA, full_bar(s), kt * kStageKBytes, a_row, pol_a);
                    tma_load_2d(st + C::A_BYTES, &tmB, full_bar(s), kt * kStageKBytes, b_row, pol_b);
                    tma_load_2d(st + C::A_BYTES + C::B_BYTES, &tmSA, full_bar(s), kt * 16, a_row, pol_a);
                    tma_load_2d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSB, full_bar(s), kt * 16,
                                tn * kPairBN, pol_b);
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(kPairBM, kPairBN);
            int it = 0, tt = 0;
            bool ok = true;
            for (int t = pair; ok && t < tiles; t += pairs, ++tt) {
                // both CTAs' epilogues must have read the previous accumulator
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
                        tc_mma_nvf4_pair(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::A_BYTES + 32 * j),
                                         idesc, sf + 4 * j, sf + 16 + 8 * j, (kt > 0 || j > 0) ? 1u : 0u);
                    tc_commit_pair(empty_bar(s));
                }
                if (ok) tc_commit_pair(acc_full_bar);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---- scale writers (TMEM lane quadrant warp % 4)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        const int total = ((tiles - pair + pairs - 1) / pairs) * KT;
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
                const uint32_t st = smem_base + (iu % S) * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
                const uint32_t sf = t_quad + C::SF_BASE + (iu % NB) * C::SF_STRIDE;
                uint32_t wa[16];
                gather_scale_words<true>(st, lane, wa);
                tmem_store_16(sf, wa);
                // B rows 0..127 and 128..255: step j uses columns 8j + 4*half + r1
                uint32_t wb0[16], wb1[16], wb[32];
                gather_scale_words<true>(st + C::SFA_BYTES, lane, wb0);
                gather_scale_words<true>(st + C::SFA_BYTES + 128 * 16, lane, wb1);
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int r1 = 0; r1 < 4; ++r1) {
                        wb[8 * j + r1] = wb0[4 * j + r1];
                        wb[8 * j + 4 + r1] = wb1[4 * j + r1];
                    }
                tmem_store_32(sf + 16, wb);
            }
            tmem_wait_store();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int u = 0; u < cnt; ++u) mbar_arrive_remote(sf_ready_bar((it + u) % NB), 0);
            it += cnt;
        }
    } else {
        // ---- epilogue (warps 2..5, TMEM lane quadrant warp % 4 = row of this CTA's half)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        int tt = 0;
        for (int t = pair; t < tiles; t += pairs, ++tt) {
            int tm, tn;
            tile_coords(t, prm.tiles_m, prm.tiles_n, tm, tn);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(acc_full_bar, (uint32_t)tt & 1u, abort_flag) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0) || *abort_flag) break;
            tc_fence_after();
            const int p = tm * kPairBM + (int)rank * 128 + quad * 32 + lane;
            const int q_base = tn * kPairBN;
            __nv_bfloat16* drow = prm.D + (size_t)p * prm.N;
#pragma unroll 1
            for (int c0 = 0; c0 < kPairBN; c0 += 32) {
                uint32_t r0[16], r1[16];
                tmem_load_16(t_quad + c0, r0);
                tmem_load_16(t_quad + c0 + 16, r1);
                tmem_wait_load();
                if (c0 + 32 >= kPairBN) {
                    // last chunk read: hand the accumulator back to the MMA issuer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(acc_empty_bar, 0);
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

    // Neither CTA frees TMEM or exits while the other may still use it: the
    // MMA of CTA 0 reads CTA 1's shared memory and TMEM, and CTA 1's
    // epilogue and writers arrive on CTA 0's barriers.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace nvfp4
