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
// Per SM this halves the B tile each K tile moves from L2 against the
// single-CTA 128 x 256 tile, for the same MMA work, and a stage takes less
// shared memory, so more K tiles are in flight.
//
// Scales come from the tensor-core atom layout of nvfp4_swizzle_scales (a
// per-call device pass; the ABI takes row-major scales): the scales of 128
// rows for one 256-element K tile are 2 KB of contiguous atoms, one bulk copy,
// where the row-major layout needs 128 separate 16-byte rows, a TMA request
// rate that costs about a quarter of the tensor-core rate at these shapes.
//
// Operand tiles and scale tiles travel in separate rings.  The MMA of a K
// tile waits only for its operand bytes, which both CTAs' loads complete on
// CTA 0's barrier (a non-multicast 2-CTA TMA load; each CTA loads its own
// rows), and for its scales, which the writer warps have usually put into
// TMEM long before: the scale ring runs ahead of the operand ring, so the
// scale transposition stays off the loop that bounds the K-tile rate (stage
// freed by an MMA -> operand load latency -> next MMA).
//
// Barriers (every wait bounded and parked rather than spinning; a timeout
// sets the device error word and the CTA's abort flag):
//   full[s]      CTA 0: operand bytes of stage s from both CTAs (expect_tx
//                by CTA 0 for the pair);
//   empty[s]     both CTAs: MMA commit (multicast to the pair) once the MMAs
//                of the K tile in operand stage s have completed, which also
//                frees the TMEM scale buffer of that K tile (the writers of
//                K tile i wait for the empty phase of K tile i - NB; NB < S
//                keeps that phase unambiguous);
//   sfull[j]     local: scale atom bytes of scale stage j;
//   sempty[j]    local: 4 writer warps have copied scale stage j to TMEM;
//   sf_ready[b]  CTA 0: 8 arrivals, the writer warps of both CTAs, once TMEM
//                scale buffer b holds the scales of its K tile;
//   acc_full     both CTAs: MMA commit after the last K tile of a tile;
//   acc_empty    CTA 0: 8 arrivals, the epilogue warps of both CTAs.
// Warp roles: warp 0 operand producer, warp 1 TMEM allocator (both CTAs) and
// MMA issuer (CTA 0), warps 2..5 epilogue, warps 6..9 scale writers, warp 10
// scale producer.  Warps w and w + 4 share TMEM lane quadrant w % 4.
//
// Used for the compute-bound shapes of "Peeling the Kernel Onion" (sections
// "The Benchmark Design" and "The Results"), from M, N >= 512 with enough
// 128 x 256 tiles for two per SM; K a multiple of 256.
#pragma once

#include "persistent_kernel.cuh"

namespace nvfp4 {

constexpr int kPairBM = 256;  // D rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;  // D columns per pair tile
constexpr int kPairThreads = 352;

struct PairConfig {
    static constexpr int A_BYTES = 128 * kStageKBytes;   // this CTA's 128 A rows
    static constexpr int B_BYTES = 128 * kStageKBytes;   // this CTA's 128 B rows
    static constexpr int AB_BYTES = A_BYTES + B_BYTES;
    static constexpr int SFA_BYTES = 128 * 16;           // scales of the 128 A rows
    static constexpr int SFB_BYTES = kPairBN * 16;       // scales of all 256 B rows
    static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;
    static constexpr int SF_STAGES = 5;
    static constexpr int STAGES = (kSmemLimit - 2048 - SF_STAGES * SF_BYTES) / AB_BYTES;
    static constexpr int SF_RING = STAGES * AB_BYTES;    // offset of the scale ring
    static constexpr int BAR_OFF = SF_RING + SF_STAGES * SF_BYTES;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + 1024;
    static constexpr int NB = 5;                         // TMEM scale buffers
    static constexpr int SF_BASE = kPairBN;              // accumulator: columns [0, 256)
    static constexpr int SF_STRIDE = 16 + 32;            // SFA 4 columns x 4 steps, SFB 8 x 4
    static constexpr int TMEM_COLS = 512;
    static_assert(SF_BASE + NB * SF_STRIDE <= TMEM_COLS, "TMEM columns");
    static_assert(STAGES >= 4, "operand ring depth");
    static_assert(NB < STAGES, "scale buffers are released through the operand ring");
    static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
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

struct PairParams {
    __nv_bfloat16* D;
    const uint8_t* sfa;    // scale atoms of A: [ceil(M/128)][K/64][512 B]
    const uint8_t* sfb;    // scale atoms of B: [ceil(N/128)][K/64][512 B]
    float alpha;
    int M, N, K;           // D is M x N
    int k_tiles;           // K / 256
    int tiles_m, tiles_n;  // 256 x 256 pair tiles
    int rb_a, rb_b;        // 128-row blocks of A and B (atom row blocks present)
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const PairParams prm) {
    using C = PairConfig;
    constexpr int S = C::STAGES;
    constexpr int SS = C::SF_STAGES;
    constexpr int NB = C::NB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    // bars: full[S], empty[S], sfull[SS], sempty[SS], sf_ready[NB], acc_full, acc_empty
    constexpr int NBARS = 2 * S + 2 * SS + NB + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_cta_rank();
    const int pair = (int)cluster_id_x(), pairs = (int)cluster_count_x();
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
    auto sfull_bar = [&](int j) { return bar_base + 8u * (2 * S + j); };
    auto sempty_bar = [&](int j) { return bar_base + 8u * (2 * S + SS + j); };
    auto sf_ready_bar = [&](int b) { return bar_base + 8u * (2 * S + 2 * SS + b); };
    const uint32_t acc_full_bar = bar_base + 8u * (2 * S + 2 * SS + NB);
    const uint32_t acc_empty_bar = acc_full_bar + 8u;
    const int tiles = prm.tiles_m * prm.tiles_n;
    const int KT = prm.k_tiles;
    const int my_tiles = (tiles - pair + pairs - 1) / pairs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int j = 0; j < SS; ++j) {
            mbar_init(sfull_bar(j), 1);
            mbar_init(sempty_bar(j), 4);
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
    }
    // both CTAs' barriers are initialised before either CTA signals the other
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
        // ---- operand producer: this CTA's A and B rows, bytes counted on CTA 0's full[s]
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
                    if (!mbar_wait_parked(empty_bar(s), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) goto producer_done;
                    const uint32_t st = smem_base + s * C::AB_BYTES;
                    if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * C::AB_BYTES);
                    const uint32_t fb = cluster_rank_addr(full_bar(s), 0);
                    tma_load_2d_pair(st, &tmA, fb, kt * kStageKBytes, a_row, pol_a);
                    tma_load_2d_pair(st + C::A_BYTES, &tmB, fb, kt * kStageKBytes, b_row, pol_b);
                }
            }
        producer_done:;
        }
    } else if (warp == 10) {
        // ---- scale producer: atoms of this CTA's 128 A rows and of all 256 B
        // rows (row blocks past the matrix are not loaded: their rows of D
        // are not stored)
        if (lane == 0) {
            const size_t steps = (size_t)prm.K / 64;
            int it = 0;
            for (int t = pair; t < tiles; t += pairs) {
                int tm, tn;
                tile_coords(t, prm.tiles_m, prm.tiles_n, tm, tn);
                const int rba = 2 * tm + (int)rank, rbb = 2 * tn;
                const bool la = rba < prm.rb_a, lb1 = rbb + 1 < prm.rb_b;
                const uint32_t bytes = (la ? 2048u : 0u) + 2048u + (lb1 ? 2048u : 0u);
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int j = it % SS;
                    if (!mbar_wait_parked(sempty_bar(j), ((uint32_t)(it / SS) & 1u) ^ 1u, abort_flag)) goto sf_producer_done;
                    const uint32_t st = smem_base + C::SF_RING + j * C::SF_BYTES;
                    mbar_arrive_expect_tx(sfull_bar(j), bytes);
                    const size_t k_off = (size_t)4 * kt * kAtomBytes;
                    if (la) bulk_load(st, prm.sfa + (size_t)rba * steps * kAtomBytes + k_off, 2048u, sfull_bar(j));
                    bulk_load(st + C::SFA_BYTES, prm.sfb + (size_t)rbb * steps * kAtomBytes + k_off, 2048u,
                              sfull_bar(j));
                    if (lb1)
                        bulk_load(st + C::SFA_BYTES + 2048, prm.sfb + (size_t)(rbb + 1) * steps * kAtomBytes + k_off,
                                  2048u, sfull_bar(j));
                }
            }
        sf_producer_done:;
        }
    } else if (warp == 1) {
        // ---- MMA issuer (CTA 0 only)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(kPairBM, kPairBN);
            int it = 0, tt = 0;
            bool ok = true;
            for (int t = pair; ok && t < tiles; t += pairs, ++tt) {
                // both CTAs' epilogues must have read the previous accumulator
                if (!mbar_wait_parked(acc_empty_bar, ((uint32_t)tt & 1u) ^ 1u, abort_flag)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S, b = it % NB;
                    if (!mbar_wait_parked(sf_ready_bar(b), (uint32_t)(it / NB) & 1u, abort_flag) ||
                        !mbar_wait_parked(full_bar(s), (uint32_t)(it / S) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_base + s * C::AB_BYTES;
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
        const int total = my_tiles * KT;
        for (int it = 0; it < total; ++it) {
            const int j = it % SS, b = it % NB;
            int got = 1;
            if (lane == 0)
                got = mbar_wait_parked(sfull_bar(j), (uint32_t)(it / SS) & 1u, abort_flag) &&
                      (it < NB || mbar_wait_parked(empty_bar((it - NB) % S), (uint32_t)((it - NB) / S) & 1u, abort_flag));
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            const uint32_t st = smem_base + C::SF_RING + j * C::SF_BYTES;
            const uint32_t sf = t_quad + C::SF_BASE + b * C::SF_STRIDE;
            uint32_t wa[16];
            gather_scale_words<false>(st, lane, wa);
            tmem_store_16(sf, wa);
            // B rows 0..127 and 128..255: step j uses columns 8j + 4*half + r1
            uint32_t wb0[16], wb1[16], wb[32];
            gather_scale_words<false>(st + C::SFA_BYTES, lane, wb0);
            gather_scale_words<false>(st + C::SFA_BYTES + 2048, lane, wb1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int r1 = 0; r1 < 4; ++r1) {
                    wb[8 * k + r1] = wb0[4 * k + r1];
                    wb[8 * k + 4 + r1] = wb1[4 * k + r1];
                }
            tmem_store_32(sf + 16, wb);
            tmem_wait_store();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sempty_bar(j));
                mbar_arrive_remote(sf_ready_bar(b), 0);
            }
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
            if (lane == 0) ok = mbar_wait_parked(acc_full_bar, (uint32_t)tt & 1u, abort_flag) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0) || *abort_flag) break;
            tc_fence_after();
            const int p = tm * kPairBM + (int)rank * 128 + quad * 32 + lane;
            const int q_base = tn * kPairBN;
            // Drain the whole accumulator row into registers as BF16 pairs,
            // hand the accumulator back, then store: the MMAs of the next
            // tile overlap the global stores.
            uint32_t pk[kPairBN / 2];
#pragma unroll
            for (int c = 0; c < kPairBN / 16; ++c) {
                uint32_t r[16];
                tmem_load_16(t_quad + 16 * c, r);
                tmem_wait_load();
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    pk[8 * c + e] = pack_bf16x2(__uint_as_float(r[2 * e]) * prm.alpha,
                                                __uint_as_float(r[2 * e + 1]) * prm.alpha);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acc_empty_bar, 0);
            if (p < prm.M) {
                __nv_bfloat16* drow = prm.D + (size_t)p * prm.N + q_base;
#pragma unroll
                for (int h = 0; h < kPairBN / 8; ++h)
                    if (q_base + 8 * h < prm.N)   // N is a multiple of 8
                        *reinterpret_cast<uint4*>(drow + 8 * h) =
                            make_uint4(pk[4 * h], pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
            }
        }
    }

    // Neither CTA frees TMEM or exits while the other may still use it: the
    // MMA of CTA 0 reads CTA 1's shared memory and TMEM, CTA 1's loads
    // complete on CTA 0's barriers, and CTA 1's epilogue and writers arrive
    // on CTA 0's barriers.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace nvfp4
