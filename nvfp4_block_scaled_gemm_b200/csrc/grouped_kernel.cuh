// Grouped (MoE) NVFP4 GEMM: G problems sharing N and K.  Rows
// [off[g], off[g+1]) of A multiply expert g's weights B[g] and are scaled by
// alpha[g] ("Peeling the Kernel Onion", sections "The Critical Connection to
// Real Inference" -- about 16 rows per expert -- and "Knowledge Created and
// Its Impact" -- persistent grouped kernels).
//
// Persistent kernel.  A work unit is (expert g, 128-row tile of B[g]).  Units
// are handed out at run time: each CTA's producer takes the next unit index
// from a global counter (atomicAdd) while its current unit streams, so CTAs
// that drew expensive units take fewer; the last CTA to finish zeroes the
// counter for the next launch on the stream.  Unit indices run over the
// experts with more than 128 rows (several passes) first, then the others,
// which makes the greedy hand-out close to longest-first.  The weights sit on
// the tensor cores' 128-row M side and the expert's tokens on the N side, in
// passes of up to 128 rows; each pass loads only ceil(rows/16) 16-row boxes
// of A and runs MMAs with N = that many rows rounded up to 16 (the instruction
// descriptor is built at run time).  Empty experts are never handed out.
//
// The weight producer passes each unit to the other roles through a small ring
// of unit descriptors in shared memory (job_full / job_empty barriers).
//
// Warp roles (352 threads): warp 0 weight producer (TMA of the weight tile and
// its scales); warp 10 token producer (TMA of the unit's token rows and their
// scales into the same ring stage: with every copy issued from one thread the
// stream stalls on issue); warp 1 TMEM allocator and MMA issuer; warps 2..5
// epilogue (TMEM -> alpha[g] -> BF16, transposed through shared memory into
// 16-byte stores to D); warps 6..9 scale writers (shared memory -> TMEM, one
// warp per lane quadrant, as in the single GEMM kernel).  The fp32
// accumulator is double-buffered in TMEM so the epilogue of one pass overlaps
// the main loop of the next.
#pragma once

#include "gemm_kernel.cuh"

namespace nvfp4 {

constexpr int kGroupedThreads = 352;
constexpr int kGroupedBQ = 128;   // max tokens per pass
constexpr int kJobSlots = 4;      // unit descriptors in flight between the producer and the other roles
constexpr int kOrderMax = 2048;   // experts ordered heavy-first in shared memory (natural order beyond)
// TMEM scale buffers: as many as the ring has stages, so the scale writers
// never wait on an MMA the ring itself does not (310 -> 305.5 us on the
// 256-expert MoE GEMM against 4 buffers)
constexpr int kGroupedScaleBuffers = 6;

struct GroupedParams {
    const float* alpha;           // [G]
    const int32_t* offsets;       // [G+1]
    __nv_bfloat16* D;             // [M_total][N]
    int G, N, K, M_total;
    int tiles_n;                  // ceil(N / 128)
    int k_tiles;                  // K / 256
    unsigned* counter;            // [2]: next unit, CTAs finished; zero between launches
};

struct GroupedConfig {
    static constexpr int BQ = kGroupedBQ;
    static constexpr int P_BYTES = kBM * kStageKBytes;            // 16 KB of weights per K tile
    static constexpr int Q_BYTES = BQ * kStageKBytes;             // up to 16 KB of tokens
    static constexpr int SFP_BYTES = 4 * kAtomBytes;
    static constexpr int SFQ_BYTES = 4 * kAtomBytes;
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;
    static constexpr int TAIL_BYTES = 1024 + 2 * kOrderMax;     // barriers, job ring, expert order
    static constexpr int EPI_BYTES = 4 * 1024;                    // per epilogue warp: 16 token rows x 32 bf16
    static constexpr int STAGES_FIT = (kSmemLimit - 1024 - TAIL_BYTES - EPI_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static_assert(STAGES >= kGroupedScaleBuffers, "scale buffers are released through the ring barriers");
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + TAIL_BYTES + EPI_BYTES;
    // TMEM: two accumulators [0,BQ) and [BQ,2BQ), then kGroupedScaleBuffers scale buffers of 32.
    static constexpr int ACC_COLS = BQ;
    static constexpr int SF_BASE = 2 * BQ;
    static constexpr int SF_STRIDE = 32;
    static constexpr int TMEM_COLS = 512;
    static_assert(SF_BASE + kGroupedScaleBuffers * SF_STRIDE <= TMEM_COLS, "TMEM columns");
    static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
};

// One unit as the roles see it: expert g, weight tile nt, its token rows.
struct UnitJob {
    int g, nt, r0, rows;
    __device__ int passes() const { return (rows + kGroupedBQ - 1) / kGroupedBQ; }
    __device__ int q_row0(int pass) const { return r0 + pass * kGroupedBQ; }
    __device__ int q_rows(int pass) const { return min(kGroupedBQ, rows - pass * kGroupedBQ); }
};

__global__ void __launch_bounds__(kGroupedThreads, 1)
    nvfp4_grouped_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmSB, const __grid_constant__ CUtensorMap tmSA,
                         const GroupedParams prm) {
    using C = GroupedConfig;
    constexpr int S = C::STAGES;
    constexpr int NB = kGroupedScaleBuffers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tail = smem + S * C::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
    // bars: [0,S) full, [S,2S) empty, [2S,2S+NB) sf_ready, [2S+NB, +2) acc_full,
    //       [2S+NB+2, +2) acc_empty, then job_full[kJobSlots], job_empty[kJobSlots]
    constexpr int NBARS = 2 * S + NB + 4 + 2 * kJobSlots;
    static_assert(NBARS * 8 + 8 <= 256, "tail layout");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int4* jobs = reinterpret_cast<volatile int4*>(tail + 256);   // unit descriptors {g, nt, r0, rows}
    int16_t* order = reinterpret_cast<int16_t*>(tail + 512);             // experts, heavy first

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
    auto sf_ready_bar = [&](int b) { return bar_base + 8u * (2 * S + b); };
    auto acc_full_bar = [&](int a) { return bar_base + 8u * (2 * S + NB + a); };
    auto acc_empty_bar = [&](int a) { return bar_base + 8u * (2 * S + NB + 2 + a); };
    auto job_full_bar = [&](int j) { return bar_base + 8u * (2 * S + NB + 4 + j); };
    auto job_empty_bar = [&](int j) { return bar_base + 8u * (2 * S + NB + 4 + kJobSlots + j); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 2);   // weight producer and token producer
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < NB; ++b) mbar_init(sf_ready_bar(b), 4);
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full_bar(a), 1);
            mbar_init(acc_empty_bar(a), 4);
        }
        for (int j = 0; j < kJobSlots; ++j) {
            mbar_init(job_full_bar(j), 1);
            mbar_init(job_empty_bar(j), 10);   // token producer, MMA issuer, 4 writer warps, 4 epilogue warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        prefetch_tensor_map(&tmB);
        prefetch_tensor_map(&tmA);
        prefetch_tensor_map(&tmSB);
        prefetch_tensor_map(&tmSA);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_launch_dependents();
    grid_dependency_wait();

    // Consumers take unit j from ring slot j % kJobSlots; false ends the loop
    // (no more units, or an abort).  Lane 0 waits; the descriptor is broadcast.
    auto take_job = [&](int j, UnitJob& jb, bool whole_warp) -> bool {
        const int slot = j % kJobSlots;
        int4 d = make_int4(-1, 0, 0, 0);
        if (lane == 0 && mbar_wait(job_full_bar(slot), (uint32_t)(j / kJobSlots) & 1u, abort_flag)) {
            d.x = jobs[slot].x;
            d.y = jobs[slot].y;
            d.z = jobs[slot].z;
            d.w = jobs[slot].w;
            mbar_arrive(job_empty_bar(slot));
        }
        if (whole_warp) {
            d.x = __shfl_sync(0xffffffffu, d.x, 0);
            d.y = __shfl_sync(0xffffffffu, d.y, 0);
            d.z = __shfl_sync(0xffffffffu, d.z, 0);
            d.w = __shfl_sync(0xffffffffu, d.w, 0);
        }
        jb.g = d.x, jb.nt = d.y, jb.r0 = d.z, jb.rows = d.w;
        return d.x >= 0;
    };

    if (warp == 0) {
        // ---- expert order (heavy first), then the producer on lane 0
        const bool ordered = prm.G <= kOrderMax;
        int listed = prm.G;
        if (ordered) {
            listed = 0;
            for (int heavy = 1; heavy >= 0; --heavy)
                for (int base = 0; base < prm.G; base += 32) {
                    const int e = base + lane;
                    const int rows = e < prm.G ? __ldg(prm.offsets + e + 1) - __ldg(prm.offsets + e) : 0;
                    const bool take = heavy ? rows > kGroupedBQ : (rows > 0 && rows <= kGroupedBQ);
                    const unsigned m = __ballot_sync(0xffffffffu, take);
                    if (take) order[listed + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
                    listed += __popc(m);
                }
        }
        __syncwarp();
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();   // each weight tile is read by one unit
            const unsigned total = (unsigned)listed * (unsigned)prm.tiles_n;
            auto describe = [&](unsigned u, UnitJob& jb) {
                const int idx = (int)(u / (unsigned)prm.tiles_n);
                jb.nt = (int)(u % (unsigned)prm.tiles_n);
                jb.g = ordered ? (int)order[idx] : idx;
                jb.r0 = __ldg(prm.offsets + jb.g);
                jb.rows = __ldg(prm.offsets + jb.g + 1) - jb.r0;
            };
            unsigned u_next = atomicAdd(prm.counter, 1u);
            int it = 0;
            for (int j = 0;; ++j) {
                UnitJob jb{-1, 0, 0, 0};
                bool have = false;
                for (unsigned u = u_next; u < total; u = atomicAdd(prm.counter, 1u)) {
                    describe(u, jb);
                    if (jb.rows > 0) {   // empty experts appear only without the order table
                        have = true;
                        break;
                    }
                }
                if (have) u_next = atomicAdd(prm.counter, 1u);   // next index, fetched while this unit streams
                const int slot = j % kJobSlots;
                if (!mbar_wait(job_empty_bar(slot), ((uint32_t)(j / kJobSlots) & 1u) ^ 1u, abort_flag)) break;
                jobs[slot].x = have ? jb.g : -1;
                jobs[slot].y = jb.nt;
                jobs[slot].z = jb.r0;
                jobs[slot].w = jb.rows;
                mbar_arrive(job_full_bar(slot));
                if (!have) break;
                const int brow = jb.g * prm.N + jb.nt * kBM;   // row of B viewed as [G*N][K/2]
                for (int pass = 0; pass < jb.passes(); ++pass) {
                    const int nbox = (jb.q_rows(pass) + 15) / 16;
                    for (int kt = 0; kt < prm.k_tiles; ++kt, ++it) {
                        const int s = it % S;
                        if (!mbar_wait(empty_bar(s), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) goto producer_done;
                        const uint32_t st = smem_base + s * C::STAGE_BYTES;
                        mbar_arrive_expect_tx(full_bar(s), C::P_BYTES + 16 * kBM);
                        tma_load_2d(st, &tmB, full_bar(s), kt * kStageKBytes, brow, pol_w);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSB, full_bar(s), kt * 16, brow, pol_w);
                    }
                }
            }
        producer_done:;
        }
    } else if (warp == kGroupedThreads / 32 - 1) {
        // ---- token producer: the unit's token rows and their scales, into
        // the same ring stages (a second issuing thread: one thread issuing
        // every copy of a stage limits the stream rate)
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();   // token rows are shared by all N tiles
            int it = 0;
            bool ok = true;
            UnitJob jb;
            for (int j = 0; ok && take_job(j, jb, false); ++j) {
                for (int pass = 0; ok && pass < jb.passes(); ++pass) {
                    const int nbox = (jb.q_rows(pass) + 15) / 16;
                    for (int kt = 0; kt < prm.k_tiles; ++kt, ++it) {
                        const int s = it % S;
                        if (!mbar_wait(empty_bar(s), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t st = smem_base + s * C::STAGE_BYTES;
                        mbar_arrive_expect_tx(full_bar(s), nbox * (16 * kStageKBytes + 16 * 16));
                        for (int bx = 0; bx < nbox; ++bx) {
                            tma_load_2d(st + C::P_BYTES + bx * 16 * kStageKBytes, &tmA, full_bar(s), kt * kStageKBytes,
                                        jb.q_row0(pass) + 16 * bx, pol_a);
                            tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + bx * 256, &tmSA, full_bar(s),
                                        kt * 16, jb.q_row0(pass) + 16 * bx, pol_a);
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, jc = 0;
            bool ok = true;
            UnitJob jb;
            for (int j = 0; ok && take_job(j, jb, false); ++j) {
                for (int pass = 0; ok && pass < jb.passes(); ++pass, ++jc) {
                    const int acc = jc & 1;
                    const uint32_t n_mma = (uint32_t)((jb.q_rows(pass) + 15) / 16 * 16);
                    const uint32_t idesc = idesc_nvf4(kBM, (int)n_mma);
                    if (!mbar_wait(acc_empty_bar(acc), ((uint32_t)(jc >> 1) & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + acc * C::ACC_COLS;
                    for (int kt = 0; kt < prm.k_tiles; ++kt, ++it) {
                        const int s = it % S, b = it % NB;
                        if (!mbar_wait(sf_ready_bar(b), (uint32_t)(it / NB) & 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t st = smem_base + s * C::STAGE_BYTES;
                        const uint32_t sf = tmem + C::SF_BASE + b * C::SF_STRIDE;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            tc_mma_nvf4(d_tmem, desc_kmajor_sw128(st + 32 * q),
                                        desc_kmajor_sw128(st + C::P_BYTES + 32 * q), idesc, sf + 4 * q, sf + 16 + 4 * q,
                                        (kt > 0 || q > 0) ? 1u : 0u);
                        tc_commit(empty_bar(s));   // frees the ring stage and scale buffer b
                    }
                    tc_commit(acc_full_bar(acc));
                }
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---- scale writers (warp w owns TMEM lane quadrant w % 4)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        int it = 0;
        bool ok = true;
        UnitJob jb;
        for (int j = 0; ok && take_job(j, jb, true); ++j) {
            const int steps = jb.passes() * prm.k_tiles;
            for (int u = 0; u < steps; ++u, ++it) {
                const int s = it % S, b = it % NB, jj = it - NB;
                int got = 1;
                // scale buffer b was last used by K tile it - NB, released by
                // the MMA commit on that tile's ring stage; with one buffer per
                // stage that is stage s's previous phase, which the producer
                // waited for before the loads that full(s) reports
                if (lane == 0)
                    got = mbar_wait(full_bar(s), (uint32_t)(it / S) & 1u, abort_flag) &&
                          (NB == S || jj < 0 || mbar_wait(empty_bar(jj % S), (uint32_t)(jj / S) & 1u, abort_flag));
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t st = smem_base + s * C::STAGE_BYTES;
                const uint32_t sf = t_quad + C::SF_BASE + b * C::SF_STRIDE;
                uint32_t wp[16], wq[16];
                gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES, lane, wp);
                gather_scale_words<true>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq);
                tmem_store_16(sf, wp);
                tmem_store_16(sf + 16, wq);
                tmem_wait_store();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sf_ready_bar(b));
            }
        }
    } else {
        // ---- epilogue (warps 2..5, TMEM lane quadrant w % 4 = weight rows)
        const int quad = warp & 3;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t epi = smem_addr(tail) + (uint32_t)(C::TAIL_BYTES + quad * 1024);
        int jc = 0;
        bool live = true;
        UnitJob jb;
        for (int j = 0; live && take_job(j, jb, true); ++j) {
            const float alpha = __ldg(prm.alpha + jb.g);
            const int n_warp = jb.nt * kBM + quad * 32;       // this warp's first output column
            for (int pass = 0; pass < jb.passes(); ++pass, ++jc) {
                const int acc = jc & 1;
                int ok = 1;
                if (lane == 0) ok = mbar_wait(acc_full_bar(acc), (uint32_t)(jc >> 1) & 1u, abort_flag) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, ok, 0) || *abort_flag) {
                    live = false;
                    break;
                }
                tc_fence_after();
                const int q0 = jb.q_row0(pass), nq = jb.q_rows(pass);
#pragma unroll 1
                for (int c0 = 0; c0 < nq; c0 += 16) {
                    uint32_t r[16];
                    tmem_load_16(t_quad + acc * C::ACC_COLS + c0, r);
                    tmem_wait_load();
                    // Transpose through this warp's 1 KB of shared memory: row c
                    // holds the 32 columns of token row q0 + c0 + c, which then
                    // leave as 16-byte pieces of 8 consecutive columns.
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(r[c]) * alpha);
                        asm volatile("st.shared.b16 [%0], %1;" ::"r"(epi + (uint32_t)(c * 64 + lane * 2)),
                                     "h"(*reinterpret_cast<const uint16_t*>(&h))
                                     : "memory");
                    }
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int idx = lane + 32 * h, c = idx >> 2, part = idx & 3;
                        const int n0 = n_warp + part * 8;   // N is a multiple of 8
                        const uint4 val = ld_shared_v4(epi + (uint32_t)(c * 64 + part * 16));
                        if (c0 + c < nq && n0 < prm.N)
                            *reinterpret_cast<uint4*>(prm.D + (size_t)(q0 + c0 + c) * prm.N + n0) = val;
                    }
                    __syncwarp();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty_bar(acc));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    // The last CTA to finish zeroes the unit counter for the next launch (no
    // CTA fetches after it has counted itself finished).
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(prm.counter + 1, 1u) == gridDim.x - 1) {
            atomicExch(prm.counter, 0u);
            atomicExch(prm.counter + 1, 0u);
            __threadfence();
        }
    }
}

}  // namespace nvfp4
