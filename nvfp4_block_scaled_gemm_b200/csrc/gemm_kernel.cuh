// NVFP4 block-scaled GEMM on the sm_100a tensor cores (tcgen05).
//
// D = alpha * (A * sA) x (B * sB)^T, E2M1 operands packed two per byte with
// one E4M3 scale per 16 elements along K, BF16 output (the format of "The
// SM120 FP4 Kernel Disaster", section "Input Knowledge Required", and "Peeling
// the Kernel Onion", section "The Benchmark Design").
//
// One CTA computes a 128 x BQ tile of the product P x Q^T, where P is the
// operand on the tensor cores' M side (128 rows) and Q the one on the N side
// (BQ rows).  Normally P = A and Q = B; for small M the roles swap (P = B, the
// weights, Q = A, the few activation rows) so that the weight matrix streams
// through the 128-row MMA side, and the epilogue writes the transpose.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: operand tiles (2-D TMA, 128-byte swizzle) and
//               scale atoms (bulk copies) into a STAGES-deep ring;
//   warp 1      TMEM allocator and MMA issuer: per stage, copies the scale
//               atoms into TMEM (tcgen05.cp) and issues four
//               tcgen05.mma.kind::mxf4nvf4.block16 (K = 64 each);
//   warps 2..5  epilogue: TMEM -> registers -> alpha, BF16 -> global, or
//               fp32 partial sums with a last-arriver reduction (split-K).
// Ring protocol: full[s] (producer arrive + TMA bytes) and empty[s]
// (tcgen05.commit after the MMAs that read stage s).  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int kBM = 128;          // rows of P per tile (MMA M)
constexpr int kStageK = 256;      // K elements per pipeline stage
constexpr int kStageKBytes = 128; // = one 128-byte swizzle row of packed E2M1
constexpr int kStepK = 64;        // K of one tcgen05.mma (mxf4nvf4, dense)
constexpr int kAtomBytes = 512;   // scale atom: 128 rows x 4 blocks of 16
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory

template <int BQ>
struct TileConfig {
    static_assert(BQ == 16 || BQ == 32 || BQ == 64 || BQ == 128 || BQ == 256, "BQ");
    static constexpr int P_BYTES = kBM * kStageKBytes;
    static constexpr int Q_BYTES = BQ * kStageKBytes;
    static constexpr int Q_BLOCKS = BQ > 128 ? BQ / 128 : 1;        // 128-row scale blocks of Q
    static constexpr int SFP_BYTES = 4 * kAtomBytes;
    static constexpr int SFQ_BYTES = 4 * kAtomBytes * Q_BLOCKS;
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;
    static constexpr int STAGES_FIT = (kSmemLimit - 2048) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 1024;
    // TMEM columns: fp32 accumulator [0, BQ), then the scale columns.
    static constexpr int SFP_COL = BQ < 32 ? 32 : BQ;
    static constexpr int SFQ_COL = SFP_COL + 16;                       // 4 steps x 4 columns
    static constexpr int COLS_USED = SFQ_COL + 16 * Q_BLOCKS;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
    static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
    static_assert(STAGES >= 2, "stages");
};

struct GemmParams {
    const uint8_t* sfp;       // P scales, tensor-core atom layout
    const uint8_t* sfq;       // Q scales, tensor-core atom layout
    __nv_bfloat16* D;
    float* partials;          // split-K: [splits][tilesP][tilesQ][128][BQ]
    unsigned* counters;       // split-K: [tilesP][tilesQ], zero between launches
    float alpha;
    int rows_p, rows_q;       // valid rows of P and Q
    int K;                    // elements, multiple of 64
    int ldd;                  // row stride of D in elements (= N)
    int k_tiles;              // ceil(K / 256)
    int k_tiles_per_split;
};

template <int BQ, bool SWAP>
__device__ __forceinline__ void store_tile_chunk(const GemmParams& prm, const float (&v)[16], int p, int q0) {
    // v[c] is the fp32 result for (P row p, Q row q0 + c); alpha already applied.
    if (p >= prm.rows_p) return;
    if (!SWAP) {
        // D[p][q]: 16 consecutive bf16 of one row -> two 16-byte stores.
        __nv_bfloat16* dst = prm.D + (size_t)p * prm.ldd + q0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (q0 + 8 * h < prm.rows_q) {   // rows_q (= N) is a multiple of 8
                uint4 w;
                w.x = pack_bf16x2(v[8 * h + 0], v[8 * h + 1]);
                w.y = pack_bf16x2(v[8 * h + 2], v[8 * h + 3]);
                w.z = pack_bf16x2(v[8 * h + 4], v[8 * h + 5]);
                w.w = pack_bf16x2(v[8 * h + 6], v[8 * h + 7]);
                *reinterpret_cast<uint4*>(dst + 8 * h) = w;
            }
        }
    } else {
        // D[q][p]: lanes hold consecutive p, so each store instruction of the
        // warp writes 32 consecutive bf16 of one output row.
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            if (q0 + c < prm.rows_q) prm.D[(size_t)(q0 + c) * prm.ldd + p] = __float2bfloat16_rn(v[c]);
        }
    }
}

template <int BQ, bool SWAP, bool SPLITK>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const GemmParams prm) {
    using C = TileConfig<BQ>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
    // bars[0..S) full, bars[S..2S) empty, bars[2S] accumulator ready
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tq = blockIdx.x, tp = blockIdx.y, split = blockIdx.z;
    const int kt_begin = split * prm.k_tiles_per_split;
    const int kt_end = min(prm.k_tiles, kt_begin + prm.k_tiles_per_split);
    const int steps_total = prm.K / kStepK;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
    const uint32_t accum_bar = bar_base + 8u * (2 * S);

    // Q scale blocks that exist in the (row-padded) atom buffer for this tile.
    const int q_row0 = tq * BQ;
    const int q_blocks_in_buf = (prm.rows_q + 127) / 128;
    const int q_block0 = BQ >= 128 ? q_row0 / 128 : 0;
    int q_blocks = C::Q_BLOCKS;
    if (q_block0 + q_blocks > q_blocks_in_buf) q_blocks = q_blocks_in_buf - q_block0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(accum_bar, 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensor_map(&tmP);
            prefetch_tensor_map(&tmQ);
            // The 128-row side is read by exactly one tile column in the
            // swapped layout (the weights): stream it; keep the shared side.
            const uint64_t pol_p = SWAP ? policy_evict_first() : policy_evict_last();
            const uint64_t pol_q = SWAP ? policy_evict_last() : policy_evict_first();
            int it = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) break;
                const int steps = min(4, steps_total - 4 * kt);
                const uint32_t sf_bytes = (uint32_t)steps * kAtomBytes;
                mbar_arrive_expect_tx(full_bar(s), C::P_BYTES + C::Q_BYTES + sf_bytes * (1 + q_blocks));
                const uint32_t st = smem_base + s * C::STAGE_BYTES;
                tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                tma_load_2d(st + C::P_BYTES, &tmQ, full_bar(s), kt * kStageKBytes, q_row0, pol_q);
                bulk_load(st + C::P_BYTES + C::Q_BYTES,
                          prm.sfp + ((size_t)tp * steps_total + 4 * kt) * kAtomBytes, sf_bytes, full_bar(s));
                for (int b = 0; b < q_blocks; ++b) {
                    bulk_load(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + b * 4 * kAtomBytes,
                              prm.sfq + ((size_t)(q_block0 + b) * steps_total + 4 * kt) * kAtomBytes, sf_bytes,
                              full_bar(s));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(kBM, BQ);
            int it = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!mbar_wait(full_bar(s), ph, abort_flag)) break;
                tc_fence_after();
                const int steps = min(4, steps_total - 4 * kt);
                const uint32_t st = smem_base + s * C::STAGE_BYTES;
                const uint32_t sfp_s = st + C::P_BYTES + C::Q_BYTES;
                const uint32_t sfq_s = sfp_s + C::SFP_BYTES;
                for (int j = 0; j < steps; ++j) {
                    tc_copy_32x128b_x4(tmem + C::SFP_COL + 4 * j, desc_scale_atom(sfp_s + j * kAtomBytes));
                    for (int b = 0; b < q_blocks; ++b)
                        tc_copy_32x128b_x4(tmem + C::SFQ_COL + 4 * C::Q_BLOCKS * j + 4 * b,
                                           desc_scale_atom(sfq_s + b * 4 * kAtomBytes + j * kAtomBytes));
                }
                for (int j = 0; j < steps; ++j) {
                    tc_mma_nvf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::P_BYTES + 32 * j),
                                idesc, tmem + C::SFP_COL + 4 * j, tmem + C::SFQ_COL + 4 * C::Q_BLOCKS * j,
                                (it > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(empty_bar(s));
            }
            // Always signal the epilogue (also after an abort), and only once
            // every MMA issued above has completed.
            tc_commit(accum_bar);
        }
        __syncwarp();
    } else {
        // Epilogue: warp w reads TMEM lane quadrant w % 4.
        const int quad = warp & 3;
        const int row = quad * 32 + lane;       // row of P within the tile
        const int p = tp * kBM + row;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(accum_bar, 0, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        tc_fence_after();
        if (ok && !*abort_flag) {
            const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16);
            if (!SPLITK) {
#pragma unroll 1
                for (int c0 = 0; c0 < BQ; c0 += 16) {
                    uint32_t r[16];
                    tmem_load_16(t_row + c0, r);
                    tmem_wait_load();
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]) * prm.alpha;
                    store_tile_chunk<BQ, SWAP>(prm, v, p, q_row0 + c0);
                }
            } else {
                const int tilesP = gridDim.y, tilesQ = gridDim.x, splits = gridDim.z;
                const size_t tile_elems = (size_t)kBM * BQ;
                const size_t tile_id = (size_t)tp * tilesQ + tq;
                float* mine = prm.partials + ((size_t)split * tilesP * tilesQ + tile_id) * tile_elems + (size_t)row * BQ;
#pragma unroll 1
                for (int c0 = 0; c0 < BQ; c0 += 16) {
                    uint32_t r[16];
                    tmem_load_16(t_row + c0, r);
                    tmem_wait_load();
#pragma unroll
                    for (int c = 0; c < 16; c += 4)
                        *reinterpret_cast<uint4*>(mine + c0 + c) = make_uint4(r[c], r[c + 1], r[c + 2], r[c + 3]);
                }
                __threadfence();
                named_barrier(1, 128);
                if (warp == 2 && lane == 0) {
                    const unsigned prev = atomicAdd(prm.counters + tile_id, 1u);
                    const int last = (prev == (unsigned)(splits - 1));
                    if (last) prm.counters[tile_id] = 0;   // ready for the next launch
                    *last_flag = last;
                }
                named_barrier(1, 128);
                if (*last_flag) {
                    __threadfence();
                    const float* base = prm.partials + tile_id * tile_elems + (size_t)row * BQ;
                    const size_t split_stride = (size_t)tilesP * tilesQ * tile_elems;
#pragma unroll 1
                    for (int c0 = 0; c0 < BQ; c0 += 16) {
                        float v[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c) v[c] = 0.0f;
                        for (int z = 0; z < splits; ++z) {   // fixed order: deterministic
                            const float4* src = reinterpret_cast<const float4*>(base + z * split_stride + c0);
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float4 f = __ldcg(src + c);
                                v[4 * c + 0] += f.x;
                                v[4 * c + 1] += f.y;
                                v[4 * c + 2] += f.z;
                                v[4 * c + 3] += f.w;
                            }
                        }
#pragma unroll
                        for (int c = 0; c < 16; ++c) v[c] *= prm.alpha;
                        store_tile_chunk<BQ, SWAP>(prm, v, p, q_row0 + c0);
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
