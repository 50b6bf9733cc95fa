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
//   warp 0      TMA producer: per 256-element K tile, the P and Q operand
//               tiles (2-D TMA, 128-byte swizzle) and their scales into a
//               STAGES-deep shared-memory ring.  Scales arrive either as
//               row-major [rows][16 B] tiles (SFR: one 2-D TMA box per
//               operand) or already in 512-byte atoms (bulk copies).
//   warp 1      TMEM allocator and MMA issuer: four
//               tcgen05.mma.kind::mxf4nvf4.block16 (K = 64 each) per K tile.
//   warps 2..5  scale writers during the main loop, epilogue afterwards.  Warp
//               w owns TMEM lane quadrant w % 4; per K tile it moves the
//               scales of both operands from shared memory into one of
//               kScaleBuffers rotating TMEM scale buffers with tcgen05.st.
//               The epilogue: TMEM -> registers -> alpha, BF16 -> global.
//
// Scale layout the MMA reads from TMEM (the one tcgen05.cp.32x128b.warpx4
// produces from a 512-byte atom): for one K step of 64 elements (4 scale
// bytes per row) and 128 rows, row r's 4 bytes sit in lane r % 32 of every
// lane quadrant, column base + r / 32.  A writer lane L therefore stores, for
// K step j, the words of rows L, L+32, L+64, L+96 in columns base + 4j + 0..3.
// Writing them with tcgen05.st from four warps keeps the single MMA-issuing
// thread free of copy instructions.
//
// Split-K: the CTAs that share an output tile form one thread-block cluster
// (blockIdx.x = cluster rank = K slice).  Rank r owns rows [r*128/S,
// (r+1)*128/S) of the tile.  Every CTA stores each fp32 partial row straight
// from registers into the owner's receive slots (distributed shared memory,
// slot = the sender's rank; a region of its own, outside the ring); after one
// cluster barrier each owner sums its S slots in rank order (deterministic),
// applies alpha and stores BF16.  The cluster barrier that guarantees every
// peer has started is arrived at kernel start and waited on just before the
// first remote store.
//
// BF16 activations (QBF16, swapped layout only): the producer brings the raw
// BF16 Q tile (BQ rows x 256 values) by TMA instead of the FP4 tile and its
// scales; the four writer warps quantize it (quant.cuh block steps) into the
// 128-byte swizzled FP4 tile and the row-major scale tile of the stage, fence
// the writes for the tensor cores, meet on the cvt barrier, and then move the
// scales into TMEM as usual.
//
// Barriers: full[s] (producer arrive + TMA bytes), empty[s] (MMA commit:
// stage s may be refilled and the TMEM scale buffer of that K tile may be
// rewritten), sf_ready[b] (4 writer arrivals: scale buffer b holds this K
// tile), accum (MMA commit after the last K tile), cvt (QBF16: 4 writer
// arrivals per K tile).  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace nvfp4 {

constexpr int kBM = 128;          // rows of P per tile (MMA M)
constexpr int kStageK = 256;      // K elements per pipeline stage
constexpr int kStageKBytes = 128; // = one 128-byte swizzle row of packed E2M1
constexpr int kStepK = 64;        // K of one tcgen05.mma (mxf4nvf4, dense)
constexpr int kAtomBytes = 512;   // scale atom: 128 rows x 4 blocks of 16
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory
constexpr int kScaleBuffers = 4;    // rotating TMEM scale buffers

// QBF16: the Q operand (the activations, swapped layout) arrives as BF16 and
// is quantized in shared memory by the writer warps: each stage also holds
// the raw BF16 tile, BQ rows x 256 values.
template <int BQ, bool SPLITK, bool QBF16 = false>
struct TileConfig {
    static_assert(BQ == 16 || BQ == 32 || BQ == 64 || BQ == 128 || BQ == 256, "BQ");
    static constexpr int P_BYTES = kBM * kStageKBytes;
    static constexpr int Q_BYTES = BQ * kStageKBytes;
    static constexpr int Q_BLOCKS = BQ > 128 ? BQ / 128 : 1;        // 128-row scale blocks of Q
    static constexpr int SFP_BYTES = 4 * kAtomBytes;
    static constexpr int SFQ_BYTES = 4 * kAtomBytes * Q_BLOCKS;
    static constexpr int QRAW_OFF = P_BYTES + Q_BYTES + SFP_BYTES + SFQ_BYTES;
    static constexpr int QRAW_BYTES = QBF16 ? BQ * 256 * 2 : 0;
    static constexpr int STAGE_BYTES = QRAW_OFF + QRAW_BYTES;
    // split-K receive slots: one fp32 row of kPartLd floats per tile row, in
    // a region of their own when that still leaves kScaleBuffers stages,
    // otherwise in the ring (then written only after the whole cluster's
    // main loops are done).
    static constexpr int SLOT_NEED = kBM * (BQ + 4) * 4;
    static constexpr bool OWN_SLOTS = SPLITK && (kSmemLimit - 2048 - SLOT_NEED) / STAGE_BYTES >= kScaleBuffers;
    static constexpr int SLOT_BYTES = OWN_SLOTS ? SLOT_NEED : 0;
    static constexpr int STAGES_FIT = (kSmemLimit - 2048 - SLOT_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + SLOT_BYTES + 1024;
    // TMEM columns: fp32 accumulator [0, BQ), then kScaleBuffers scale buffers
    // of (P: 4 steps x 4) + (Q: 4 steps x 4 x Q_BLOCKS) columns.
    static constexpr int SF_BASE = BQ < 32 ? 32 : BQ;
    static constexpr int SF_STRIDE = 16 + 16 * Q_BLOCKS;
    static constexpr int COLS_USED = SF_BASE + kScaleBuffers * SF_STRIDE;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "TMEM columns");
    static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
    static_assert(STAGES >= kScaleBuffers, "scale buffers are released through the ring barriers");
};

struct GemmParams {
    const uint8_t* sfp;       // P scales, atom layout (non-SFR)
    const uint8_t* sfq;       // Q scales, atom layout (non-SFR)
    __nv_bfloat16* D;
    float alpha;
    int rows_p, rows_q;       // valid rows of P and Q
    int K;                    // elements, multiple of 64
    int ldd;                  // row stride of D in elements (= N)
    int k_tiles;              // ceil(K / 256)
    int tiles_q;              // tiles along Q; blockIdx.y = tq + tiles_q * tp
    int prefetch_b;           // B is constant: fetch its first tiles before waiting on the previous grid
    float gq;                 // QBF16: global scale of the BF16 activations
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

// The 16 scale words of one 128-row block for one K tile, in TMEM column
// order: out[4*j + r1] = scales of row L + 32*r1 for K step j.  SFR: the
// block is row-major (row r at byte 16*r, word j = step j); otherwise it is
// four atoms (atom j at byte 512*j, line L holds rows L, L+32, L+64, L+96).
template <bool SFR>
__device__ __forceinline__ void gather_scale_words(uint32_t base, int lane, uint32_t (&out)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = ld_shared_v4(SFR ? base + 16u * (lane + 32 * i) : base + 512u * i + 16u * lane);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            // SFR: i = row group r1, k = step j;  atoms: i = step j, k = row group r1
            const int j = SFR ? k : i, r1 = SFR ? i : k;
            out[4 * j + r1] = w[k];
        }
    }
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_rank_addr(uint32_t smem_addr_local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr_local), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Row stride (floats) of a partial row slot in shared memory; the +4 keeps
// the 16-byte accesses of a warp (one row per lane) free of bank conflicts.
template <int BQ>
constexpr int kPartLd = BQ + 4;

// Split-K reduction, run by the 128 epilogue threads of the owner (cluster
// rank r) after the cluster barrier: its rows_per rows, summed over the S
// slots [z][rows_per][kPartLd] in rank order, scaled by alpha and stored.
template <int BQ, bool SWAP>
__device__ __forceinline__ void reduce_owned_rows(const GemmParams& prm, uint32_t slots, int tp, int q_row0, int t) {
    const int S = (int)gridDim.x, rank = (int)blockIdx.x;
    const int rows_per = kBM / S;
    const int row0 = rank * rows_per;
    constexpr int C4 = BQ / 4;                     // float4 columns per row
    const int n4 = rows_per * C4;
    const uint32_t slot_bytes = (uint32_t)(rows_per * kPartLd<BQ>) * 4u;
    for (int i = t; i < n4; i += 128) {
        // swapped: consecutive threads take consecutive P rows (contiguous in D)
        const int r = SWAP ? (i % rows_per) : (i / C4);
        const int c4 = SWAP ? (i / rows_per) : (i % C4);
        const uint32_t off = slots + (uint32_t)(r * kPartLd<BQ> + 4 * c4) * 4u;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int z = 0; z < S; ++z) {          // rank order
            const uint4 v = ld_shared_v4(off + (uint32_t)z * slot_bytes);
            acc.x += __uint_as_float(v.x);
            acc.y += __uint_as_float(v.y);
            acc.z += __uint_as_float(v.z);
            acc.w += __uint_as_float(v.w);
        }
        const int p = tp * kBM + row0 + r;
        const int q = q_row0 + 4 * c4;
        if (p >= prm.rows_p) continue;
        const float o[4] = {acc.x * prm.alpha, acc.y * prm.alpha, acc.z * prm.alpha, acc.w * prm.alpha};
        if (!SWAP) {
            if (q < prm.rows_q)   // rows_q (= N) is a multiple of 8
                *reinterpret_cast<uint2*>(prm.D + (size_t)p * prm.ldd + q) =
                    make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (q + j < prm.rows_q) prm.D[(size_t)(q + j) * prm.ldd + p] = __float2bfloat16_rn(o[j]);
        }
    }
}

template <int BQ, bool SWAP, bool SPLITK, bool SFR, bool QBF16 = false>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmSP, const __grid_constant__ CUtensorMap tmSQ,
                      const GemmParams prm) {
    static_assert(!QBF16 || (SWAP && SFR && BQ <= 64), "BF16 activations: swapped layout, row-major scale tiles");
    using C = TileConfig<BQ, SPLITK, QBF16>;
    constexpr int S = C::STAGES;
    constexpr int NB = kScaleBuffers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // [ring: S stages][split-K receive slots][barriers]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES + C::SLOT_BYTES);
    // bars: [0,S) full, [S,2S) empty, [2S,2S+NB) sf_ready, [2S+NB] accum,
    //       [2S+NB+1] cvt (QBF16: the four writer warps quantized a K tile)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + NB + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, splits = gridDim.x;
    const int tq = blockIdx.y % prm.tiles_q, tp = blockIdx.y / prm.tiles_q;
    // even K partition: every slice non-empty while splits <= k_tiles
    const int kt_begin = (int)((long long)split * prm.k_tiles / splits);
    const int kt_end = (int)((long long)(split + 1) * prm.k_tiles / splits);
    const int steps_total = prm.K / kStepK;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t bar_base = smem_addr(bars);
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
    auto sf_ready_bar = [&](int b) { return bar_base + 8u * (2 * S + b); };
    const uint32_t accum_bar = bar_base + 8u * (2 * S + NB);
    const uint32_t cvt_bar = bar_base + 8u * (2 * S + NB + 1);

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
        for (int b = 0; b < NB; ++b) mbar_init(sf_ready_bar(b), 4);
        mbar_init(accum_bar, 1);
        mbar_init(cvt_bar, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        prefetch_tensor_map(&tmP);
        prefetch_tensor_map(&tmQ);
        if (SFR) {
            prefetch_tensor_map(&tmSP);
            prefetch_tensor_map(&tmSQ);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (SPLITK) cluster_arrive_relaxed();   // "this CTA has started" (waited on before the push)
    // Everything above overlaps the previous kernel's tail when launched with
    // programmatic stream serialisation; global memory is touched only below.
    grid_launch_dependents();
    const bool producer = (warp == 0 && lane == 0);
    if (!producer) grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            // The 128-row side is read by exactly one tile column in the
            // swapped layout (the weights): stream it; keep the shared side.
            // Swapped (small M): the weights P are read by exactly one tile
            // column -- stream them; the few activation rows Q are shared by
            // every CTA -- keep them.  Otherwise the row block P is shared by
            // the CTAs of one wave and the column block Q by every wave.
            const uint64_t pol_p = SWAP ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_q = policy_evict_last();
            // With a constant B, its first ring's worth of tiles is requested
            // before waiting for the previous grid (only B is touched then).
            // bytes of one stage: P tile + P scales + the Q side (FP4 tile and
            // scales, or the raw BF16 tile that the writers quantize)
            constexpr uint32_t kStageTx =
                C::P_BYTES + 16 * kBM + (QBF16 ? (uint32_t)C::QRAW_BYTES : (uint32_t)(C::Q_BYTES + 16 * BQ));
            auto load_q = [&](uint32_t st, uint32_t bar, int kt) {
                if (QBF16) {
                    tma_load_2d(st + C::QRAW_OFF, &tmQ, bar, kt * 256, q_row0, pol_q);
                } else {
                    tma_load_2d(st + C::P_BYTES, &tmQ, bar, kt * kStageKBytes, q_row0, pol_q);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSQ, bar, kt * 16, q_row0, pol_q);
                }
            };
            int pre = 0;
            if (SFR && prm.prefetch_b) {
                pre = min(S, kt_end - kt_begin);
                for (int i = 0; i < pre; ++i) {
                    const int kt = kt_begin + i;
                    const uint32_t st = smem_base + i * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(full_bar(i), kStageTx);
                    if (SWAP) {   // B is P
                        tma_load_2d(st, &tmP, full_bar(i), kt * kStageKBytes, tp * kBM, pol_p);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(i), kt * 16, tp * kBM, pol_p);
                    } else {      // B is Q
                        tma_load_2d(st + C::P_BYTES, &tmQ, full_bar(i), kt * kStageKBytes, q_row0, pol_q);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSQ, full_bar(i), kt * 16, q_row0,
                                    pol_q);
                    }
                }
            }
            grid_dependency_wait();
            int it = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                const uint32_t st = smem_base + s * C::STAGE_BYTES;
                if (it < pre) {   // the other operand of a prefetched stage
                    if (SWAP) {
                        load_q(st, full_bar(s), kt);
                    } else {
                        tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(s), kt * 16, tp * kBM, pol_p);
                    }
                    continue;
                }
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) break;
                if (SFR) {
                    // row-major scale tiles: 16 bytes (= 4 K steps) per row
                    mbar_arrive_expect_tx(full_bar(s), kStageTx);
                    tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(s), kt * 16, tp * kBM, pol_p);
                    load_q(st, full_bar(s), kt);
                } else {
                    const int steps = min(4, steps_total - 4 * kt);
                    const uint32_t sf_bytes = (uint32_t)steps * kAtomBytes;
                    mbar_arrive_expect_tx(full_bar(s), C::P_BYTES + C::Q_BYTES + sf_bytes * (1 + q_blocks));
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
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(kBM, BQ);
            int it = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                const int s = it % S;
                const int b = it % NB;
                // sf_ready[b] is arrived after the writers saw full[s]: the
                // operand tiles of stage s have landed as well.
                if (!mbar_wait(sf_ready_bar(b), (uint32_t)(it / NB) & 1u, abort_flag)) break;
                tc_fence_after();
                const int steps = min(4, steps_total - 4 * kt);
                const uint32_t st = smem_base + s * C::STAGE_BYTES;
                const uint32_t sf = tmem + C::SF_BASE + b * C::SF_STRIDE;
                for (int j = 0; j < steps; ++j) {
                    tc_mma_nvf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::P_BYTES + 32 * j),
                                idesc, sf + 4 * j, sf + 16 + 4 * C::Q_BLOCKS * j, (it > 0 || j > 0) ? 1u : 0u);
                }
                // one commit frees both the ring stage and the TMEM scale
                // buffer this K tile used
                tc_commit(empty_bar(s));
            }
            // Always signal the epilogue (also after an abort), and only once
            // every MMA issued above has completed.
            tc_commit(accum_bar);
        }
        __syncwarp();
    } else {
        const int quad = warp & 3;               // TMEM lane quadrant of this warp
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        // ---- scale writers: shared memory -> TMEM scale buffer, per K tile.
        // K tiles that have already landed (up to half the buffers) are
        // written before one tcgen05.wait::st, sharing the store round trip.
        {
            int it = 0;
            for (int kt = kt_begin; kt < kt_end;) {
                int got = 1, cnt = 1;
                if (lane == 0) {
                    // Scale buffer it % NB was last used by K tile it - NB; the MMA
                    // commit on that tile's ring stage (empty) also releases it.
                    // With NB <= S that barrier cannot run a phase ahead meanwhile.
                    const int s0 = it % S, j0 = it - NB;
                    got = mbar_wait(full_bar(s0), (uint32_t)(it / S) & 1u, abort_flag) &&
                          (j0 < 0 || mbar_wait(empty_bar(j0 % S), (uint32_t)(j0 / S) & 1u, abort_flag));
                    // take the following K tiles that have landed too, up to half
                    // the scale buffers, so the MMA keeps the other half busy
                    while (got && !QBF16 && cnt < NB / 2 && kt + cnt < kt_end) {
                        const int i1 = it + cnt, s1 = i1 % S, j1 = i1 - NB;
                        if (!mbar_test(full_bar(s1), (uint32_t)(i1 / S) & 1u) ||
                            (j1 >= 0 && !mbar_test(empty_bar(j1 % S), (uint32_t)(j1 / S) & 1u)))
                            break;
                        ++cnt;
                    }
                }
                if (!__shfl_sync(0xffffffffu, got, 0)) break;
                cnt = __shfl_sync(0xffffffffu, cnt, 0);
                if (QBF16) {
                    // Quantize this K tile's BF16 activations (BQ rows x 16
                    // blocks of 16) into the FP4 Q tile, in the 128-byte
                    // swizzled K-major layout the MMA descriptor reads, and
                    // their scales into the row-major scale tile; then make
                    // the writes visible to the tensor cores and wait for the
                    // other writer warps' rows.
                    const uint32_t st = smem_base + (it % S) * C::STAGE_BYTES;
                    const uint32_t raw = st + C::QRAW_OFF, qt = st + C::P_BYTES;
                    const uint32_t sq = st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES;
                    const float gq = prm.gq, six_gq = __fmul_rn(6.0f, prm.gq);
                    for (int bidx = (warp - 2) * 32 + lane; bidx < BQ * 16; bidx += 128) {
                        const int r = bidx >> 4, kb = bidx & 15;
                        float x[16];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint4 v = ld_shared_v4(raw + (uint32_t)(r * 512 + kb * 32 + 16 * h));
                            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                x[8 * h + 2 * j] = __uint_as_float(w[j] << 16);
                                x[8 * h + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                            }
                        }
                        uint32_t sc, cd[2];
                        quantize_block16(x, gq, six_gq, sc, cd);
                        const uint32_t dst = qt + (uint32_t)(r * 128 + ((((kb >> 1) ^ (r & 7)) << 4) | ((kb & 1) << 3)));
                        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst), "r"(cd[0]), "r"(cd[1]) : "memory");
                        asm volatile("st.shared.u8 [%0], %1;" ::"r"(sq + (uint32_t)(r * 16 + kb)), "h"((uint16_t)sc)
                                     : "memory");
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    int cv = 1;
                    if (lane == 0) {
                        mbar_arrive(cvt_bar);
                        cv = mbar_wait(cvt_bar, (uint32_t)it & 1u, abort_flag) ? 1 : 0;
                    }
                    if (!__shfl_sync(0xffffffffu, cv, 0)) break;
                }
                for (int u = 0; u < cnt; ++u) {
                    const int iu = it + u;
                    const uint32_t st = smem_base + (iu % S) * C::STAGE_BYTES;
                    const uint32_t sf = t_quad + C::SF_BASE + (iu % NB) * C::SF_STRIDE;
                    uint32_t wp[16];
                    gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES, lane, wp);
                    tmem_store_16(sf, wp);
                    if (C::Q_BLOCKS == 1) {
                        uint32_t wq[16];
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq);
                        tmem_store_16(sf + 16, wq);
                    } else {
                        // two 128-row blocks: step j uses columns 8j + 4*block + r1
                        uint32_t wq0[16], wq1[16], wq[32];
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq0);
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + 4 * kAtomBytes, lane,
                                                wq1);
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
                kt += cnt;
            }
        }

        // ---- epilogue (direct); the split-K epilogue follows the role branches
        int ok = 1;
        if (lane == 0) ok = mbar_wait(accum_bar, 0, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        tc_fence_after();
        if (!SPLITK && ok && !*abort_flag) {
            const int p = tp * kBM + quad * 32 + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < BQ; c0 += 16) {
                uint32_t r[16];
                tmem_load_16(t_quad + c0, r);
                tmem_wait_load();
                float v[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]) * prm.alpha;
                store_tile_chunk<BQ, SWAP>(prm, v, p, q_row0 + c0);
            }
        }
    }

    if (SPLITK) {
        if (C::OWN_SLOTS) {
            cluster_wait();   // every peer has started: its receive slots may be written
        } else {
            cluster_wait();
            cluster_sync();   // every peer is past its main loop: its ring may be written
        }
        const uint32_t slots = C::OWN_SLOTS ? smem_base + S * C::STAGE_BYTES : smem_base;
        if (warp >= 2 && !*abort_flag) {
            const int quad = warp & 3;
            const int row = quad * 32 + lane;
            const int rows_per = kBM / splits;
            const uint32_t owner = (uint32_t)(row / rows_per);
            const uint32_t local = slots + (uint32_t)((split * rows_per + row % rows_per) * kPartLd<BQ>) * 4u;
            const uint32_t dst = cluster_rank_addr(local, owner);
            const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < BQ; c0 += 16) {
                uint32_t r[16];
                tmem_load_16(t_quad + c0, r);
                tmem_wait_load();
#pragma unroll
                for (int c = 0; c < 16; c += 4)
                    st_cluster_v4(dst + 4u * (c0 + c), r[c], r[c + 1], r[c + 2], r[c + 3]);
            }
        }
        cluster_sync();   // every partial row has reached its owner; no remote access after this
        if (warp >= 2 && !*abort_flag) reduce_owned_rows<BQ, SWAP>(prm, slots, tp, q_row0, threadIdx.x - 64);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace nvfp4
