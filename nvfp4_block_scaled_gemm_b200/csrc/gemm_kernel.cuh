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
// Warp roles (192 threads, 224 where gemm_two_producers holds):
//   warp 0      TMA producer: per 256-element K tile, the P and Q operand
//               tiles (2-D TMA, 128-byte swizzle) and their scales into a
//               STAGES-deep shared-memory ring.  Scales arrive either as
//               row-major [rows][16 B] tiles (SFR: one 2-D TMA box per
//               operand) or already in 512-byte atoms (bulk copies).
//   warp 6      (gemm_two_producers only) the Q tile and its scales, so
//               that warp 0 issues only the P side.
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
// (r+1)*128/S) of the tile.  Every CTA writes its fp32 partial tile from
// registers to a global workspace (L2) with coalesced 16-byte stores; after
// one cluster barrier (release/acquire at cluster scope, which orders the
// global stores too) each owner reads its rows of all S partials back, sums
// them in rank order (deterministic), applies alpha and stores BF16 with
// 16-byte stores.  Moving the partials through L2 rather than distributed
// shared memory is several times faster per SM (measured: a 64 KB partial
// took 2.8 us to push into a peer's shared memory).
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

// Instantiations whose Q-side copies (tile and scales) come from a second
// producer warp, warp 6: one thread issuing every copy of a stage delays the
// stream when a stage's boxes are many or large.  Measured on graph-replayed
// calls with constant weights (us, one producer -> two): 512 x 768 x 6144
// (128-wide tiles) 9.63 -> 9.22, 512 x 2048 x 6144 12.79 -> 12.43, 4 and
// 8 x 8192 x 8192 (16-row swapped tiles) 14.3 -> 13.4; the 64-wide tiles lost
// about 1% (128 x 768, 256 x 2048) and the 32-row swapped tiles 0.05 us.
template <int BQ, bool SWAP, bool SFR, bool QBF16>
__host__ __device__ constexpr bool gemm_two_producers() {
    return SFR && !QBF16 && ((!SWAP && BQ >= 128) || (SWAP && BQ == 16));
}

template <int BQ, bool SWAP, bool SFR, bool QBF16>
__host__ __device__ constexpr int gemm_threads() {
    return gemm_two_producers<BQ, SWAP, SFR, QBF16>() ? kThreads + 32 : kThreads;
}
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
    static constexpr int STAGES_FIT = (kSmemLimit - 2048) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 1024;
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
    float4* ws;               // split-K partials: [tile][rank][BQ/4][128 rows] float4 (global workspace)
};

template <int BQ, bool SWAP>
__device__ __forceinline__ void store_tile_chunk(const GemmParams& prm, const float (&v)[16], int p, int q0) {
    static_assert(!SWAP, "the swapped layout is stored through shared memory");
    // v[c] is the fp32 result for (P row p, Q row q0 + c); alpha already applied.
    // D[p][q]: 16 consecutive bf16 of one row -> two 16-byte stores.
    if (p >= prm.rows_p) return;
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

// MXFP4 row-major scale box (16 bytes = two K tiles per row): move the words
// of the second K tile (2, 3) into the places of the first (0, 1) when `hi`.
// out[4 w + r1] is word w of row group r1, as gather_scale_words leaves it.
__device__ __forceinline__ void mx_box_half(uint32_t (&w)[16], bool hi) {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = hi ? w[i + 8] : w[i];
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

// Split-K partial of this CTA in the workspace: float4 index (c4 * 128 + row)
// of a [BQ/4][128] block per (tile, rank), so that the 32 lanes of a warp
// (32 consecutive rows) store 512 contiguous bytes per instruction.
template <int BQ>
__device__ __forceinline__ float4* partial_block(const GemmParams& prm, int rank) {
    return prm.ws + ((size_t)blockIdx.y * gridDim.x + rank) * (size_t)(BQ / 4) * kBM;
}

// Split-K reduction, run by the 128 epilogue threads of the owner (cluster
// rank `split`) after the cluster barrier: its rows_per rows of every rank's
// partial, summed in rank order, scaled by alpha and stored as BF16 with
// 16-byte stores.
template <int BQ, bool SWAP, int S>
__device__ __forceinline__ void reduce_from_workspace(const GemmParams& prm, int tp, int q_row0, int t) {
    const int split = (int)blockIdx.x;
    const int rows_per = kBM / S;
    const int row0 = split * rows_per;
    const int lane = t & 31;
    if (SWAP) {
        // Item (4 token columns c4, weight row r): lanes take consecutive r
        // (coalesced float4 loads); 8 consecutive r in 8 consecutive lanes,
        // whose sums lane r % 8 == i gathers for column 4 c4 + i and writes
        // as D[q][p .. p+7].  Every lane runs every shuffle (uniform loop).
        const int items = rows_per * (BQ / 4);
        for (int base = 0; base < items; base += 128) {
            const int it = base + t;
            const bool live = it < items;
            const int r = live ? it % rows_per : 0, c4 = live ? it / rows_per : 0;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (live) {
                float4 v[S];   // every rank's load in flight at once, then the sums in rank order
#pragma unroll
                for (int z = 0; z < S; ++z) v[z] = partial_block<BQ>(prm, z)[c4 * kBM + row0 + r];
#pragma unroll
                for (int z = 0; z < S; ++z) acc.x += v[z].x, acc.y += v[z].y, acc.z += v[z].z, acc.w += v[z].w;
            }
            const float a[4] = {acc.x * prm.alpha, acc.y * prm.alpha, acc.z * prm.alpha, acc.w * prm.alpha};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float g[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) g[j] = __shfl_sync(0xffffffffu, a[i], (lane & ~7) | j);
                const int q = q_row0 + 4 * c4 + i, p = tp * kBM + row0 + r;
                if (live && (r & 7) == i && rows_per >= 8 && q < prm.rows_q && p - i < prm.rows_p) {
                    uint4 w;
                    w.x = pack_bf16x2(g[0], g[1]);
                    w.y = pack_bf16x2(g[2], g[3]);
                    w.z = pack_bf16x2(g[4], g[5]);
                    w.w = pack_bf16x2(g[6], g[7]);
                    *reinterpret_cast<uint4*>(prm.D + (size_t)q * prm.ldd + (p - i)) = w;   // p - i: the group's first row
                }
            }
            if (rows_per < 8 && live) {   // fewer than 8 owned rows: one BF16 per element
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int q = q_row0 + 4 * c4 + i, p = tp * kBM + row0 + r;
                    if (q < prm.rows_q && p < prm.rows_p) prm.D[(size_t)q * prm.ldd + p] = __float2bfloat16_rn(a[i]);
                }
            }
        }
    } else {
        // Item (token row r, 8 weight columns c8): two float4 per rank,
        // one 16-byte store of D[p][q .. q+7]; lanes take consecutive r.
        // With up to four ranks a thread has two items' loads in flight (every
        // rank's, issued together), halving the round trips to L2.
        constexpr int U = S <= 4 ? 2 : 1;
        const int items = rows_per * (BQ / 8);
        for (int base = t; base < items; base += 128 * U) {
            float4 a[U][S], b[U][S];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int it = base + 128 * u;
                if (it < items) {
                    const int r = it % rows_per, c8 = it / rows_per;
#pragma unroll
                    for (int z = 0; z < S; ++z) {
                        const float4* blk = partial_block<BQ>(prm, z);
                        a[u][z] = blk[(2 * c8) * kBM + row0 + r];
                        b[u][z] = blk[(2 * c8 + 1) * kBM + row0 + r];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int it = base + 128 * u;
                if (it >= items) break;
                const int r = it % rows_per, c8 = it / rows_per;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
                for (int z = 0; z < S; ++z) {   // rank order
                    acc[0] += a[u][z].x, acc[1] += a[u][z].y, acc[2] += a[u][z].z, acc[3] += a[u][z].w;
                    acc[4] += b[u][z].x, acc[5] += b[u][z].y, acc[6] += b[u][z].z, acc[7] += b[u][z].w;
                }
                const int p = tp * kBM + row0 + r, q = q_row0 + 8 * c8;
                if (p < prm.rows_p && q < prm.rows_q) {   // rows_q (= N) is a multiple of 8
                    uint4 w;
                    w.x = pack_bf16x2(acc[0] * prm.alpha, acc[1] * prm.alpha);
                    w.y = pack_bf16x2(acc[2] * prm.alpha, acc[3] * prm.alpha);
                    w.z = pack_bf16x2(acc[4] * prm.alpha, acc[5] * prm.alpha);
                    w.w = pack_bf16x2(acc[6] * prm.alpha, acc[7] * prm.alpha);
                    *reinterpret_cast<uint4*>(prm.D + (size_t)p * prm.ldd + q) = w;
                }
            }
        }
    }
}

// MX: the MXFP4 form (E8M0 scale per 32 values, kind::mxf4 block32): a K
// tile has 8 scale bytes per row, two TMEM words (steps 0-1, 2-3), and step
// j reads word j / 2 at byte 2 * (j % 2).  Without SFR the scales come
// pre-laid out in 512-byte atoms of two K steps each (two per 128-row block
// and K tile).  With SFR they are row-major [rows][K/32] (K % 512 == 0): a
// TMA box starts on a 16-byte boundary, so K tile kt loads the 16-byte box of
// K tiles kt & ~1 and kt | 1, and the writers take its half kt % 2.
template <int BQ, bool SWAP, bool SPLITK, bool SFR, bool QBF16 = false, bool MX = false>
__global__ void __launch_bounds__(gemm_threads<BQ, SWAP, SFR, QBF16>(), 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmSP, const __grid_constant__ CUtensorMap tmSQ,
                      const GemmParams prm) {
    static_assert(!QBF16 || (SWAP && SFR && BQ <= 64), "BF16 activations: swapped layout, row-major scale tiles");
    static_assert(!MX || !QBF16, "MXFP4: FP4 activations");
    using C = TileConfig<BQ, SPLITK, QBF16>;
    constexpr int S = C::STAGES;
    constexpr int NB = kScaleBuffers;
    constexpr bool TWO = gemm_two_producers<BQ, SWAP, SFR, QBF16>();   // warp 6 loads the Q side
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // [ring: S stages][split-K receive slots][barriers]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
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
            mbar_init(full_bar(s), TWO ? 2 : 1);   // the producer warp(s)
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
    // Everything above overlaps the previous kernel's tail when launched with
    // programmatic stream serialisation; global memory is touched only below.
    grid_launch_dependents();
    const bool producer = ((warp == 0 || (TWO && warp == 6)) && lane == 0);
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
            // x (bytes) of K tile kt's row-major scale box: 16 scale bytes
            // per K tile (NVFP4), or the 16 bytes of K tiles kt & ~1, kt | 1 (MXFP4)
            auto sf_x = [](int kt) { return MX ? 16 * (kt >> 1) : 16 * kt; };
            // With a constant B, its first ring's worth of tiles is requested
            // before waiting for the previous grid (only B is touched then).
            // bytes of one stage from this warp: P tile + P scales, and (one
            // producer) the Q side: FP4 tile and scales, or the raw BF16 tile
            // that the writers quantize
            constexpr uint32_t kStageTx =
                C::P_BYTES + 16 * kBM +
                (TWO ? 0u : QBF16 ? (uint32_t)C::QRAW_BYTES : (uint32_t)(C::Q_BYTES + 16 * BQ));
            auto load_q = [&](uint32_t st, uint32_t bar, int kt) {
                if (QBF16) {
                    tma_load_2d(st + C::QRAW_OFF, &tmQ, bar, kt * 256, q_row0, pol_q);
                } else {
                    tma_load_2d(st + C::P_BYTES, &tmQ, bar, kt * kStageKBytes, q_row0, pol_q);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSQ, bar, sf_x(kt), q_row0, pol_q);
                }
            };
            int pre = 0;
            if (SFR && prm.prefetch_b && (SWAP || !TWO)) {   // B is P, or this warp also loads Q = B
                pre = min(S, kt_end - kt_begin);
                for (int i = 0; i < pre; ++i) {
                    const int kt = kt_begin + i;
                    const uint32_t st = smem_base + i * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(full_bar(i), kStageTx);
                    if (SWAP) {   // B is P
                        tma_load_2d(st, &tmP, full_bar(i), kt * kStageKBytes, tp * kBM, pol_p);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(i), sf_x(kt), tp * kBM, pol_p);
                    } else {      // B is Q
                        tma_load_2d(st + C::P_BYTES, &tmQ, full_bar(i), kt * kStageKBytes, q_row0, pol_q);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSQ, full_bar(i), sf_x(kt), q_row0,
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
                        if (!TWO) load_q(st, full_bar(s), kt);
                    } else {
                        tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                        tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(s), sf_x(kt), tp * kBM, pol_p);
                    }
                    continue;
                }
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) break;
                if (SFR) {
                    // row-major scale tiles: 16 bytes (= 4 K steps) per row
                    mbar_arrive_expect_tx(full_bar(s), kStageTx);
                    tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                    tma_load_2d(st + C::P_BYTES + C::Q_BYTES, &tmSP, full_bar(s), sf_x(kt), tp * kBM, pol_p);
                    if (!TWO) load_q(st, full_bar(s), kt);
                } else {
                    // atoms per 128-row block: one per K step (NVFP4) or per
                    // pair of K steps (MXFP4)
                    const int steps = min(4, steps_total - 4 * kt);
                    const int atoms_total = MX ? (steps_total + 1) / 2 : steps_total;
                    const int atom0 = MX ? 2 * kt : 4 * kt;
                    const uint32_t sf_bytes = (uint32_t)(MX ? (steps + 1) / 2 : steps) * kAtomBytes;
                    mbar_arrive_expect_tx(full_bar(s), C::P_BYTES + C::Q_BYTES + sf_bytes * (1 + q_blocks));
                    tma_load_2d(st, &tmP, full_bar(s), kt * kStageKBytes, tp * kBM, pol_p);
                    tma_load_2d(st + C::P_BYTES, &tmQ, full_bar(s), kt * kStageKBytes, q_row0, pol_q);
                    bulk_load(st + C::P_BYTES + C::Q_BYTES,
                              prm.sfp + ((size_t)tp * atoms_total + atom0) * kAtomBytes, sf_bytes, full_bar(s));
                    for (int b = 0; b < q_blocks; ++b) {
                        bulk_load(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + b * 4 * kAtomBytes,
                                  prm.sfq + ((size_t)(q_block0 + b) * atoms_total + atom0) * kAtomBytes, sf_bytes,
                                  full_bar(s));
                    }
                }
            }
        }
    } else if (TWO && warp == 6) {
        // ---- Q-side producer: the Q tile and its row-major scale box per K
        // tile, on the same stage barriers (each stage expects both warps)
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_last();
            auto sf_x = [](int kt) { return MX ? 16 * (kt >> 1) : 16 * kt; };
            constexpr uint32_t kQTx = C::Q_BYTES + 16 * BQ;
            auto load_q = [&](int i, int kt) {
                const uint32_t st = smem_base + (i % S) * C::STAGE_BYTES;
                mbar_arrive_expect_tx(full_bar(i % S), kQTx);
                tma_load_2d(st + C::P_BYTES, &tmQ, full_bar(i % S), kt * kStageKBytes, q_row0, pol_q);
                tma_load_2d(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, &tmSQ, full_bar(i % S), sf_x(kt), q_row0,
                            pol_q);
            };
            // a constant B on the Q side (not swapped): its first ring's worth
            // of tiles before the wait for the previous grid
            int pre = 0;
            if (!SWAP && prm.prefetch_b) {
                pre = min(S, kt_end - kt_begin);
                for (int i = 0; i < pre; ++i) load_q(i, kt_begin + i);
            }
            grid_dependency_wait();
            int it = pre;
            for (int kt = kt_begin + pre; kt < kt_end; ++kt, ++it) {
                if (!mbar_wait(empty_bar(it % S), ((uint32_t)(it / S) & 1u) ^ 1u, abort_flag)) break;
                load_q(it, kt);
            }
        }
        __syncwarp();
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
                // A whole K tile: its four MMAs unrolled, with nothing between
                // them (measured: an MMA loop with a run-time trip count and a
                // barrier wait in the same loop issues one MMA per ~110 ns,
                // against ~35 ns when the MMAs stand alone).
                if (!MX && steps == 4) {
                    const uint64_t dp = desc_kmajor_sw128(st), dq = desc_kmajor_sw128(st + C::P_BYTES);
                    const uint32_t acc0 = it > 0 ? 1u : 0u;
                    tc_mma_nvf4(tmem, dp, dq, idesc, sf, sf + 16, acc0);
                    tc_mma_nvf4(tmem, dp + 2u, dq + 2u, idesc, sf + 4, sf + 16 + 4 * C::Q_BLOCKS, 1u);
                    tc_mma_nvf4(tmem, dp + 4u, dq + 4u, idesc, sf + 8, sf + 16 + 8 * C::Q_BLOCKS, 1u);
                    tc_mma_nvf4(tmem, dp + 6u, dq + 6u, idesc, sf + 12, sf + 16 + 12 * C::Q_BLOCKS, 1u);
                    tc_commit(empty_bar(s));
                    continue;
                }
                if (MX && steps == 4) {
                    // steps 2w and 2w + 1 share scale word w, bytes 0-1 and 2-3
                    const uint64_t dp = desc_kmajor_sw128(st), dq = desc_kmajor_sw128(st + C::P_BYTES);
                    constexpr uint32_t id0 = idesc_mxf4(kBM, BQ, 0), id2 = idesc_mxf4(kBM, BQ, 2);
                    const uint32_t acc0 = it > 0 ? 1u : 0u;
                    tc_mma_mxf4(tmem, dp, dq, id0, sf, sf + 16, acc0);
                    tc_mma_mxf4(tmem, dp + 2u, dq + 2u, id2, sf, sf + 16, 1u);
                    tc_mma_mxf4(tmem, dp + 4u, dq + 4u, id0, sf + 4, sf + 16 + 4 * C::Q_BLOCKS, 1u);
                    tc_mma_mxf4(tmem, dp + 6u, dq + 6u, id2, sf + 4, sf + 16 + 4 * C::Q_BLOCKS, 1u);
                    tc_commit(empty_bar(s));
                    continue;
                }
                for (int j = 0; j < steps; ++j) {
                    if (MX) {
                        // the atoms' word (j / 2) landed in TMEM column group j / 2
                        tc_mma_mxf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::P_BYTES + 32 * j),
                                    (j & 1) ? idesc_mxf4(kBM, BQ, 2) : idesc_mxf4(kBM, BQ, 0), sf + 4 * (j >> 1),
                                    sf + 16 + 4 * C::Q_BLOCKS * (j >> 1), (it > 0 || j > 0) ? 1u : 0u);
                    } else {
                        tc_mma_nvf4(tmem, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::P_BYTES + 32 * j),
                                    idesc, sf + 4 * j, sf + 16 + 4 * C::Q_BLOCKS * j, (it > 0 || j > 0) ? 1u : 0u);
                    }
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
    } else if (warp < 6) {
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
                    // MXFP4 row-major: this K tile's two words are words 2h, 2h + 1 of the box
                    const bool hi = MX && SFR && ((kt_begin + iu) & 1);
                    uint32_t wp[16];
                    gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES, lane, wp);
                    mx_box_half(wp, hi);
                    tmem_store_16(sf, wp);
                    if (C::Q_BLOCKS == 1) {
                        uint32_t wq[16];
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq);
                        mx_box_half(wq, hi);
                        tmem_store_16(sf + 16, wq);
                    } else {
                        // two 128-row blocks: step j uses columns 8j + 4*block + r1
                        uint32_t wq0[16], wq1[16], wq[32];
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES, lane, wq0);
                        gather_scale_words<SFR>(st + C::P_BYTES + C::Q_BYTES + C::SFP_BYTES + 4 * kAtomBytes, lane,
                                                wq1);
                        mx_box_half(wq0, hi);
                        mx_box_half(wq1, hi);
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
                if (!SWAP) {
                    store_tile_chunk<BQ, false>(prm, v, p, q_row0 + c0);
                } else {
                    // D[q][p]: the warp's 32 rows p x 16 columns q go through
                    // shared memory (stage 0, free once every MMA is done and
                    // nothing else reads it) and leave as 16-byte pieces of 8
                    // consecutive p.
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
                        const int q = q_row0 + c0 + c, pp = tp * kBM + quad * 32 + part * 8;
                        const uint4 val = ld_shared_v4(tb + (uint32_t)(c * 64 + part * 16));
                        if (q < prm.rows_q && pp < prm.rows_p)   // rows_p (= N) is a multiple of 8
                            *reinterpret_cast<uint4*>(prm.D + (size_t)q * prm.ldd + pp) = val;
                    }
                    __syncwarp();
                }
            }
        }
    }

    if (SPLITK) {
        // Partial tile -> workspace (after the grid dependency wait, which
        // every epilogue thread passed at the start), one cluster barrier,
        // then each owner's sum.
        if (warp >= 2 && warp < 6 && !*abort_flag) {
            const int quad = warp & 3;
            const int row = quad * 32 + lane;
            float4* dst = partial_block<BQ>(prm, split);
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
        if (warp >= 2 && warp < 6 && !*abort_flag) {
            const int t = threadIdx.x - 64;
            switch (splits) {
                case 2: reduce_from_workspace<BQ, SWAP, 2>(prm, tp, q_row0, t); break;
                case 4: reduce_from_workspace<BQ, SWAP, 4>(prm, tp, q_row0, t); break;
                case 8: reduce_from_workspace<BQ, SWAP, 8>(prm, tp, q_row0, t); break;
                default: reduce_from_workspace<BQ, SWAP, 16>(prm, tp, q_row0, t); break;
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
