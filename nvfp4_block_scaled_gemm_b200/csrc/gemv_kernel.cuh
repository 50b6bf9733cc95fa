// NVFP4 GEMM for a handful of activation rows (decode, M <= 16) on the CUDA
// cores.
//
// With one to a few token rows the GEMM is a matrix-vector product: two
// FLOPs per weight element read, so it is bound by the weight bytes (small-
// batch decode is memory-bound: "The SM120 FP4 Kernel Disaster", section
// "Finding 4: Memory Bandwidth Is the Real Wall"; the batch-1 attention and
// MoE projections are the first shapes measured in "Peeling the Kernel
// Onion", section "The Chain of Reasoning"), and a 3 MB weight matrix is half
// a microsecond of HBM time.  The
// tensor-core kernels spend several microseconds per call in hand-offs
// (tensor map fetch, TMA, TMEM scale stores, MMA, split-K exchange through
// distributed shared memory); this kernel has none of them: every thread
// loads its 16-byte chunks of the weight rows straight into registers, with
// all of a CTA's loads in flight at once, decodes them and accumulates.
//
// Arithmetic, exact up to the fp32 sum over blocks:
//   * E2M1 pairs decode to f16x2 (cvt.rn.f16x2.e2m1x2); the two halves of an
//     fma.rn.f16x2 chain over the 8 bytes of a 16-value block add up the 8
//     even and the 8 odd products.  Each product is a multiple of 1/4 of at
//     most 36 in magnitude, so each half stays a multiple of 1/4 below 288,
//     which f16 holds exactly: no rounding anywhere in the block.
//   * The block sum (the two halves in fp32, exact) times sA * sB (two E4M3
//     values, an exact fp32 product) is exact as well; one fp32 fma per block
//     adds it to the running sum.  Only that sum over K/16 blocks rounds.
//   * The CTA's per-thread sums are added in a fixed order (a butterfly over
//     the warp, then the four warps in turn), so results are deterministic;
//     alpha is applied in fp32 and the result rounded to BF16 (RNE).
//
// Work split: a CTA of 128 threads takes RW consecutive weight rows (output
// columns n) at a time, with all M token rows; its threads take the K chunks
// of 32 values (16 bytes, two scale blocks) round-robin, so consecutive
// threads read consecutive 16-byte pieces of each row.  The activations (M
// rows, a few KB) are read through L1 by every CTA.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int kGemvThreads = 128;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvGroup = 2;   // K chunks per thread whose loads are issued together

struct GemvParams {
    const uint8_t* A;    // [M][K/2] E2M1 codes
    const uint8_t* sA;   // [M][K/16] E4M3 scales
    const uint8_t* B;    // [N][K/2]
    const uint8_t* sB;   // [N][K/16]
    __nv_bfloat16* D;    // [M][N]
    float alpha;
    int M, N, K;
    int prefetch_b;      // B is constant: load its first chunks before waiting on the previous grid
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_cached_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_cached_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Four bytes of E2M1 pairs -> four f16x2 (byte i -> h[i], element 2i in the
// low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// 16 code bytes (32 values, two blocks) -> 16 f16x2.
__device__ __forceinline__ void decode_chunk(const uint4& c, uint32_t (&h)[16]) {
    uint32_t t[4];
    e2m1x8_to_f16x2(c.x, t);
    h[0] = t[0], h[1] = t[1], h[2] = t[2], h[3] = t[3];
    e2m1x8_to_f16x2(c.y, t);
    h[4] = t[0], h[5] = t[1], h[6] = t[2], h[7] = t[3];
    e2m1x8_to_f16x2(c.z, t);
    h[8] = t[0], h[9] = t[1], h[10] = t[2], h[11] = t[3];
    e2m1x8_to_f16x2(c.w, t);
    h[12] = t[0], h[13] = t[1], h[14] = t[2], h[15] = t[3];
}

// E4M3 byte -> its exact float value (the sign bit honoured).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
    const float v = e == 0 ? (float)m * 0.001953125f                       // m * 2^-9
                           : __uint_as_float(((e + 120u) << 23) | (m << 20));   // (1 + m/8) 2^(e-7)
    return (b & 0x80u) ? -v : v;
}

// The two halves of an f16x2 summed in fp32 (exact for these sums): the low
// half converted, the high half added to it by a mixed f16 + f32 add.
__device__ __forceinline__ float half2_sum_f32(__half2 s) {
    const float lo = __low2float(s);
    const unsigned short hi = __half_as_ushort(__high2half(s));
    float r;
    asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(r) : "h"(hi), "f"(lo));
    return r;
}

// Exact sum of the 16 products of one block: 8 f16x2 of each operand.
__device__ __forceinline__ float block_dot(const uint32_t* a, const uint32_t* b) {
    __half2 s = __hmul2(*reinterpret_cast<const __half2*>(&a[0]), *reinterpret_cast<const __half2*>(&b[0]));
#pragma unroll
    for (int i = 1; i < 8; ++i)
        s = __hfma2(*reinterpret_cast<const __half2*>(&a[i]), *reinterpret_cast<const __half2*>(&b[i]), s);
    return half2_sum_f32(s);
}

// Sum NV per-thread values over the warp.  Each step halves the values a
// lane keeps (the lane with the step's bit set keeps the upper half) until
// one is left, then adds across the remaining lane bits.  On return lane l
// holds, in v[j] for j < max(NV / 32, 1), the warp total of value
// gemv_reduced_index<NV>(l, j).
template <int NV>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[NV], int lane) {
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int o = 16 >> s;
        const int C = NV >> s;   // values still held (a constant once unrolled)
        if (C > 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int j = 0; j < C / 2; ++j) {
                const float send = upper ? v[j] : v[j + C / 2];
                const float keep = upper ? v[j + C / 2] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
}

template <int NV>
__device__ __forceinline__ int gemv_reduced_index(int lane, int j) {
    int idx = j;
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int C = NV >> s;
        if (C > 1 && (lane & (16 >> s))) idx += C / 2;
    }
    return idx;
}

// Lanes that write a reduced value: with NV < 32 each total sits in 32 / NV
// lanes, and the one whose low lane bits are zero writes it.
template <int NV>
__device__ __forceinline__ bool gemv_writer_lane(int lane) {
    if (NV >= 32) return true;
    constexpr int dup = NV >= 32 ? 1 : 32 / NV;
    return (lane & (dup - 1)) == 0;
}

// MT: token rows the instance can hold (M <= MT); RW: weight rows per CTA
// and row group.  The grid is at most as many CTAs as are resident at once;
// each walks the row groups n0 = RW * (blockIdx.x + i * gridDim.x), and the
// first weight chunks of its next group are requested before the current
// group's reduction and store.
template <int MT, int RW>
__global__ void __launch_bounds__(kGemvThreads) nvfp4_gemv_kernel(const GemvParams prm) {
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];   // alternate row groups: one barrier per group
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;                        // 16-byte chunks per row
    const size_t row_bytes = (size_t)prm.K >> 1;      // code bytes per row
    const size_t srow_bytes = (size_t)prm.K >> 4;     // scale bytes per row
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;

    // the weight rows of a row group; rows past N (never, with N % 8 == 0
    // and RW <= 4) read row N - 1 and are not stored
    const uint8_t* brow[RW];
    const uint8_t* bsrow[RW];
    auto set_rows = [&](int n0) {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int n = min(n0 + r, prm.N - 1);
            brow[r] = prm.B + (size_t)n * row_bytes;
            bsrow[r] = prm.sB + (size_t)n * srow_bytes;
        }
    };

    // Weight chunks in flight: the group being decoded and the next one,
    // whose loads are issued before the current group's arithmetic.
    uint4 bq[kGemvGroup][RW], nq[kGemvGroup][RW];
    uint32_t bs[kGemvGroup][RW], ns[kGemvGroup][RW];
    auto load_group = [&](uint4 (&q)[kGemvGroup][RW], uint32_t (&sc)[kGemvGroup][RW], int c0) {
#pragma unroll
        for (int g = 0; g < kGemvGroup; ++g) {
            const int c = c0 + g * kGemvThreads;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                if (c < kc) {
                    q[g][r] = ld_stream_v4(brow[r] + 16 * (size_t)c);
                    sc[g][r] = ld_stream_u16(bsrow[r] + 2 * (size_t)c);
                } else {
                    q[g][r] = make_uint4(0u, 0u, 0u, 0u);
                    sc[g][r] = 0u;
                }
            }
        }
    };

    grid_launch_dependents();
    const int step = kGemvGroup * kGemvThreads;
    int n0 = blockIdx.x * RW;
    set_rows(n0);
    if (prm.prefetch_b) load_group(bq, bs, t);   // only B is touched before the wait
    grid_dependency_wait();
    if (!prm.prefetch_b) load_group(bq, bs, t);

    for (int it = 0; n0 < prm.N; n0 += group_stride, ++it) {
        float acc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

        for (int c0 = t; c0 < kc; c0 += step) {
            const bool more = c0 + step < kc;
            if (more) load_group(nq, ns, c0 + step);
#pragma unroll
            for (int g = 0; g < kGemvGroup; ++g) {
                const int c = c0 + g * kGemvThreads;
                if (c >= kc) break;
                uint32_t bh[RW][16];
                float sb0[RW], sb1[RW];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    decode_chunk(bq[g][r], bh[r]);
                    sb0[r] = e4m3_value(bs[g][r] & 0xFFu);
                    sb1[r] = e4m3_value(bs[g][r] >> 8);
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const uint4 aq = ld_cached_v4(prm.A + (size_t)m * row_bytes + 16 * (size_t)c);
                        const uint32_t as = ld_cached_u16(prm.sA + (size_t)m * srow_bytes + 2 * (size_t)c);
                        uint32_t ah[16];
                        decode_chunk(aq, ah);
                        const float sa0 = e4m3_value(as & 0xFFu), sa1 = e4m3_value(as >> 8);
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            acc[r][m] = fmaf(block_dot(ah, bh[r]), sa0 * sb0[r], acc[r][m]);
                            acc[r][m] = fmaf(block_dot(ah + 8, bh[r] + 8), sa1 * sb1[r], acc[r][m]);
                        }
                    }
                }
            }
            if (more) {
#pragma unroll
                for (int g = 0; g < kGemvGroup; ++g)
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        bq[g][r] = nq[g][r];
                        bs[g][r] = ns[g][r];
                    }
            }
        }

        // the next row group's first chunks, in flight during this group's
        // reduction and store
        const int n_next = n0 + group_stride;
        if (n_next < prm.N) {
            set_rows(n_next);
            load_group(bq, bs, t);
        }

        float v[NV];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[r * MT + m] = acc[r][m];
        warp_reduce_scatter<NV>(v, lane);
        float (*rb)[NV] = red[it & 1];
        if (gemv_writer_lane<NV>(lane)) {
#pragma unroll
            for (int j = 0; j < (NV >= 32 ? NV / 32 : 1); ++j) rb[warp][gemv_reduced_index<NV>(lane, j)] = v[j];
        }
        // Also orders this group's reads of red[it & 1] before the writes of
        // group it + 2 (every thread passes the barrier of group it + 1 first).
        __syncthreads();
        for (int i = t; i < NV; i += kGemvThreads) {
            const int r = i / MT, m = i % MT;
            if (m < M && n0 + r < prm.N) {
                float s = rb[0][i];
#pragma unroll
                for (int w = 1; w < kGemvWarps; ++w) s += rb[w][i];
                prm.D[(size_t)m * prm.N + n0 + r] = __float2bfloat16_rn(s * prm.alpha);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// One or two token rows: the same work split and arithmetic with fewer
// instructions per weight chunk, which is what bounds the kernel above on
// large weight matrices (about 100 warp instructions per 32-value chunk and
// row, issue ~60% busy, at 8192 x 8192).
//   * Each thread's K chunks of the token rows (CPT of them: c = t + 128 j)
//     are decoded once, before the first row group, and kept as f16x2 with
//     their scales as fp32: the row groups only decode weights.
//   * A weight chunk's two E4M3 scales become an f16x2 in one conversion
//     (every E4M3 value is an f16 value), then two fp32 values.
//   * All CPT chunks of every row of a group are loaded at once; the next
//     group's loads are issued before this group's reduction and store.
// The per-block arithmetic is the kernel above's (exact block sums, an exact
// fp32 scale product, one fp32 fma per block, chunks in the same order per
// thread, the same warp and CTA reduction), so the results are identical.
__device__ __forceinline__ uint32_t ld_stream_b16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.b16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Two E4M3 bytes (low byte: the first block) -> their exact values.
__device__ __forceinline__ float2 e4m3x2_values(uint32_t two) {
    uint32_t h;
    const unsigned short v = (unsigned short)two;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Resident CTAs per SM asked of the register allocator (__launch_bounds__
// minimum): two token rows (64 registers of decoded chunks) four, or three
// with 4-row groups; one row with up to two chunks per thread four (the
// 4-row form then takes 94 registers, so five fit; asking for five made it
// spill).
template <int MT, int RW, int CPT>
constexpr int gemv_areg_min_ctas() {
    return MT == 2 ? (RW * CPT >= 8 ? 3 : 4) : (CPT <= 2 ? 4 : 1);
}

template <int MT, int RW, int CPT>
__global__ void __launch_bounds__(kGemvThreads, gemv_areg_min_ctas<MT, RW, CPT>())
    nvfp4_gemv_areg_kernel(const GemvParams prm) {
    static_assert(MT * CPT <= 4, "token chunks held in registers");
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;
    const size_t row_bytes = (size_t)prm.K >> 1;
    const size_t srow_bytes = (size_t)prm.K >> 4;
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;
    // chunks this thread owns: t, t + 128, ... below kc
    int nch = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) nch += (t + j * kGemvThreads < kc) ? 1 : 0;

    uint4 bq[CPT][RW];
    uint32_t bs[CPT][RW];
    auto load_group = [&](int n0) {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int n = min(n0 + r, prm.N - 1);
            const uint8_t* br = prm.B + (size_t)n * row_bytes + 16 * (size_t)t;
            const uint8_t* bsr = prm.sB + (size_t)n * srow_bytes + 2 * (size_t)t;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                if (j < nch) {
                    bq[j][r] = ld_stream_v4(br + 16 * (size_t)(j * kGemvThreads));
                    bs[j][r] = ld_stream_b16(bsr + 2 * (size_t)(j * kGemvThreads));
                } else {
                    bq[j][r] = make_uint4(0u, 0u, 0u, 0u);
                    bs[j][r] = 0u;
                }
            }
        }
    };

    grid_launch_dependents();
    int n0 = blockIdx.x * RW;
    if (prm.prefetch_b) load_group(n0);   // only B is touched before the wait
    grid_dependency_wait();

    uint32_t ah[MT][CPT][16];
    float sa[MT][CPT][2];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + j * kGemvThreads;
            if (m < M && j < nch) {
                decode_chunk(ld_cached_v4(prm.A + (size_t)m * row_bytes + 16 * (size_t)c), ah[m][j]);
                const float2 v = e4m3x2_values(ld_cached_u16(prm.sA + (size_t)m * srow_bytes + 2 * (size_t)c));
                sa[m][j][0] = v.x;
                sa[m][j][1] = v.y;
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) ah[m][j][i] = 0u;
                sa[m][j][0] = sa[m][j][1] = 0.0f;
            }
        }
    if (!prm.prefetch_b) load_group(n0);

    for (int it = 0; n0 < prm.N; n0 += group_stride, ++it) {
        float acc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            if (j >= nch) break;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                uint32_t bh[16];
                decode_chunk(bq[j][r], bh);
                const float2 sb = e4m3x2_values(bs[j][r]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        acc[r][m] = fmaf(block_dot(ah[m][j], bh), sa[m][j][0] * sb.x, acc[r][m]);
                        acc[r][m] = fmaf(block_dot(ah[m][j] + 8, bh + 8), sa[m][j][1] * sb.y, acc[r][m]);
                    }
                }
            }
        }
        // the next row group's chunks, in flight during this group's reduction and store
        const int n_next = n0 + group_stride;
        if (n_next < prm.N) load_group(n_next);

        float v[NV];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[r * MT + m] = acc[r][m];
        warp_reduce_scatter<NV>(v, lane);
        float (*rb)[NV] = red[it & 1];
        if (gemv_writer_lane<NV>(lane)) {
#pragma unroll
            for (int j = 0; j < (NV >= 32 ? NV / 32 : 1); ++j) rb[warp][gemv_reduced_index<NV>(lane, j)] = v[j];
        }
        __syncthreads();   // also orders group it's reads of red[it & 1] before group it + 2's writes
        for (int i = t; i < NV; i += kGemvThreads) {
            const int r = i / MT, m = i % MT;
            if (m < M && n0 + r < prm.N) {
                float s = rb[0][i];
#pragma unroll
                for (int w = 1; w < kGemvWarps; ++w) s += rb[w][i];
                prm.D[(size_t)m * prm.N + n0 + r] = __float2bfloat16_rn(s * prm.alpha);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// MXFP4 (OCP microscaling: E2M1 values, one E8M0 scale 2^(byte - 127) per 32
// values) for a handful of token rows, on the CUDA cores.  A 16-byte chunk of
// codes is exactly one scale block, so each thread reads one scale byte per
// chunk and operand.  The chunk's 32 products are summed exactly as in the
// NVFP4 kernel (two f16x2 chains of 16 values, each exact, added in fp32),
// then scaled by 2^(ea + eb - 254) with ldexpf (exact while the result is an
// fp32 number) and added to the fp32 sum over chunks; the CTA's sums meet in
// a fixed order.  No prefetch across row groups: the decode shapes have one
// or two groups per CTA.
struct GemvMxParams {
    const uint8_t* A;    // [M][K/2] E2M1 codes
    const uint8_t* sA;   // [M][K/32] E8M0 scales
    const uint8_t* B;    // [N][K/2]
    const uint8_t* sB;   // [N][K/32]
    __nv_bfloat16* D;    // [M][N]
    float alpha;
    int M, N, K;
    int prefetch_b;      // B is constant: load its first chunks before waiting on the previous grid
};

__device__ __forceinline__ uint32_t ld_stream_u8(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

template <int MT, int RW>
__global__ void __launch_bounds__(kGemvThreads) nvfp4_gemv_mx_kernel(const GemvMxParams prm) {
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;                        // 16-byte chunks (= scale blocks) per row
    const size_t row_bytes = (size_t)prm.K >> 1;
    const size_t srow_bytes = (size_t)prm.K >> 5;
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;

    uint4 bq[kGemvGroup][RW];
    uint32_t bs[kGemvGroup][RW];
    auto load_group = [&](int n0, int c0) {
#pragma unroll
        for (int g = 0; g < kGemvGroup; ++g) {
            const int c = c0 + g * kGemvThreads;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int n = min(n0 + r, prm.N - 1);
                if (c < kc) {
                    bq[g][r] = ld_stream_v4(prm.B + (size_t)n * row_bytes + 16 * (size_t)c);
                    bs[g][r] = ld_stream_u8(prm.sB + (size_t)n * srow_bytes + (size_t)c);
                } else {
                    bq[g][r] = make_uint4(0u, 0u, 0u, 0u);
                    bs[g][r] = 127u;
                }
            }
        }
    };

    grid_launch_dependents();
    const int step = kGemvGroup * kGemvThreads;
    int n0 = blockIdx.x * RW;
    if (prm.prefetch_b && n0 < prm.N) load_group(n0, t);   // only B is touched before the wait
    grid_dependency_wait();

    for (int it = 0; n0 < prm.N; n0 += group_stride, ++it) {
        float acc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
        for (int c0 = t; c0 < kc; c0 += step) {
            if (!(it == 0 && c0 == t && prm.prefetch_b)) load_group(n0, c0);
#pragma unroll
            for (int g = 0; g < kGemvGroup; ++g) {
                const int c = c0 + g * kGemvThreads;
                if (c >= kc) break;
                uint32_t bh[RW][16];
#pragma unroll
                for (int r = 0; r < RW; ++r) decode_chunk(bq[g][r], bh[r]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const uint4 aq = ld_cached_v4(prm.A + (size_t)m * row_bytes + 16 * (size_t)c);
                        const int ea = (int)__ldg(prm.sA + (size_t)m * srow_bytes + (size_t)c);
                        uint32_t ah[16];
                        decode_chunk(aq, ah);
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const float blk = block_dot(ah, bh[r]) + block_dot(ah + 8, bh[r] + 8);   // exact
                            acc[r][m] += ldexpf(blk, ea + (int)bs[g][r] - 254);
                        }
                    }
                }
            }
        }

        float v[NV];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[r * MT + m] = acc[r][m];
        warp_reduce_scatter<NV>(v, lane);
        float (*rb)[NV] = red[it & 1];
        if (gemv_writer_lane<NV>(lane)) {
#pragma unroll
            for (int j = 0; j < (NV >= 32 ? NV / 32 : 1); ++j) rb[warp][gemv_reduced_index<NV>(lane, j)] = v[j];
        }
        __syncthreads();
        for (int i = t; i < NV; i += kGemvThreads) {
            const int r = i / MT, m = i % MT;
            if (m < M && n0 + r < prm.N) {
                float sum = rb[0][i];
#pragma unroll
                for (int w = 1; w < kGemvWarps; ++w) sum += rb[w][i];
                prm.D[(size_t)m * prm.N + n0 + r] = __float2bfloat16_rn(sum * prm.alpha);
            }
        }
    }
}

// One or two token rows of MXFP4 (the counterpart of nvfp4_gemv_areg_kernel):
// each thread's token chunks are decoded once and held in registers with
// their E8M0 exponents, all CPT weight chunks of a row group are loaded at
// once and the next group's before this group's reduction.  A chunk's exact
// sum is scaled by 2^(ea + eb - 254) with one multiply while that power is a
// normal fp32 number -- the same value ldexpf gives, exact unless the result
// is subnormal, where both round to nearest even -- and by ldexpf otherwise;
// the sums and their order are nvfp4_gemv_mx_kernel's, so the results are
// identical.
template <int MT, int RW, int CPT>
__global__ void __launch_bounds__(kGemvThreads) nvfp4_gemv_mx_areg_kernel(const GemvMxParams prm) {
    static_assert(MT * CPT <= 4, "token chunks held in registers");
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;
    const size_t row_bytes = (size_t)prm.K >> 1;
    const size_t srow_bytes = (size_t)prm.K >> 5;
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;
    int nch = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) nch += (t + j * kGemvThreads < kc) ? 1 : 0;

    uint4 bq[CPT][RW];
    uint32_t bs[CPT][RW];
    auto load_group = [&](int n0) {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int n = min(n0 + r, prm.N - 1);
            const uint8_t* br = prm.B + (size_t)n * row_bytes + 16 * (size_t)t;
            const uint8_t* bsr = prm.sB + (size_t)n * srow_bytes + (size_t)t;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                if (j < nch) {
                    bq[j][r] = ld_stream_v4(br + 16 * (size_t)(j * kGemvThreads));
                    bs[j][r] = ld_stream_u8(bsr + (size_t)(j * kGemvThreads));
                } else {
                    bq[j][r] = make_uint4(0u, 0u, 0u, 0u);
                    bs[j][r] = 127u;
                }
            }
        }
    };

    grid_launch_dependents();
    int n0 = blockIdx.x * RW;
    if (prm.prefetch_b) load_group(n0);   // only B is touched before the wait
    grid_dependency_wait();

    uint32_t ah[MT][CPT][16];
    int ea[MT][CPT];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + j * kGemvThreads;
            if (m < M && j < nch) {
                decode_chunk(ld_cached_v4(prm.A + (size_t)m * row_bytes + 16 * (size_t)c), ah[m][j]);
                ea[m][j] = (int)__ldg(prm.sA + (size_t)m * srow_bytes + (size_t)c);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) ah[m][j][i] = 0u;
                ea[m][j] = 127;
            }
        }
    if (!prm.prefetch_b) load_group(n0);

    for (int it = 0; n0 < prm.N; n0 += group_stride, ++it) {
        float acc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            if (j >= nch) break;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                uint32_t bh[16];
                decode_chunk(bq[j][r], bh);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const float blk = block_dot(ah[m][j], bh) + block_dot(ah[m][j] + 8, bh + 8);   // exact
                        const int e = ea[m][j] + (int)bs[j][r] - 254;
                        const float scaled = (e >= -126 && e <= 127)
                                                 ? blk * __uint_as_float((uint32_t)(e + 127) << 23)
                                                 : ldexpf(blk, e);
                        acc[r][m] += scaled;
                    }
                }
            }
        }
        const int n_next = n0 + group_stride;
        if (n_next < prm.N) load_group(n_next);

        float v[NV];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[r * MT + m] = acc[r][m];
        warp_reduce_scatter<NV>(v, lane);
        float (*rb)[NV] = red[it & 1];
        if (gemv_writer_lane<NV>(lane)) {
#pragma unroll
            for (int q = 0; q < (NV >= 32 ? NV / 32 : 1); ++q) rb[warp][gemv_reduced_index<NV>(lane, q)] = v[q];
        }
        __syncthreads();
        for (int e = t; e < NV; e += kGemvThreads) {
            const int r = e / MT, m = e % MT;
            if (m < M && n0 + r < prm.N) {
                float sum = rb[0][e];
#pragma unroll
                for (int w = 1; w < kGemvWarps; ++w) sum += rb[w][e];
                prm.D[(size_t)m * prm.N + n0 + r] = __float2bfloat16_rn(sum * prm.alpha);
            }
        }
    }
}

}  // namespace nvfp4
