// 2:4-sparse NVFP4 weights: the decode kernel that reads them directly, and
// the re-expansion to dense codes that larger token counts use.
//
// Layout (FP4 structured sparsity is named, without a layout, in "Peeling the
// Kernel Onion", sections "Assumptions Embedded in the Benchmark" and
// "Knowledge Created and Its Impact"; this library's reading): of every 4
// consecutive packed bytes of a weight row -- pairs of E2M1 values -- at most
// 2 are non-zero.  Per row of K values:
//   values [K/4]:  the 2 kept bytes of each group of 4, lower position first;
//   meta   [K/16]: one nibble p0 | p1 << 2 per group (p0 < p1), the even
//                  group in the low nibble;
//   scales [K/16]: the dense E4M3 block scales.
// Weight bytes per row drop from 9K/16 to 6K/16.
//
// The decode kernel follows nvfp4_gemv_kernel (gemv_kernel.cuh): a thread
// owns 32-value chunks of K, which here are 8 value bytes, 2 metadata bytes
// and 2 scale bytes per weight row.  One byte permute per two groups gathers
// the activation bytes at the kept positions next to the kept weight bytes
// (its selector built once per weight row and chunk from the metadata), so
// only kept pairs are decoded and multiplied: a 16-value block is 4
// fma.rn.f16x2 (4 products per half, at most 144 in magnitude: exact), and
// the rest -- exact block sum times sA * sB, fp32 sum over blocks, warp
// butterfly, fixed-order CTA sum -- is the dense kernel's.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gemv_kernel.cuh"

namespace nvfp4 {

struct GemvSp24Params {
    const uint8_t* A;    // [M][K/2] dense E2M1 codes
    const uint8_t* sA;   // [M][K/16]
    const uint8_t* Bv;   // [N][K/4] kept bytes
    const uint8_t* Bm;   // [N][K/16] position nibbles
    const uint8_t* sB;   // [N][K/16]
    __nv_bfloat16* D;    // [M][N]
    float alpha;
    int M, N, K;
    int prefetch_b;
};

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Byte-permute selector that gathers, from two 4-byte activation groups
// (first group bytes 0..3, second 4..7), the bytes at the kept positions of
// one metadata byte (low nibble: first group's p0 | p1 << 2, high nibble: the
// second group's): each 2-bit position becomes a selector nibble, the second
// group's offset by 4.
__device__ __forceinline__ uint32_t gather_selector(uint32_t m) {
    return (m & 0x3u) | ((m & 0xCu) << 2) | ((m & 0x30u) << 4) | ((m & 0xC0u) << 6) | 0x4400u;
}

template <int MT, int RW>
__global__ void __launch_bounds__(kGemvThreads) nvfp4_gemv_sp24_kernel(const GemvSp24Params prm) {
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;                        // 32-value chunks per row
    const size_t arow_bytes = (size_t)prm.K >> 1;     // dense code bytes per activation row
    const size_t vrow_bytes = (size_t)prm.K >> 2;     // kept bytes per weight row
    const size_t srow_bytes = (size_t)prm.K >> 4;     // scale (and metadata) bytes per row
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;

    const uint8_t* vrow[RW];
    const uint8_t* mrow[RW];
    const uint8_t* srow[RW];
    auto set_rows = [&](int n0) {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int n = min(n0 + r, prm.N - 1);
            vrow[r] = prm.Bv + (size_t)n * vrow_bytes;
            mrow[r] = prm.Bm + (size_t)n * srow_bytes;
            srow[r] = prm.sB + (size_t)n * srow_bytes;
        }
    };

    uint2 bq[kGemvGroup][RW], nq[kGemvGroup][RW];
    uint32_t bm[kGemvGroup][RW], nm[kGemvGroup][RW];
    uint32_t bs[kGemvGroup][RW], ns[kGemvGroup][RW];
    auto load_group = [&](uint2 (&q)[kGemvGroup][RW], uint32_t (&mt)[kGemvGroup][RW], uint32_t (&sc)[kGemvGroup][RW],
                          int c0) {
#pragma unroll
        for (int g = 0; g < kGemvGroup; ++g) {
            const int c = c0 + g * kGemvThreads;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                if (c < kc) {
                    q[g][r] = ld_stream_v2(vrow[r] + 8 * (size_t)c);
                    mt[g][r] = ld_stream_u16(mrow[r] + 2 * (size_t)c);
                    sc[g][r] = ld_stream_u16(srow[r] + 2 * (size_t)c);
                } else {
                    q[g][r] = make_uint2(0u, 0u);
                    mt[g][r] = 0x4444u;   // positions 0, 1 in every group; the values are zero
                    sc[g][r] = 0u;
                }
            }
        }
    };

    grid_launch_dependents();
    const int step = kGemvGroup * kGemvThreads;
    int n0 = blockIdx.x * RW;
    set_rows(n0);
    if (prm.prefetch_b) load_group(bq, bm, bs, t);   // only B is touched before the wait
    grid_dependency_wait();
    if (!prm.prefetch_b) load_group(bq, bm, bs, t);

    for (int it = 0; n0 < prm.N; n0 += group_stride, ++it) {
        float acc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

        for (int c0 = t; c0 < kc; c0 += step) {
            const bool more = c0 + step < kc;
            if (more) load_group(nq, nm, ns, c0 + step);
#pragma unroll
            for (int g = 0; g < kGemvGroup; ++g) {
                const int c = c0 + g * kGemvThreads;
                if (c >= kc) break;
                // kept weight pairs, decoded: bh[r][2j], bh[r][2j+1] for group j
                uint32_t bh[RW][8];
                float sb0[RW], sb1[RW];
                uint32_t sel01[RW], sel23[RW];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    sel01[r] = gather_selector(bm[g][r] & 0xFFu);
                    sel23[r] = gather_selector((bm[g][r] >> 8) & 0xFFu);
                    uint32_t h4[4];
                    e2m1x8_to_f16x2(bq[g][r].x, h4);
                    bh[r][0] = h4[0], bh[r][1] = h4[1], bh[r][2] = h4[2], bh[r][3] = h4[3];
                    e2m1x8_to_f16x2(bq[g][r].y, h4);
                    bh[r][4] = h4[0], bh[r][5] = h4[1], bh[r][6] = h4[2], bh[r][7] = h4[3];
                    sb0[r] = e4m3_value(bs[g][r] & 0xFFu);
                    sb1[r] = e4m3_value(bs[g][r] >> 8);
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const uint4 aq = ld_cached_v4(prm.A + (size_t)m * arow_bytes + 16 * (size_t)c);
                        const uint32_t as = ld_cached_u16(prm.sA + (size_t)m * srow_bytes + 2 * (size_t)c);
                        const float sa0 = e4m3_value(as & 0xFFu), sa1 = e4m3_value(as >> 8);
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            // the activation bytes at the kept positions, in the
                            // order of the kept weight bytes: groups 0, 1 from
                            // words x, y; groups 2, 3 from z, w
                            uint32_t ah[8], t4[4];
                            e2m1x8_to_f16x2(__byte_perm(aq.x, aq.y, sel01[r]), t4);
                            ah[0] = t4[0], ah[1] = t4[1], ah[2] = t4[2], ah[3] = t4[3];
                            e2m1x8_to_f16x2(__byte_perm(aq.z, aq.w, sel23[r]), t4);
                            ah[4] = t4[0], ah[5] = t4[1], ah[6] = t4[2], ah[7] = t4[3];
                            float bsum[2];
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t* a = ah + 4 * h;
                                const uint32_t* w = bh[r] + 4 * h;
                                __half2 s2 = __hmul2(*reinterpret_cast<const __half2*>(&a[0]),
                                                     *reinterpret_cast<const __half2*>(&w[0]));
#pragma unroll
                                for (int i = 1; i < 4; ++i)
                                    s2 = __hfma2(*reinterpret_cast<const __half2*>(&a[i]),
                                                 *reinterpret_cast<const __half2*>(&w[i]), s2);
                                bsum[h] = half2_sum_f32(s2);
                            }
                            acc[r][m] = fmaf(bsum[0], sa0 * sb0[r], acc[r][m]);
                            acc[r][m] = fmaf(bsum[1], sa1 * sb1[r], acc[r][m]);
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
                        bm[g][r] = nm[g][r];
                        bs[g][r] = ns[g][r];
                    }
            }
        }

        const int n_next = n0 + group_stride;
        if (n_next < prm.N) {
            set_rows(n_next);
            load_group(bq, bm, bs, t);
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

// The same selector in fewer operations: v = m | m << 4 puts fields 0 and 2
// at bits 0-1 and 8-9 and, shifted by 2, fields 1 and 3 at bits 4-5 and
// 12-13 (equal to gather_selector for all 256 bytes).
__device__ __forceinline__ uint32_t gather_selector_fast(uint32_t m) {
    const uint32_t v = m | (m << 4);
    return (v & 0x0303u) | ((v << 2) & 0x3030u) | 0x4400u;
}

// One or two token rows (the counterpart of nvfp4_gemv_areg_kernel): each
// thread's token chunks (packed codes) and their scales (as fp32) are loaded
// once and kept in registers, a weight chunk's two scales are converted in one
// instruction, and all CPT chunks of a row group are loaded at once, the next
// group's before this group's reduction.  The kept-pair arithmetic and the
// summation order are nvfp4_gemv_sp24_kernel's, so the results are identical.
template <int MT, int RW, int CPT>
__global__ void __launch_bounds__(kGemvThreads) nvfp4_gemv_sp24_areg_kernel(const GemvSp24Params prm) {
    static_assert(MT * CPT <= 4, "token chunks held in registers");
    constexpr int NV = RW * MT;
    __shared__ float red[2][kGemvWarps][NV];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kc = prm.K >> 5;
    const size_t arow_bytes = (size_t)prm.K >> 1;
    const size_t vrow_bytes = (size_t)prm.K >> 2;
    const size_t srow_bytes = (size_t)prm.K >> 4;
    const int M = prm.M;
    const int group_stride = gridDim.x * RW;
    int nch = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) nch += (t + j * kGemvThreads < kc) ? 1 : 0;

    uint2 bq[CPT][RW];
    uint32_t bm[CPT][RW], bs[CPT][RW];
    auto load_group = [&](int n0) {
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int n = min(n0 + r, prm.N - 1);
            const uint8_t* vr = prm.Bv + (size_t)n * vrow_bytes + 8 * (size_t)t;
            const uint8_t* mr = prm.Bm + (size_t)n * srow_bytes + 2 * (size_t)t;
            const uint8_t* sr = prm.sB + (size_t)n * srow_bytes + 2 * (size_t)t;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                if (j < nch) {
                    bq[j][r] = ld_stream_v2(vr + 8 * (size_t)(j * kGemvThreads));
                    bm[j][r] = ld_stream_u16(mr + 2 * (size_t)(j * kGemvThreads));
                    bs[j][r] = ld_stream_u16(sr + 2 * (size_t)(j * kGemvThreads));
                } else {
                    bq[j][r] = make_uint2(0u, 0u);
                    bm[j][r] = 0x4444u;
                    bs[j][r] = 0u;
                }
            }
        }
    };

    grid_launch_dependents();
    int n0 = blockIdx.x * RW;
    if (prm.prefetch_b) load_group(n0);   // only B is touched before the wait
    grid_dependency_wait();

    uint4 aq[MT][CPT];
    float sa[MT][CPT][2];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + j * kGemvThreads;
            if (m < M && j < nch) {
                aq[m][j] = ld_cached_v4(prm.A + (size_t)m * arow_bytes + 16 * (size_t)c);
                const float2 v = e4m3x2_values(ld_cached_u16(prm.sA + (size_t)m * srow_bytes + 2 * (size_t)c));
                sa[m][j][0] = v.x;
                sa[m][j][1] = v.y;
            } else {
                aq[m][j] = make_uint4(0u, 0u, 0u, 0u);
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
                const uint32_t sel01 = gather_selector_fast(bm[j][r] & 0xFFu);
                const uint32_t sel23 = gather_selector_fast((bm[j][r] >> 8) & 0xFFu);
                uint32_t bh[8], h4[4];
                e2m1x8_to_f16x2(bq[j][r].x, h4);
                bh[0] = h4[0], bh[1] = h4[1], bh[2] = h4[2], bh[3] = h4[3];
                e2m1x8_to_f16x2(bq[j][r].y, h4);
                bh[4] = h4[0], bh[5] = h4[1], bh[6] = h4[2], bh[7] = h4[3];
                const float2 sb = e4m3x2_values(bs[j][r]);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        uint32_t ah[8], t4[4];
                        e2m1x8_to_f16x2(__byte_perm(aq[m][j].x, aq[m][j].y, sel01), t4);
                        ah[0] = t4[0], ah[1] = t4[1], ah[2] = t4[2], ah[3] = t4[3];
                        e2m1x8_to_f16x2(__byte_perm(aq[m][j].z, aq[m][j].w, sel23), t4);
                        ah[4] = t4[0], ah[5] = t4[1], ah[6] = t4[2], ah[7] = t4[3];
                        float bsum[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t* a = ah + 4 * h;
                            const uint32_t* w = bh + 4 * h;
                            __half2 s2 = __hmul2(*reinterpret_cast<const __half2*>(&a[0]),
                                                 *reinterpret_cast<const __half2*>(&w[0]));
#pragma unroll
                            for (int i = 1; i < 4; ++i)
                                s2 = __hfma2(*reinterpret_cast<const __half2*>(&a[i]),
                                             *reinterpret_cast<const __half2*>(&w[i]), s2);
                            bsum[h] = half2_sum_f32(s2);
                        }
                        acc[r][m] = fmaf(bsum[0], sa[m][j][0] * sb.x, acc[r][m]);
                        acc[r][m] = fmaf(bsum[1], sa[m][j][1] * sb.y, acc[r][m]);
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

// Kept bytes and position nibbles -> dense packed codes, one metadata byte
// (two groups, 8 dense bytes) per item.
__global__ void sparse24_expand_kernel(const uint8_t* __restrict__ values, const uint8_t* __restrict__ meta,
                                       long long items, uint8_t* __restrict__ dense) {
    grid_dependency_wait();
    grid_launch_dependents();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < items;
         i += (long long)gridDim.x * blockDim.x) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(values + 4 * i);
        const uint32_t mb = meta[i];
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t nib = (mb >> (4 * h)) & 0xFu;
            const uint32_t p0 = nib & 3u, p1 = nib >> 2;
            const uint32_t v0 = (v >> (16 * h)) & 0xFFu, v1 = (v >> (16 * h + 8)) & 0xFFu;
            w[h] = (v0 << (8 * p0)) | (p1 != p0 ? (v1 << (8 * p1)) : 0u);
        }
        *reinterpret_cast<uint2*>(dense + 8 * i) = make_uint2(w[0], w[1]);
    }
}

}  // namespace nvfp4
