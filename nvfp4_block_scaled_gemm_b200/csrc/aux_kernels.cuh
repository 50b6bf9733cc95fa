// Quantize-and-pack, scale re-layout and the wait-timeout diagnostic kernel.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace nvfp4 {

// ------------------------------------------------------------ scale re-layout
// Row-major E4M3 scales [rows][K/16] -> 512-byte atoms (128 rows x 4 blocks):
// row r, block j of an atom at byte 16*(r%32) + 4*(r/32) + j; atoms ordered
// along K (one per 64-element MMA step) within each 128-row block; padding
// rows are zero.  One thread writes one 16-byte line of an atom: the word of
// K step `ks` from rows L, L+32, L+64, L+96 of row block `rb`.
__global__ void swizzle_scales_kernel(const uint8_t* __restrict__ s, int rows, int kb_row, int steps,
                                      long long lines, uint8_t* __restrict__ out) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= lines) return;
    const int L = (int)(idx & 31);
    const long long t = idx >> 5;
    const int ks = (int)(t % steps);
    const long long rb = t / steps;
    uint32_t w[4];
#pragma unroll
    for (int r1 = 0; r1 < 4; ++r1) {
        const long long r = rb * 128 + L + 32 * r1;
        w[r1] = r < rows ? __ldg(reinterpret_cast<const uint32_t*>(s + r * kb_row + 4 * ks)) : 0u;
    }
    *reinterpret_cast<uint4*>(out + (rb * steps + ks) * 512 + 16 * L) = make_uint4(w[0], w[1], w[2], w[3]);
}

// MXFP4 scales (E8M0, one per 32 values), row-major [rows][K/32], into the
// 512-byte atoms the kind::mxf4 MMA reads through TMEM: atom w of a 128-row
// block holds K steps 2w and 2w+1 (64 values each); line L is the four bytes
// of rows L, L+32, L+64, L+96, each byte quadruple being that row's scales of
// blocks 4w .. 4w+3 (the even step's two blocks in bytes 0-1, the odd step's
// in bytes 2-3).  Bytes past K or past the rows are zero.  One thread per
// line; byte loads, so any row stride works.
__global__ void swizzle_scales_mx_kernel(const uint8_t* __restrict__ s, int rows, int kb_row, int pairs,
                                         long long lines, uint8_t* __restrict__ out) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= lines) return;
    const int L = (int)(idx & 31);
    const long long t = idx >> 5;
    const int w = (int)(t % pairs);
    const long long rb = t / pairs;
    uint32_t v[4];
#pragma unroll
    for (int r1 = 0; r1 < 4; ++r1) {
        const long long r = rb * 128 + L + 32 * r1;
        uint32_t word = 0u;
        if (r < rows) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int kb = 4 * w + b;
                if (kb < kb_row) word |= (uint32_t)__ldg(s + r * kb_row + kb) << (8 * b);
            }
        }
        v[r1] = word;
    }
    *reinterpret_cast<uint4*>(out + (rb * pairs + w) * 512 + 16 * L) = make_uint4(v[0], v[1], v[2], v[3]);
}

// The same layout for two scale tensors in one launch, K a multiple of 256:
// one 128-thread CTA per (tensor, 128-row block, 256-element K tile).  Thread
// t reads the 16 scale bytes of row t of the block (one request per row), the
// CTA transposes them through shared memory and writes the four 512-byte
// atoms of the K tile as contiguous, fully coalesced lines.
struct ScaleTileJob {
    const uint8_t* s;   // row-major [rows][K/16]
    uint8_t* out;       // atoms [ceil(rows/128)][K/64][512 B]
    int rows;
    int row_blocks;     // ceil(rows / 128)
    int vec16;          // s and its rows are 16-byte aligned
};

__global__ void __launch_bounds__(128) swizzle_scale_tiles_kernel(ScaleTileJob a, ScaleTileJob b, int kb_row,
                                                                  int k_tiles) {
    __shared__ uint32_t tile[128][5];   // odd row pitch: conflict-free column reads
    int blk = (int)blockIdx.x;
    const int blocks_a = a.row_blocks * k_tiles;
    const ScaleTileJob& job = blk < blocks_a ? a : b;
    if (blk >= blocks_a) blk -= blocks_a;
    const int rb = blk / k_tiles, kt = blk - rb * k_tiles;
    const int t = (int)threadIdx.x;
    const long long r = (long long)rb * 128 + t;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (r < job.rows) {
        const uint8_t* src = job.s + r * kb_row + 16 * kt;
        if (job.vec16) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
            w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = __ldg(reinterpret_cast<const uint32_t*>(src) + j);
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[t][j] = w[j];
    __syncthreads();
    const int j = t >> 5, L = t & 31;   // warp j writes the atom of K step 4*kt + j
    const size_t steps = (size_t)k_tiles * 4;
    uint8_t* atom = job.out + ((size_t)rb * steps + 4 * (size_t)kt + j) * 512;
    *reinterpret_cast<uint4*>(atom + 16 * L) = make_uint4(tile[L][j], tile[L + 32][j], tile[L + 64][j], tile[L + 96][j]);
}

// ------------------------------------------------------------ quantization
// Pass 1: amax over the tensor, as the bit pattern of a non-negative float
// (monotone as an unsigned integer) accumulated with atomicMax.
__global__ void amax_kernel(const float4* __restrict__ x, long long n4, unsigned* __restrict__ amax_bits) {
    float m = 0.0f;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        const float4 v = __ldg(x + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float warp_max[32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(m));
    }
}

// Pass 2: one thread per 16-element block.
__global__ void quantize_kernel(const float* __restrict__ X, long long blocks, const unsigned* __restrict__ amax_bits,
                                uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= blocks) return;
    const float g = global_scale_from_amax(__uint_as_float(*amax_bits));
    const float six_g = __fmul_rn(6.0f, g);
    float x[16];
    const float4* src = reinterpret_cast<const float4*>(X + b * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(src + i);
        x[4 * i] = f.x;
        x[4 * i + 1] = f.y;
        x[4 * i + 2] = f.z;
        x[4 * i + 3] = f.w;
    }
    uint32_t s, out[2];
    quantize_block16(x, g, six_g, s, out);
    *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(out[0], out[1]);
    scales[b] = (uint8_t)s;
}

// One pass with the global scale g given (a scale fixed in advance for the
// activation tensor): the same block steps as quantize_kernel, on fp32 or
// BF16 input (BF16 widens to fp32 exactly).  Launched with programmatic
// dependent launch: it lets the next kernel (the GEMM) start its prologue at
// once and waits for the previous kernel before reading X.
template <bool BF16>
__global__ void quantize_scaled_kernel(const void* __restrict__ X, long long blocks, float g,
                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    grid_launch_dependents();
    grid_dependency_wait();
    const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= blocks) return;
    const float six_g = __fmul_rn(6.0f, g);
    float x[16];
    if (BF16) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + b * 16);   // BF16 bits
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint4 v = __ldg(src + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(X) + b * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = __ldg(src + i);
            x[4 * i] = f.x;
            x[4 * i + 1] = f.y;
            x[4 * i + 2] = f.z;
            x[4 * i + 3] = f.w;
        }
    }
    uint32_t s, out[2];
    quantize_block16(x, g, six_g, s, out);
    *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(out[0], out[1]);
    scales[b] = (uint8_t)s;
}

// Pass 3: replace the amax bits by the global scale g.
__global__ void finalize_global_scale_kernel(float* g_inout) {
    g_inout[0] = global_scale_from_amax(__uint_as_float(*reinterpret_cast<unsigned*>(g_inout)));
}

// ------------------------------------------------------------ diagnostics
// Waits on a barrier nothing arrives on, bounded by limit_ns; records the
// timeout in the error word and returns.
__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(smem_addr(&bar), 0, &abort_flag, limit_ns);
    __syncthreads();
}

}  // namespace nvfp4
