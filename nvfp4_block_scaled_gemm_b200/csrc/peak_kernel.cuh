// Calibration of the dense FP4 tensor-core rate: back-to-back block-scaled
// MMAs (kind::mxf4nvf4, block16) on operands that stay in shared memory and
// scales that stay in TMEM, one CTA per SM (or one CTA pair per two SMs with
// the 2-CTA form), nothing else running.  The time of a launch gives the
// throughput that the GEMM kernels' roofline fractions are quoted against
// beside the nominal figure.  The operand values are a fixed non-zero pattern;
// the accumulator is never read.
#pragma once

#include "pair_kernel.cuh"

namespace nvfp4 {

constexpr int kPeakThreads = 128;
constexpr int kPeakA = 128 * kStageKBytes;   // 16 KB: 128 rows x one 256-K tile
constexpr int kPeakB = 256 * kStageKBytes;   // 32 KB: 256 rows
// More shared memory than two CTAs can share on one SM: one CTA per SM, so
// every SM's tensor cores are busy and no CTA waits for another's TMEM.
constexpr int kPeakSmem = 160 * 1024;
static_assert(1024 + kPeakA + kPeakB + 1024 <= kPeakSmem, "peak kernel shared memory");

// PAIR = false: tcgen05.mma.cta_group::1, M = 128, N = 256, K = 64 per
// instruction.  PAIR = true: cta_group::2 on a 2-CTA cluster, M = 256 (128 rows
// of A per CTA), N = 256 (128 rows of B per CTA).  `steps` instructions per
// CTA (per pair), all accumulating into one TMEM accumulator.
template <bool PAIR>
__global__ void __launch_bounds__(kPeakThreads, 1) fp4_peak_kernel(long long steps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kPeakA + kPeakB);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_cta_rank() : 0u;

    // operands: E2M1 codes 1 (0.5) and 2 (1.0) alternating; scales 0x38 (1.0)
    for (int i = threadIdx.x; i < (kPeakA + kPeakB) / 4; i += kPeakThreads)
        reinterpret_cast<uint32_t*>(smem)[i] = 0x21212121u;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(bar), 1);
        fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor-core reads
    if (PAIR) cluster_sync();
    else __syncthreads();
    if (warp == 0) {
        if (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // scales: columns 256.. (4 for A, 8 for B per K step; one set reused)
    {
        const uint32_t t_quad = tmem + ((uint32_t)(warp * 32) << 16);
        uint32_t w[32], w16[16];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = 0x38383838u;
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = 0x38383838u;
        tmem_store_32(t_quad + 256, w);
        tmem_store_16(t_quad + 288, w16);
        tmem_wait_store();
    }
    tc_fence_before();
    if (PAIR) cluster_sync();
    else __syncthreads();
    tc_fence_after();

    if (warp == 0 && lane == 0 && rank == 0) {
        const uint32_t sa = smem_addr(smem), sb = sa + kPeakA;
        const uint64_t da = desc_kmajor_sw128(sa), db = desc_kmajor_sw128(sb);
        if (PAIR) {
            constexpr uint32_t idesc = idesc_nvf4(256, 256);
            for (long long i = 0; i < steps; ++i) {
                const int j = (int)(i & 3);
                tc_mma_nvf4_pair(tmem, da + 2u * j, db + 2u * j, idesc, tmem + 256 + 4 * j, tmem + 272 + 8 * j,
                                 i > 0 ? 1u : 0u);
            }
            tc_commit_pair(smem_addr(bar));
        } else {
            constexpr uint32_t idesc = idesc_nvf4(128, 256);
            for (long long i = 0; i < steps; ++i) {
                const int j = (int)(i & 3);
                tc_mma_nvf4(tmem, da + 2u * j, db + 2u * j, idesc, tmem + 256 + 4 * j, tmem + 272 + 8 * j,
                            i > 0 ? 1u : 0u);
            }
            tc_commit(smem_addr(bar));
        }
    }
    // every CTA waits for the MMAs that used its TMEM and shared memory
    if (warp == 0 && lane == 0) mbar_wait(smem_addr(bar), 0u, nullptr, 4000000000ull);
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

}  // namespace nvfp4
