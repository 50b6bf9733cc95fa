// C ABI of libnvfp4gemm.so (declared in include/nvfp4_gemm.h): host-side
// validation, scratch management, TMA descriptor creation and dispatch to the
// sm_100a kernels.  All arithmetic of the GEMM happens in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "../../include/nvfp4_gemm.h"
#include "aux_kernels.cuh"
#include "gemm_kernel.cuh"
#include "gemv_kernel.cuh"
#include "sparse_kernel.cuh"
#include "grouped_kernel.cuh"
#include "pair_kernel.cuh"
#include "peak_kernel.cuh"
#include "persistent_kernel.cuh"
#include "splitk_kernel.cuh"

namespace {

using nvfp4::GemmParams;
using nvfp4::TileConfig;

constexpr int kVersion = 100;  // 0.1.0

// Kernels enqueued (or captured into a graph) by this library, all devices.
std::atomic<unsigned long long> g_launches{0};

// ------------------------------------------------------------ device checks
struct DeviceInfo {
    bool checked = false;
    bool supported = false;
    int num_sms = 0;
    uint64_t smem_attr_set = 0;  // bit per kernel instantiation
    uint64_t smem_attr_set_mx = 0;  // the same for the MXFP4 instantiations
    int pair_clusters = -1;      // co-resident 2-CTA clusters of the pair kernel (-1: not queried)
    std::map<uint32_t, int> split_clusters;   // co-resident split-K clusters per (kernel, cluster size)
};
std::mutex g_mu;
std::map<int, DeviceInfo> g_devices;

nvfp4_status current_device(int* dev, DeviceInfo** info) {
    if (cudaGetDevice(dev) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_devices[*dev];
    if (!d.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        d.checked = true;
        d.supported = (major == 10 && minor == 0);
        d.num_sms = sms;
    }
    *info = &d;
    return d.supported ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED_DEVICE;
}

// ------------------------------------------------------------ scratch
// Per (device, stream) scratch: the re-laid-out scales when they cannot be
// loaded row-major by TMA.

struct Scratch {
    uint8_t* ptr = nullptr;
    size_t cap = 0;
};
// Kinds of per-(device, stream) scratch, each its own buffer because one call
// may need several at once.
enum ScratchKind { kScratchScales = 0, kScratchAct = 1, kScratchSplitK = 2 };
std::map<std::pair<int, uintptr_t>, Scratch> g_scratch[3];

nvfp4_status get_scratch(int dev, cudaStream_t stream, size_t bytes, uint8_t** out, int kind = kScratchScales) {
    std::lock_guard<std::mutex> lk(g_mu);
    Scratch& s = g_scratch[kind][{dev, reinterpret_cast<uintptr_t>(stream)}];
    if (s.cap < bytes) {
        size_t want = std::max(bytes, s.cap * 2);
        want = (want + 0xFFFFF) & ~size_t(0xFFFFF);
        if (s.ptr != nullptr) {
            // Only this stream uses this buffer: once its queue drains, it is free.
            if (cudaStreamSynchronize(stream) != cudaSuccess) return NVFP4_ERR_CUDA;
            cudaFree(s.ptr);
            s.ptr = nullptr;
            s.cap = 0;
        }
        void* p = nullptr;
        if (cudaMalloc(&p, want) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_NO_MEMORY;
        }
        s.ptr = static_cast<uint8_t*>(p);
        s.cap = want;
    }
    *out = s.ptr;
    return NVFP4_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per (device, stream) pair of unit counters for the grouped kernel's
// run-time hand-out of work units: zeroed once here, and by the last CTA of
// every launch after that.  Launches on one stream run in order, so they
// share it; other streams get their own.
std::map<std::pair<int, uintptr_t>, unsigned*> g_unit_counters;

nvfp4_status get_unit_counter(int dev, cudaStream_t stream, unsigned** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    unsigned*& c = g_unit_counters[{dev, reinterpret_cast<uintptr_t>(stream)}];
    if (c == nullptr) {
        void* p = nullptr;
        if (cudaMalloc(&p, 2 * sizeof(unsigned)) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_NO_MEMORY;
        }
        if (cudaMemsetAsync(p, 0, 2 * sizeof(unsigned), stream) != cudaSuccess) {
            cudaGetLastError();
            cudaFree(p);
            return NVFP4_ERR_CUDA;
        }
        c = static_cast<unsigned*>(p);
    }
    *out = c;
    return NVFP4_OK;
}

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// 2-D map over a row-major byte matrix [rows][row_bytes]; box 128 bytes x
// box_rows, 128-byte swizzle, zero fill out of bounds.
bool make_operand_map(CUtensorMap* map, const void* base, long long rows, long long row_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    const cuuint32_t elem_strides[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over row-major scales [rows][row_bytes] (row_bytes a multiple of
// 16); box 16 bytes (= 256 elements of K) x box_rows, no swizzle.
bool make_scale_map(CUtensorMap* map, const void* base, long long rows, long long row_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {16u, (cuuint32_t)box_rows};
    const cuuint32_t elem_strides[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over row-major BF16 [rows][cols]; box 256 values (one 256-element
// K tile, 512 bytes) x box_rows, no swizzle (the writer warps read it).
bool make_bf16_map(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {256u, (cuuint32_t)box_rows};
    const cuuint32_t elem_strides[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

nvfp4_status launch_swizzle(const void* s, int rows, int K, void* out, cudaStream_t stream) {
    const int steps = K / 64;
    const long long lines = (long long)((rows + 127) / 128) * steps * 32;
    if (lines == 0) return NVFP4_OK;
    const int threads = 256;
    const long long blocks = (lines + threads - 1) / threads;
    nvfp4::swizzle_scales_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const uint8_t*>(s), rows, K / 16, steps, lines, static_cast<uint8_t*>(out));
    g_launches++;
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// ------------------------------------------------------------ GEMM dispatch
struct Plan {
    bool swap;
    int bq;
    int tiles_p, tiles_q;
    int splits, k_tiles;   // splits = thread-block cluster size along K
};

// Tuning override: NVFP4_GEMM_PLAN="swap:bq:splits" (e.g. "1:16:8") forces the
// tile shape of every nvfp4_gemm call whose shape allows it.  Read on each
// call (a getenv), so a tuning run can change it between calls.
struct PlanOverride {
    bool set = false;
    int swap = 0, bq = 0, splits = 0;
};

PlanOverride plan_override() {
    PlanOverride o;
    const char* e = std::getenv("NVFP4_GEMM_PLAN");
    int a, b, c;
    if (e && std::sscanf(e, "%d:%d:%d", &a, &b, &c) == 3 && (b == 16 || b == 32 || b == 64 || b == 128 || b == 256) &&
        (c == 1 || c == 2 || c == 4 || c == 8 || c == 16)) {
        o.set = true;
        o.swap = a != 0;
        o.bq = b;
        o.splits = c;
    }
    return o;
}

// How many clusters of `splits` CTAs of a split-K instantiation fit on the
// GPU at once (cudaOccupancyMaxActiveClusters, queried once and cached).  A
// grid with more clusters than this runs in two waves, which for these
// latency-bound shapes costs more than halving the split.
template <int BQ, bool SWAP, bool SFR>
int split_cluster_capacity(DeviceInfo* info, int splits) {
    using C = TileConfig<BQ, true>;
    auto kern = nvfp4::nvfp4_gemm_kernel<BQ, SWAP, true, SFR>;
    const uint32_t key = (uint32_t)BQ | (SWAP ? 1u << 10 : 0u) | (SFR ? 1u << 11 : 0u) | ((uint32_t)splits << 12);
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = info->split_clusters.find(key);
    if (it != info->split_clusters.end()) return it->second;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) == cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3((unsigned)splits, 1, 1);
        q.blockDim = dim3(nvfp4::gemm_threads<BQ, SWAP, SFR, false>(), 1, 1);
        q.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute ca[1];
        ca[0].id = cudaLaunchAttributeClusterDimension;
        ca[0].val.clusterDim.x = (unsigned)splits;
        ca[0].val.clusterDim.y = 1;
        ca[0].val.clusterDim.z = 1;
        q.attrs = ca;
        q.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    info->split_clusters[key] = n;
    return n;
}

template <bool SWAP, bool SFR>
int split_cluster_capacity_bq(DeviceInfo* info, int bq, int splits) {
    switch (bq) {
        case 16: return split_cluster_capacity<16, SWAP, SFR>(info, splits);
        case 32: return split_cluster_capacity<32, SWAP, SFR>(info, splits);
        case 64: return split_cluster_capacity<64, SWAP, SFR>(info, splits);
        case 128: return split_cluster_capacity<128, SWAP, SFR>(info, splits);
        case 256: return split_cluster_capacity<256, SWAP, SFR>(info, splits);
        default: return 0;
    }
}

int split_cluster_capacity_of(DeviceInfo* info, bool swap, int bq, bool sfr, int splits) {
    if (swap) return sfr ? split_cluster_capacity_bq<true, true>(info, bq, splits)
                         : split_cluster_capacity_bq<true, false>(info, bq, splits);
    return sfr ? split_cluster_capacity_bq<false, true>(info, bq, splits)
               : split_cluster_capacity_bq<false, false>(info, bq, splits);
}

Plan make_plan(int M, int N, int K, DeviceInfo* info, bool sfr, int max_splits = 8) {
    const int num_sms = info->num_sms;
    Plan p{};
    p.k_tiles = (K + 255) / 256;
    const PlanOverride o = plan_override();
    if (o.set && o.splits <= p.k_tiles) {
        p.swap = o.swap;
        p.bq = o.bq;
        p.tiles_p = o.swap ? (N + 127) / 128 : (M + 127) / 128;
        p.tiles_q = o.swap ? (M + o.bq - 1) / o.bq : (N + o.bq - 1) / o.bq;
        p.splits = o.splits;
        // without row-major scale tiles, a narrow Q tile must start on a 128-row block
        if (sfr || p.bq >= 128 || p.tiles_q == 1) return p;
    }
    // Split K over a cluster of up to 8 CTAs (a power of two, so that the 128
    // tile rows divide evenly in the reduction) while the grid stays at or
    // below ~128 CTAs, which leaves room for the next kernel's CTAs to start
    // (programmatic dependent launch), and all of its clusters fit on the GPU
    // at once.  (Clusters of 16 win for one shape timed alone but lose in a
    // sequence of different shapes: they wait for whole free GPCs.)
    const int cap = std::min(num_sms, 128);
    auto splits_for = [&](int bq, int tiles) {
        int splits = 1;
        for (int s = 2; s <= max_splits && s <= p.k_tiles && tiles * s <= cap; s *= 2)
            if (split_cluster_capacity_of(info, p.swap, bq, sfr, s) >= tiles) splits = s;
        return splits;
    };
    // Tile shape (measured on the attention and MoE decode shapes): weight
    // rows on the 128-row MMA side with narrow token tiles for small M, then
    // 64- and 128-wide N tiles; 256-wide tiles once the grid is large.
    if (M <= 64) {
        p.swap = true;
        p.bq = M <= 16 ? 16 : 32;
        if (!sfr && M > p.bq) p.bq = 64;   // one Q tile: scale atoms start on row 0
    } else {
        p.swap = false;
        if (N <= 256 && M > 256)
            p.bq = M <= 512 ? 32 : 64;   // few weight columns: more, narrower tiles
        else
            p.bq = M <= 256 ? 64 : M <= 1024 ? 128 : (N >= 256 ? 256 : 128);
        // Tiles narrower than 128 (64 < M <= 256, or few weight columns),
        // unless they would need more tiles than SMs or leave each CTA a
        // stream of 12 or more K tiles: there the 128-wide tiles (which have
        // the second producer warp) win.  Graph-replayed, constant weights,
        // us (narrow -> 128-wide): 96 x 8192 x 8192 33.6 -> 23.2, 128 x 8192 x
        // 8192 21.7 -> 16.3, 128 x 4096 x 6144 11.9 -> 10.7, 256 x 2048 x 6144
        // 11.0 -> 10.2, 256 x 6144 x 768 11.8 -> 7.5, 256 x 8192 x 8192 38.1
        // -> 23.8, 2048 x 256 x 6144 10.8 -> 9.9; with shorter streams the
        // narrow tiles win or tie (128 x 2048 x 6144 8.5 against 9.2, 256 x
        // 1024 x 6144 8.25 against 8.96, 256 x 768 x 6144 and 512 x 256 x 6144
        // even).
        if (sfr && p.bq < 128) {
            const int tiles_n = ((M + 127) / 128) * ((N + p.bq - 1) / p.bq);
            if (tiles_n > num_sms || p.k_tiles / splits_for(p.bq, tiles_n) >= 12) p.bq = 128;
        }
        // Without row-major scale tiles the scales of a Q tile come as whole
        // 128-row atoms, so a narrower Q tile is only possible alone.
        if (!sfr && p.bq < 128 && N > p.bq) p.bq = 128;
    }
    p.tiles_p = p.swap ? (N + 127) / 128 : (M + 127) / 128;
    p.tiles_q = p.swap ? (M + p.bq - 1) / p.bq : (N + p.bq - 1) / p.bq;
    p.splits = splits_for(p.bq, p.tiles_p * p.tiles_q);
    return p;
}

// Split-K workspace of a plan: one fp32 partial tile per (tile, rank).
size_t splitk_ws_bytes(const Plan& p) {
    return p.splits > 1 ? (size_t)p.tiles_p * p.tiles_q * p.splits * (size_t)p.bq * 128u * 4u : 0;
}

// The workspace: per-stream scratch (allocated on a stream's first need of
// that size), or, when `fixed` is given, that caller-owned region of
// `fixed_cap` bytes (no allocation; too small -> UNSUPPORTED_SHAPE).
nvfp4_status splitk_ws(int dev, cudaStream_t stream, const Plan& p, uint8_t* fixed, size_t fixed_cap, float4** out) {
    *out = nullptr;
    const size_t bytes = splitk_ws_bytes(p);
    if (bytes == 0) return NVFP4_OK;
    if (fixed != nullptr) {
        if (bytes > fixed_cap) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        *out = reinterpret_cast<float4*>(fixed);
        return NVFP4_OK;
    }
    uint8_t* ptr = nullptr;
    const nvfp4_status st = get_scratch(dev, stream, bytes, &ptr, kScratchSplitK);
    *out = reinterpret_cast<float4*>(ptr);
    return st;
}

struct Maps {
    CUtensorMap p, q, sp, sq;
};

template <int BQ, bool SWAP, bool SPLITK, bool SFR, bool QBF16 = false, bool MX = false>
nvfp4_status launch_gemm_kernel(DeviceInfo* info, uint64_t bit, const Maps& m, const GemmParams& prm, dim3 grid,
                                cudaStream_t stream) {
    using C = TileConfig<BQ, SPLITK, QBF16>;
    auto kern = nvfp4::nvfp4_gemm_kernel<BQ, SWAP, SPLITK, SFR, QBF16, MX>;
    uint64_t& attr_set = MX ? info->smem_attr_set_mx : info->smem_attr_set;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(attr_set & bit)) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            // clusters of 16 split-K CTAs are opt-in (beyond the portable 8)
            if (SPLITK && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            attr_set |= bit;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(nvfp4::gemm_threads<BQ, SWAP, SFR, QBF16>(), 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    // Let this kernel's launch and prologue overlap the previous kernel in
    // the stream; the kernel waits for it before touching global memory.
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (SPLITK) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = grid.x;   // the split-K CTAs of one tile
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, m.p, m.q, m.sp, m.sq, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

template <bool SWAP, bool SPLITK, bool SFR>
nvfp4_status launch_by_bq(int bq, DeviceInfo* info, const Maps& m, const GemmParams& prm, dim3 grid,
                          cudaStream_t stream) {
    const int base = (SWAP ? 1 : 0) * 20 + (SPLITK ? 10 : 0) + (SFR ? 5 : 0);
    switch (bq) {
        case 16: return launch_gemm_kernel<16, SWAP, SPLITK, SFR>(info, 1ull << (base + 0), m, prm, grid, stream);
        case 32: return launch_gemm_kernel<32, SWAP, SPLITK, SFR>(info, 1ull << (base + 1), m, prm, grid, stream);
        case 64: return launch_gemm_kernel<64, SWAP, SPLITK, SFR>(info, 1ull << (base + 2), m, prm, grid, stream);
        case 128: return launch_gemm_kernel<128, SWAP, SPLITK, SFR>(info, 1ull << (base + 3), m, prm, grid, stream);
        case 256: return launch_gemm_kernel<256, SWAP, SPLITK, SFR>(info, 1ull << (base + 4), m, prm, grid, stream);
        default: return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
}

// Persistent large-tile kernel: one CTA per SM walking the tile list.
template <int BQ>
nvfp4_status launch_persistent(DeviceInfo* info, uint64_t bit, const Maps& m, const nvfp4::PersistParams& prm,
                               int tiles, cudaStream_t stream) {
    using C = nvfp4::PersistConfig<BQ>;
    auto kern = nvfp4::nvfp4_gemm_persistent_kernel<BQ>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(info->smem_attr_set & bit)) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            info->smem_attr_set |= bit;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(tiles, info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kPersistThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, m.p, m.q, m.sp, m.sq, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

// Whether large problems use the CTA-pair kernel: NVFP4_GEMM_PAIR=0 turns it
// off (the single-CTA persistent kernel runs instead), anything else or unset
// leaves it on.
bool pair_kernel_enabled() {
    const char* e = std::getenv("NVFP4_GEMM_PAIR");
    return !(e && e[0] == '0');
}

// Whether nvfp4_gemm runs the CUDA-core kernel for a few activation rows
// (nvfp4_gemv_kernel) instead of the tensor-core kernels.  Measured on
// graph-replayed back-to-back calls (us per call, tensor cores -> CUDA cores):
// M = 1 wins everywhere (768x6144 5.8 -> 2.7, 2048x6144 7.2 -> 3.6,
// 8192x8192 12.9 -> 11.3, 6144x768 5.5 -> 4.3); M = 2 wins with K >= 4096 up
// to N = 2048 (7.2 -> 4.9) and loses at 8192x8192 and at K = 768, where most
// of a CTA's threads have no K chunk; M = 4 wins only up to N ~ 768 (5.9 ->
// 4.3); M >= 8 loses.  NVFP4_GEMM_GEMV=0 turns the kernel off;
// NVFP4_GEMM_GEMV=<n> (1..16) sends every M <= n to it (tuning and tests);
// NVFP4_GEMM_GEMV_RW=1|2|4 forces the weight rows per CTA.
bool use_gemv_areg(int M, int K);

bool use_gemv(int M, int N, int K) {
    if (plan_override().set) return false;
    if (const char* e = std::getenv("NVFP4_GEMM_GEMV")) {
        const int v = std::atoi(e);
        return M <= (v < 0 ? 0 : v > 16 ? 16 : v);
    }
    if (M == 1) return true;
    if (M == 2 && use_gemv_areg(M, K)) return true;   // 8192 x 8192: 13.1 against 15.1 us
    if (K < 4096) return false;
    return (M == 2 && N <= 4096) || (M <= 4 && N <= 1024);
}

// At most as many CTAs as fit on the GPU at once (the kernel walks the rest
// of the row groups itself).
template <int MT, int RW>
nvfp4_status launch_gemv_kernel(DeviceInfo* info, const nvfp4::GemvParams& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_kernel<MT, RW>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

template <int MT>
nvfp4_status launch_gemv_rw(DeviceInfo* info, int rw, const nvfp4::GemvParams& prm, cudaStream_t stream) {
    switch (rw) {
        case 1: return launch_gemv_kernel<MT, 1>(info, prm, stream);
        case 2: return launch_gemv_kernel<MT, 2>(info, prm, stream);
        default:
            if constexpr (MT >= 16) return launch_gemv_kernel<MT, 2>(info, prm, stream);   // 4 x 16 would spill
            else return launch_gemv_kernel<MT, 4>(info, prm, stream);
    }
}

// The one-or-two-row form with the token chunks held in registers
// (nvfp4_gemv_areg_kernel): M <= 2 and at most four chunks per thread for one
// row (K <= 16384), two for two rows (K <= 8192).  NVFP4_GEMV_AREG=0 turns it
// off (the general kernel then runs).
template <int MT, int RW, int CPT>
nvfp4_status launch_gemv_areg(DeviceInfo* info, const nvfp4::GemvParams& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_areg_kernel<MT, RW, CPT>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

template <int MT, int CPT>
nvfp4_status launch_gemv_areg_rw(DeviceInfo* info, int rw, const nvfp4::GemvParams& prm, cudaStream_t stream) {
    switch (rw) {
        case 1: return launch_gemv_areg<MT, 1, CPT>(info, prm, stream);
        case 2: return launch_gemv_areg<MT, 2, CPT>(info, prm, stream);
        default: return launch_gemv_areg<MT, 4, CPT>(info, prm, stream);
    }
}

bool use_gemv_areg(int M, int K) {
    if (const char* e = std::getenv("NVFP4_GEMV_AREG"))
        if (e[0] == '0' && e[1] == '\0') return false;
    const int cpt = (K / 32 + nvfp4::kGemvThreads - 1) / nvfp4::kGemvThreads;
    return M >= 1 && M <= 2 && M * cpt <= 4;
}

nvfp4_status gemv_areg_gemm(DeviceInfo* info, int rw, const nvfp4::GemvParams& prm, cudaStream_t stream) {
    const int cpt = (prm.K / 32 + nvfp4::kGemvThreads - 1) / nvfp4::kGemvThreads;
    if (prm.M == 1) {
        if (cpt <= 1) return launch_gemv_areg_rw<1, 1>(info, rw, prm, stream);
        if (cpt <= 2) return launch_gemv_areg_rw<1, 2>(info, rw, prm, stream);
        return launch_gemv_areg_rw<1, 4>(info, rw, prm, stream);
    }
    if (cpt <= 1) return launch_gemv_areg_rw<2, 1>(info, rw, prm, stream);
    return launch_gemv_areg_rw<2, 2>(info, rw, prm, stream);
}

// The CUDA-core path for M <= 16.  Weight rows per CTA (measured): one row
// for a single token row and a small matrix (spread over the most CTAs),
// four from N = 2048 up, two with two or more token rows (each decoded
// activation chunk serves both rows).
nvfp4_status gemv_gemm(DeviceInfo* info, const void* A, const void* sA, const void* B, const void* sB, float alpha,
                       void* D, int M, int N, int K, unsigned flags, cudaStream_t stream) {
    nvfp4::GemvParams prm{};
    prm.A = static_cast<const uint8_t*>(A);
    prm.sA = static_cast<const uint8_t*>(sA);
    prm.B = static_cast<const uint8_t*>(B);
    prm.sB = static_cast<const uint8_t*>(sB);
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.prefetch_b = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
    int rw = M == 1 ? (N >= 2048 ? 4 : 1) : 2;
    if (use_gemv_areg(M, K)) {
        // measured (us, 1 row): 2048 x 6144 rw4 2.55-2.68 / rw2 2.53-3.07
        // (four runs); 8192 x 8192 rw4 7.73 / rw2 8.65; 768 x 6144 rw1 1.82 /
        // rw2 1.99.  Two rows: 256 x 6144 rw1 2.16 / rw2 2.38; 2048 x 6144
        // rw2 4.03 / rw4 4.90; 8192 x 8192 rw4 12.7 / rw2 12.4-14.6.
        rw = M == 1 ? (N >= 2048 ? 4 : 1) : (N >= 4096 ? 4 : (N <= 256 ? 1 : 2));
    }
    if (const char* e = std::getenv("NVFP4_GEMM_GEMV_RW")) {
        const int v = std::atoi(e);
        if (v == 1 || v == 2 || v == 4) rw = v;
    }
    if (use_gemv_areg(M, K)) return gemv_areg_gemm(info, rw, prm, stream);
    if (M <= 1) return launch_gemv_rw<1>(info, rw, prm, stream);
    if (M <= 2) return launch_gemv_rw<2>(info, rw, prm, stream);
    if (M <= 4) return launch_gemv_rw<4>(info, rw, prm, stream);
    if (M <= 8) return launch_gemv_rw<8>(info, rw, prm, stream);
    return launch_gemv_rw<16>(info, rw, prm, stream);
}

// ---------------------------------------------------- 2:4-sparse weights
template <int MT, int RW>
nvfp4_status launch_gemv_sp24_kernel(DeviceInfo* info, const nvfp4::GemvSp24Params& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_sp24_kernel<MT, RW>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

// One or two token rows: nvfp4_gemv_sp24_areg_kernel (the token chunks held
// in registers), with the same limits as the dense form.
template <int MT, int RW, int CPT>
nvfp4_status launch_gemv_sp24_areg(DeviceInfo* info, const nvfp4::GemvSp24Params& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_sp24_areg_kernel<MT, RW, CPT>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

template <int MT, int CPT>
nvfp4_status launch_gemv_sp24_areg_rw(DeviceInfo* info, int rw, const nvfp4::GemvSp24Params& prm,
                                      cudaStream_t stream) {
    switch (rw) {
        case 1: return launch_gemv_sp24_areg<MT, 1, CPT>(info, prm, stream);
        case 2: return launch_gemv_sp24_areg<MT, 2, CPT>(info, prm, stream);
        default: return launch_gemv_sp24_areg<MT, 4, CPT>(info, prm, stream);
    }
}

nvfp4_status gemv_sp24_areg_gemm(DeviceInfo* info, int rw, const nvfp4::GemvSp24Params& prm, cudaStream_t stream) {
    const int cpt = (prm.K / 32 + nvfp4::kGemvThreads - 1) / nvfp4::kGemvThreads;
    if (prm.M == 1) {
        if (cpt <= 1) return launch_gemv_sp24_areg_rw<1, 1>(info, rw, prm, stream);
        if (cpt <= 2) return launch_gemv_sp24_areg_rw<1, 2>(info, rw, prm, stream);
        return launch_gemv_sp24_areg_rw<1, 4>(info, rw, prm, stream);
    }
    if (cpt <= 1) return launch_gemv_sp24_areg_rw<2, 1>(info, rw, prm, stream);
    return launch_gemv_sp24_areg_rw<2, 2>(info, rw, prm, stream);
}

template <int MT>
nvfp4_status launch_gemv_sp24_rw(DeviceInfo* info, int rw, const nvfp4::GemvSp24Params& prm, cudaStream_t stream) {
    if (rw == 1) return launch_gemv_sp24_kernel<MT, 1>(info, prm, stream);
    if constexpr (MT <= 2) {
        if (rw == 4) return launch_gemv_sp24_kernel<MT, 4>(info, prm, stream);
    }
    return launch_gemv_sp24_kernel<MT, 2>(info, prm, stream);
}

// Token rows up to which the 2:4-sparse GEMM runs the CUDA-core kernel on the
// compressed weights; above it the weights are expanded to dense codes in
// scratch and the dense GEMM runs.  NVFP4_GEMM_SP24_GEMV=<n> (0..16) moves
// the limit (tuning and tests).
int sp24_gemv_max_m() {
    if (const char* e = std::getenv("NVFP4_GEMM_SP24_GEMV")) {
        const int v = std::atoi(e);
        return v < 0 ? 0 : v > 16 ? 16 : v;
    }
    return 8;
}

nvfp4_status launch_pair(DeviceInfo* info, const CUtensorMap& tmA, const CUtensorMap& tmB,
                         const nvfp4::PairParams& prm, cudaStream_t stream) {
    using C = nvfp4::PairConfig;
    auto kern = nvfp4::nvfp4_gemm_pair_kernel;
    int clusters;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(info->smem_attr_set & (1ull << 59))) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            info->smem_attr_set |= (1ull << 59);
        }
        if (info->pair_clusters < 0) {
            // A persistent grid larger than what fits at once would serialise
            // whole clusters: size it by the co-resident cluster count.
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(2, 1, 1);
            q.blockDim = dim3(nvfp4::kPairThreads, 1, 1);
            q.dynamicSmemBytes = C::SMEM_BYTES;
            cudaLaunchAttribute ca[1];
            ca[0].id = cudaLaunchAttributeClusterDimension;
            ca[0].val.clusterDim.x = 2;
            ca[0].val.clusterDim.y = 1;
            ca[0].val.clusterDim.z = 1;
            q.attrs = ca;
            q.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) {
                cudaGetLastError();
                return NVFP4_ERR_CUDA;
            }
            info->pair_clusters = n;
        }
        clusters = info->pair_clusters;
    }
    const int tiles = prm.tiles_m * prm.tiles_n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * (unsigned)std::min(tiles, clusters), 1, 1);
    cfg.blockDim = dim3(nvfp4::kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

// The CTA-pair kernel: scales re-laid out into tensor-core atoms in scratch,
// then 256 x 256 tiles on CTA pairs.
nvfp4_status pair_gemm(int dev, DeviceInfo* info, const void* A, const void* sA, const void* B, const void* sB,
                       float alpha, void* D, int M, int N, int K, cudaStream_t stream) {
    const size_t sfa_bytes = nvfp4_swizzled_scale_bytes(M, K);
    const size_t off_sfb = align_up(sfa_bytes, 256);
    const size_t sfb_bytes = nvfp4_swizzled_scale_bytes(N, K);
    uint8_t* ws = nullptr;
    nvfp4_status st = get_scratch(dev, stream, off_sfb + sfb_bytes, &ws);
    if (st != NVFP4_OK) return st;
    CUtensorMap tmA, tmB;
    if (!make_operand_map(&tmA, A, M, K / 2, 128) || !make_operand_map(&tmB, B, N, K / 2, 128)) return NVFP4_ERR_CUDA;
    {
        nvfp4::ScaleTileJob ja{static_cast<const uint8_t*>(sA), ws, M, (M + 127) / 128, aligned(sA, 16) ? 1 : 0};
        nvfp4::ScaleTileJob jb{static_cast<const uint8_t*>(sB), ws + off_sfb, N, (N + 127) / 128,
                               aligned(sB, 16) ? 1 : 0};
        const long long blocks = (long long)(ja.row_blocks + jb.row_blocks) * (K / 256);
        nvfp4::swizzle_scale_tiles_kernel<<<(unsigned)blocks, 128, 0, stream>>>(ja, jb, K / 16, K / 256);
        g_launches++;
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    nvfp4::PairParams pp{};
    pp.D = static_cast<__nv_bfloat16*>(D);
    pp.sfa = ws;
    pp.sfb = ws + off_sfb;
    pp.alpha = alpha;
    pp.M = M;
    pp.N = N;
    pp.K = K;
    pp.k_tiles = K / 256;
    pp.tiles_m = (M + nvfp4::kPairBM - 1) / nvfp4::kPairBM;
    pp.tiles_n = (N + nvfp4::kPairBN - 1) / nvfp4::kPairBN;
    pp.rb_a = (M + 127) / 128;
    pp.rb_b = (N + 127) / 128;
    return launch_pair(info, tmA, tmB, pp, stream);
}

template <bool SFR>
nvfp4_status launch_mode(const Plan& plan, DeviceInfo* info, const Maps& m, const GemmParams& prm, dim3 grid,
                         cudaStream_t stream) {
    if (plan.swap)
        return plan.splits > 1 ? launch_by_bq<true, true, SFR>(plan.bq, info, m, prm, grid, stream)
                               : launch_by_bq<true, false, SFR>(plan.bq, info, m, prm, grid, stream);
    return plan.splits > 1 ? launch_by_bq<false, true, SFR>(plan.bq, info, m, prm, grid, stream)
                           : launch_by_bq<false, false, SFR>(plan.bq, info, m, prm, grid, stream);
}

// ------------------------------------------------- split-K kernel for few token rows
// Plan of nvfp4_gemm_splitk_kernel: weights in 128-row tiles against the
// token rows (swapped, M <= 64), or token rows in 128-row tiles against 64-
// or 128-row weight tiles; K split over a cluster of up to 16 CTAs; every
// CTA small enough to share its SM with a CTA of the next launch.
struct SkPlan {
    bool use = false;
    bool swap = false;
    int bq = 0, splits = 1, stages = 1, tiles_p = 0, tiles_q = 0;
    int smem = 0;
    uint32_t tmem_cols = 32;
};

// Two CTAs of at most this much dynamic shared memory fit an SM (228 KB, less
// 1 KB reserved per CTA); a CTA above kSkSoloSmem has its SM to itself.
constexpr int kSkCoresidentSmem = 115712;
constexpr int kSkSoloSmem = 118784;

template <int BQ>
void sk_fill(SkPlan& p, int nkt, int max_stages) {
    using C = nvfp4::SkConfig<BQ>;
    const bool split = p.splits > 1;
    const int want = std::min({nkt, nvfp4::kSkMaxStages, max_stages});
    // Co-resident: the whole K slice in a ring that leaves room for a CTA of
    // the next launch.  Otherwise the deepest ring that fits (the SM to this
    // CTA): a ring shallower than the K slice is bound by its round trips.
    int stages = want;
    while (stages > 1 && nvfp4::sk_smem_bytes<BQ>(stages, split) > kSkCoresidentSmem) --stages;
    bool solo = false;
    if (stages < want) {
        int deep = want;
        while (deep > 1 && nvfp4::sk_smem_bytes<BQ>(deep, split) > nvfp4::kSmemLimit) --deep;
        if (deep > stages) {
            stages = deep;
            solo = true;
        }
    }
    p.stages = std::max(1, stages);
    p.smem = nvfp4::sk_smem_bytes<BQ>(p.stages, split);
    const int cols = C::ACC_COLS + p.stages * C::SF_STRIDE;
    p.tmem_cols = cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
    // More than half of TMEM, or a deep ring: keep the SM to this CTA (a
    // second CTA's TMEM allocation would wait for the first to finish).
    if (solo || p.tmem_cols > 256) p.smem = std::max(p.smem, kSkSoloSmem);
}

// The plan: swapped tiles up to 64 token rows; above that 128 token rows
// against 64 weight rows.  K is split so that the CTAs all run at once, and
// little enough that the fp32 partials exchanged (splits x M x N x 4 bytes)
// stay near the size of the weights (N x K / 2 bytes).
// NVFP4_GEMM_SK=0 turns the kernel off; NVFP4_GEMM_SK="swap:bq:splits:stages"
// forces a plan where it runs (tuning and tests).
SkPlan make_sk_plan(int M, int N, int K, const DeviceInfo* info) {
    SkPlan p;
    int f_swap = -1, f_bq = 0, f_splits = 0, f_stages = 0;
    if (const char* e = std::getenv("NVFP4_GEMM_SK")) {
        if (e[0] == '0' && e[1] == '\0') return p;
        int a = 0, b = 0, c = 0, d = 0;
        if (std::sscanf(e, "%d:%d:%d:%d", &a, &b, &c, &d) == 4 && (c == 1 || c == 2 || c == 4 || c == 8 || c == 16) &&
            d >= 1 && d <= nvfp4::kSkMaxStages &&
            ((a == 1 && (b == 16 || b == 32 || b == 64)) || (a == 0 && (b == 64 || b == 128)))) {
            f_swap = a;
            f_bq = b;
            f_splits = c;
            f_stages = d;
        }
    }
    // Measured against the tiled split-K kernel (graph-replayed back-to-back
    // calls, constant weights): this kernel is faster up to 16 token rows
    // (768 x 6144: 5.3 against 6.1 us; 2048 x 6144: 6.9 against 7.8;
    // 256 x 6144: 4.5 against 5.7) and for 64 rows against 256 weight rows;
    // beyond that the tiled kernel's deeper K pipeline wins.  It also loses
    // with many weight tiles or a short K (8192 x 8192: 20.0 against 13.0 us;
    // 6144 x 768: 7.2 against 5.5), so it takes at most 2048 weight rows and
    // K >= 2048.
    const int k_tiles = K / 256;
    if (f_swap < 0 && !((M <= 16 || (M <= 64 && N <= 256)) && N <= 2048 && k_tiles >= 8)) return p;
    p.swap = f_swap >= 0 ? f_swap == 1 : M <= 64;
    if (p.swap) {
        p.bq = f_bq ? f_bq : (M <= 16 ? 16 : 32);
        p.tiles_p = (N + 127) / 128;
        p.tiles_q = (M + p.bq - 1) / p.bq;
    } else {
        p.bq = f_bq ? f_bq : 64;
        p.tiles_p = (M + 127) / 128;
        p.tiles_q = (N + p.bq - 1) / p.bq;
    }
    const int tiles = p.tiles_p * p.tiles_q;
    if (tiles > info->num_sms) return p;   // enough tiles without splitting K: the other kernels
    const int max_stages = f_stages ? f_stages : nvfp4::kSkMaxStages;
    auto fill = [&](int splits) {
        p.splits = splits;
        const int nkt = (k_tiles + splits - 1) / splits;
        switch (p.bq) {
            case 16: sk_fill<16>(p, nkt, max_stages); break;
            case 32: sk_fill<32>(p, nkt, max_stages); break;
            case 64: sk_fill<64>(p, nkt, max_stages); break;
            default: sk_fill<128>(p, nkt, max_stages); break;
        }
    };
    if (f_splits) {
        int splits = std::min(f_splits, std::max(1, k_tiles));
        while (splits > 1 && 128 % splits != 0) splits /= 2;
        fill(splits);
    } else {
        // The largest split (a power of two up to 16, at most one per K tile)
        // whose CTAs all run at once -- two per SM when they are small enough
        // to share one, else one -- and whose fp32 partials stay within twice
        // the weight bytes.
        int splits = 16;
        for (; splits > 1; splits /= 2) {
            if (splits > k_tiles || (long long)splits * M * 8 > 2LL * K) continue;
            fill(splits);
            const int per_sm = p.smem <= kSkCoresidentSmem ? 2 : 1;
            if (tiles * splits <= per_sm * info->num_sms) break;
        }
        if (splits == 1) fill(1);
    }
    p.use = true;
    return p;
}

template <int BQ, bool SWAP>
nvfp4_status launch_sk_kernel(DeviceInfo* info, uint64_t bit, const Maps& m, const nvfp4::SkParams& prm,
                              const SkPlan& plan, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemm_splitk_kernel<BQ, SWAP>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(info->smem_attr_set & bit)) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, nvfp4::kSmemLimit) !=
                    cudaSuccess ||
                cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
                cudaGetLastError();
                return NVFP4_ERR_CUDA;
            }
            info->smem_attr_set |= bit;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.splits, (unsigned)(plan.tiles_p * plan.tiles_q), 1);
    cfg.blockDim = dim3(nvfp4::kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (plan.splits > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)plan.splits;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, m.p, m.q, m.sp, m.sq, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

// Split-K workspace of the split-K kernel: one fp32 partial tile per (tile, rank).
size_t sk_ws_bytes(const SkPlan& p) {
    return p.splits > 1 ? (size_t)p.tiles_p * p.tiles_q * p.splits * (size_t)p.bq * 128u * 4u : 0;
}

// `ws_fixed`: the caller-owned workspace of nvfp4_gemm_noalloc (at least
// sk_ws_bytes(plan) bytes), else per-stream scratch.
nvfp4_status sk_gemm(int dev, DeviceInfo* info, const SkPlan& plan, const void* A, const void* sA, const void* B,
                     const void* sB, float alpha, void* D, int M, int N, int K, unsigned flags, cudaStream_t stream,
                     uint8_t* ws_fixed = nullptr) {
    const void* P = plan.swap ? B : A;
    const void* Q = plan.swap ? A : B;
    const void* sP = plan.swap ? sB : sA;
    const void* sQ = plan.swap ? sA : sB;
    const int rows_p = plan.swap ? N : M;
    const int rows_q = plan.swap ? M : N;
    Maps maps;
    if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq) ||
        !make_scale_map(&maps.sp, sP, rows_p, K / 16, 128) || !make_scale_map(&maps.sq, sQ, rows_q, K / 16, plan.bq))
        return NVFP4_ERR_CUDA;
    nvfp4::SkParams prm{};
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.rows_p = rows_p;
    prm.rows_q = rows_q;
    prm.ldd = N;
    prm.k_tiles = K / 256;
    prm.tiles_q = plan.tiles_q;
    prm.stages = plan.stages;
    prm.prefetch_w = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
    prm.tmem_cols = plan.tmem_cols;
    const size_t ws_bytes = sk_ws_bytes(plan);
    if (ws_bytes > 0) {
        uint8_t* ws = ws_fixed;
        if (ws == nullptr) {
            const nvfp4_status st = get_scratch(dev, stream, ws_bytes, &ws, kScratchSplitK);
            if (st != NVFP4_OK) return st;
        }
        prm.ws = reinterpret_cast<float4*>(ws);
    }
    if (plan.swap) {
        switch (plan.bq) {
            case 16: return launch_sk_kernel<16, true>(info, 1ull << 50, maps, prm, plan, stream);
            case 32: return launch_sk_kernel<32, true>(info, 1ull << 51, maps, prm, plan, stream);
            default: return launch_sk_kernel<64, true>(info, 1ull << 52, maps, prm, plan, stream);
        }
    }
    return plan.bq == 64 ? launch_sk_kernel<64, false>(info, 1ull << 54, maps, prm, plan, stream)
                         : launch_sk_kernel<128, false>(info, 1ull << 53, maps, prm, plan, stream);
}

// The tensor-core GEMM with row-major scale tiles loaded by TMA (K % 256 == 0,
// scales 16-byte aligned).  Few token rows take the split-K kernel, large
// problems the single-CTA persistent kernel, the others the tiled kernel of
// the plan, whose split-K partials need a workspace: per-stream scratch, or
// with `ws_fixed` that caller-owned region (when the plan's workspace does
// not fit it, the plan is made again without a K split).
nvfp4_status sfr_gemm(int dev, DeviceInfo* info, Plan plan, const void* A, const void* sA, const void* B,
                      const void* sB, float alpha, void* D, int M, int N, int K, unsigned flags,
                      cudaStream_t stream, uint8_t* ws_fixed = nullptr, size_t ws_cap = 0) {
    if (!plan_override().set) {
        const SkPlan sk = make_sk_plan(M, N, K, info);
        if (sk.use && (ws_fixed == nullptr || sk_ws_bytes(sk) <= ws_cap))
            return sk_gemm(dev, info, sk, A, sA, B, sB, alpha, D, M, N, K, flags, stream, ws_fixed);
    }
    if (ws_fixed != nullptr && splitk_ws_bytes(plan) > ws_cap) plan = make_plan(M, N, K, info, true, 1);
    const void* P = plan.swap ? B : A;
    const void* Q = plan.swap ? A : B;
    const void* sP = plan.swap ? sB : sA;
    const void* sQ = plan.swap ? sA : sB;
    const int rows_p = plan.swap ? N : M;
    const int rows_q = plan.swap ? M : N;
    Maps maps;
    if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq) ||
        !make_scale_map(&maps.sp, sP, rows_p, K / 16, 128) || !make_scale_map(&maps.sq, sQ, rows_q, K / 16, plan.bq))
        return NVFP4_ERR_CUDA;
    const int tiles = plan.tiles_p * plan.tiles_q;
    if (!plan.swap && plan.splits == 1 && tiles > info->num_sms && (plan.bq == 128 || plan.bq == 256) &&
        !plan_override().set) {
        nvfp4::PersistParams pp{};
        pp.D = static_cast<__nv_bfloat16*>(D);
        pp.alpha = alpha;
        pp.M = M;
        pp.N = N;
        pp.K = K;
        pp.k_tiles = K / 256;
        pp.tiles_m = plan.tiles_p;
        pp.tiles_n = plan.tiles_q;
        return plan.bq == 256 ? launch_persistent<256>(info, 1ull << 60, maps, pp, tiles, stream)
                              : launch_persistent<128>(info, 1ull << 61, maps, pp, tiles, stream);
    }
    GemmParams prm{};
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.rows_p = rows_p;
    prm.rows_q = rows_q;
    prm.K = K;
    prm.ldd = N;
    prm.k_tiles = plan.k_tiles;
    prm.tiles_q = plan.tiles_q;
    prm.prefetch_b = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
    nvfp4_status st = splitk_ws(dev, stream, plan, ws_fixed, ws_cap, &prm.ws);
    if (st != NVFP4_OK) return st;
    const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
    return launch_mode<true>(plan, info, maps, prm, grid, stream);
}

// The MXFP4 instantiations (scale atoms pre-laid out, never row-major tiles).
template <bool SWAP, bool SPLITK>
nvfp4_status launch_mx_by_bq(int bq, DeviceInfo* info, const Maps& m, const GemmParams& prm, dim3 grid,
                             cudaStream_t stream) {
    const int base = (SWAP ? 1 : 0) * 10 + (SPLITK ? 5 : 0);
    switch (bq) {
        case 16: return launch_gemm_kernel<16, SWAP, SPLITK, false, false, true>(info, 1ull << (base + 0), m, prm, grid, stream);
        case 32: return launch_gemm_kernel<32, SWAP, SPLITK, false, false, true>(info, 1ull << (base + 1), m, prm, grid, stream);
        case 64: return launch_gemm_kernel<64, SWAP, SPLITK, false, false, true>(info, 1ull << (base + 2), m, prm, grid, stream);
        case 128: return launch_gemm_kernel<128, SWAP, SPLITK, false, false, true>(info, 1ull << (base + 3), m, prm, grid, stream);
        case 256: return launch_gemm_kernel<256, SWAP, SPLITK, false, false, true>(info, 1ull << (base + 4), m, prm, grid, stream);
        default: return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
}

// The row-major-scale (SFR) MXFP4 instances: bits 20.. of the MX attribute mask.
template <bool SWAP, bool SPLITK>
nvfp4_status launch_mx_sfr_by_bq(int bq, DeviceInfo* info, const Maps& m, const GemmParams& prm, dim3 grid,
                                 cudaStream_t stream) {
    const int base = 20 + (SWAP ? 1 : 0) * 10 + (SPLITK ? 5 : 0);
    switch (bq) {
        case 16: return launch_gemm_kernel<16, SWAP, SPLITK, true, false, true>(info, 1ull << (base + 0), m, prm, grid, stream);
        case 32: return launch_gemm_kernel<32, SWAP, SPLITK, true, false, true>(info, 1ull << (base + 1), m, prm, grid, stream);
        case 64: return launch_gemm_kernel<64, SWAP, SPLITK, true, false, true>(info, 1ull << (base + 2), m, prm, grid, stream);
        case 128: return launch_gemm_kernel<128, SWAP, SPLITK, true, false, true>(info, 1ull << (base + 3), m, prm, grid, stream);
        case 256: return launch_gemm_kernel<256, SWAP, SPLITK, true, false, true>(info, 1ull << (base + 4), m, prm, grid, stream);
        default: return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
}

nvfp4_status launch_swizzle_mx(const void* s, int rows, int K, void* out, cudaStream_t stream) {
    const int pairs = (K / 64 + 1) / 2;
    const long long lines = (long long)((rows + 127) / 128) * pairs * 32;
    if (lines == 0) return NVFP4_OK;
    const int threads = 256;
    const long long blocks = (lines + threads - 1) / threads;
    nvfp4::swizzle_scales_mx_kernel<<<(unsigned)blocks, threads, 0, stream>>>(static_cast<const uint8_t*>(s), rows,
                                                                            K / 32, pairs, lines,
                                                                            static_cast<uint8_t*>(out));
    g_launches++;
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

size_t mx_atom_bytes(int rows, int K) { return (size_t)((rows + 127) / 128) * (size_t)((K / 64 + 1) / 2) * 512u; }

template <int MT, int RW, int CPT>
nvfp4_status launch_gemv_mx_areg(DeviceInfo* info, const nvfp4::GemvMxParams& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_mx_areg_kernel<MT, RW, CPT>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

template <int MT, int CPT>
nvfp4_status launch_gemv_mx_areg_rw(DeviceInfo* info, int rw, const nvfp4::GemvMxParams& prm, cudaStream_t stream) {
    switch (rw) {
        case 1: return launch_gemv_mx_areg<MT, 1, CPT>(info, prm, stream);
        case 2: return launch_gemv_mx_areg<MT, 2, CPT>(info, prm, stream);
        default: return launch_gemv_mx_areg<MT, 4, CPT>(info, prm, stream);
    }
}

template <int MT, int RW>
nvfp4_status launch_gemv_mx_kernel(DeviceInfo* info, const nvfp4::GemvMxParams& prm, cudaStream_t stream) {
    auto kern = nvfp4::nvfp4_gemv_mx_kernel<MT, RW>;
    static const int per_sm = [kern] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, nvfp4::kGemvThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            b = 0;
        }
        return b > 0 ? b : 1;
    }();
    const int groups = (prm.N + RW - 1) / RW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(groups, per_sm * info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGemvThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

nvfp4_status check_gemm_args(const void* A, const void* sA, const void* B, const void* sB, const void* D, int M,
                             int N, int K) {
    if (M < 0 || N < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!A || !sA || !B || !sB || !D) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) || !aligned(sB, 4))
        return NVFP4_ERR_INVALID_ARG;
    return NVFP4_OK;
}

}  // namespace

extern "C" {

int nvfp4_version(void) { return kVersion; }

unsigned long long nvfp4_kernel_launches(void) { return g_launches.load(); }

const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE";
        case NVFP4_ERR_UNSUPPORTED_DEVICE: return "NVFP4_ERR_UNSUPPORTED_DEVICE";
        case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
        case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
        case NVFP4_ERR_NO_MEMORY: return "NVFP4_ERR_NO_MEMORY";
    }
    return "NVFP4_ERR_UNKNOWN";
}

size_t nvfp4_swizzled_scale_bytes(int rows, int K) {
    if (rows < 0 || K <= 0 || K % 64 != 0) return 0;
    return (size_t)((rows + 127) / 128) * (size_t)(K / 64) * 512u;
}

nvfp4_status nvfp4_swizzle_scales(const void* s, int rows, int K, void* out, void* stream) {
    if (rows < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0) return NVFP4_OK;
    if (!s || !out || !aligned(s, 4) || !aligned(out, 16)) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    return launch_swizzle(s, rows, K, out, static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_quantize(const float* X, int rows, int K, void* codes, void* scales, float* g_out,
                            void* stream_) {
    if (rows < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!g_out || (rows > 0 && (!X || !codes || !scales))) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!aligned(X, 16) || !aligned(codes, 8))) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(g_out, 4)) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (cudaMemsetAsync(g_out, 0, sizeof(float), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    const long long n = (long long)rows * K;
    if (n > 0) {
        const long long n4 = n / 4;
        const int threads = 256;
        const int blocks = (int)std::min<long long>((n4 + threads - 1) / threads, (long long)info->num_sms * 8);
        nvfp4::amax_kernel<<<std::max(blocks, 1), threads, 0, stream>>>(reinterpret_cast<const float4*>(X), n4,
                                                                        reinterpret_cast<unsigned*>(g_out));
        const long long nb = n / 16;
        nvfp4::quantize_kernel<<<(unsigned)((nb + threads - 1) / threads), threads, 0, stream>>>(
            X, nb, reinterpret_cast<const unsigned*>(g_out), static_cast<uint8_t*>(codes),
            static_cast<uint8_t*>(scales));
        g_launches += 2;
    }
    nvfp4::finalize_global_scale_kernel<<<1, 1, 0, stream>>>(g_out);
    g_launches++;
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_gemm(const void* A, const void* sA, const void* B, const void* sB, float alpha, void* D, int M,
                        int N, int K, void* stream_) {
    return nvfp4_gemm_ex(A, sA, B, sB, alpha, D, M, N, K, 0u, stream_);
}

nvfp4_status nvfp4_gemm_ex(const void* A, const void* sA, const void* B, const void* sB, float alpha, void* D, int M,
                           int N, int K, unsigned flags, void* stream_) {
    if (flags & ~NVFP4_GEMM_B_CONSTANT) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_gemm_args(A, sA, B, sB, D, M, N, K);
    if (st != NVFP4_OK || M == 0 || N == 0) return st;
    int dev;
    DeviceInfo* info;
    st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (use_gemv(M, N, K)) return gemv_gemm(info, A, sA, B, sB, alpha, D, M, N, K, flags, stream);

    // Scales go to the kernel row-major (TMA tiles, laid out for the tensor
    // cores inside the kernel) when a 256-element K tile of scales is a
    // 16-byte aligned TMA box; otherwise they are re-laid out in global
    // scratch first.
    const bool sfr = (K % 256 == 0) && aligned(sA, 16) && aligned(sB, 16);
    const Plan plan = make_plan(M, N, K, info, sfr);
    // Enough 128 x 256 tiles to fill the SMs twice over: the CTA-pair kernel
    // on 256 x 256 tiles (measured faster than the split-K and single-CTA
    // persistent plans from 512 x 6144 and 768 x 4096 up, and on every
    // saturation shape).
    if (K % 256 == 0 && !plan.swap && plan.splits == 1 && M >= 512 && N >= 512 &&
        2 * ((M + 127) / 128) * ((N + 255) / 256) >= info->num_sms && pair_kernel_enabled() &&
        !plan_override().set)
        return pair_gemm(dev, info, A, sA, B, sB, alpha, D, M, N, K, stream);
    if (sfr) return sfr_gemm(dev, info, plan, A, sA, B, sB, alpha, D, M, N, K, flags, stream);

    // Scales re-laid out into tensor-core atoms in per-stream scratch.
    const void* P = plan.swap ? B : A;
    const void* Q = plan.swap ? A : B;
    const void* sP = plan.swap ? sB : sA;
    const void* sQ = plan.swap ? sA : sB;
    const int rows_p = plan.swap ? N : M;
    const int rows_q = plan.swap ? M : N;
    const size_t sfp_bytes = nvfp4_swizzled_scale_bytes(rows_p, K);
    const size_t sfq_bytes = nvfp4_swizzled_scale_bytes(rows_q, K);
    const size_t off_sfq = align_up(sfp_bytes, 256);
    uint8_t* ws = nullptr;
    if ((st = get_scratch(dev, stream, off_sfq + sfq_bytes, &ws)) != NVFP4_OK) return st;
    Maps maps;
    if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq))
        return NVFP4_ERR_CUDA;
    if ((st = launch_swizzle(sP, rows_p, K, ws, stream)) != NVFP4_OK) return st;
    if ((st = launch_swizzle(sQ, rows_q, K, ws + off_sfq, stream)) != NVFP4_OK) return st;
    maps.sp = maps.p;
    maps.sq = maps.q;
    GemmParams prm{};
    prm.sfp = ws;
    prm.sfq = ws + off_sfq;
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.rows_p = rows_p;
    prm.rows_q = rows_q;
    prm.K = K;
    prm.ldd = N;
    prm.k_tiles = plan.k_tiles;
    prm.tiles_q = plan.tiles_q;
    prm.prefetch_b = 0;   // the early prefetch reads row-major scale tiles only
    if ((st = splitk_ws(dev, stream, plan, nullptr, 0, &prm.ws)) != NVFP4_OK) return st;
    const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
    return launch_mode<false>(plan, info, maps, prm, grid, stream);
}

nvfp4_status nvfp4_grouped_gemm(const void* A, const void* sA, const void* B, const void* sB, const float* alpha,
                                const int32_t* row_offsets, int G, void* D, int M_total, int N, int K,
                                void* stream_) {
    if (G < 1) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_gemm_args(A, sA, B, sB, D, M_total, N, K);
    if (st != NVFP4_OK) return st;
    if (M_total == 0 || N == 0) return NVFP4_OK;
    if (!alpha || !row_offsets || !aligned(alpha, 4) || !aligned(row_offsets, 4)) return NVFP4_ERR_INVALID_ARG;
    // The grouped kernel loads row-major scale tiles with TMA.
    if (K % 256 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(sA, 16) || !aligned(sB, 16)) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    using GC = nvfp4::GroupedConfig;
    CUtensorMap tmB, tmA, tmSB, tmSA;
    const long long b_rows = (long long)G * N;
    if (!make_operand_map(&tmB, B, b_rows, K / 2, 128) || !make_operand_map(&tmA, A, M_total, K / 2, 16) ||
        !make_scale_map(&tmSB, sB, b_rows, K / 16, 128) || !make_scale_map(&tmSA, sA, M_total, K / 16, 16))
        return NVFP4_ERR_CUDA;
    nvfp4::GroupedParams prm{};
    prm.alpha = alpha;
    prm.offsets = row_offsets;
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.G = G;
    prm.N = N;
    prm.K = K;
    prm.M_total = M_total;
    prm.tiles_n = (N + 127) / 128;
    prm.k_tiles = K / 256;
    if ((st = get_unit_counter(dev, stream, &prm.counter)) != NVFP4_OK) return st;
    auto kern = nvfp4::nvfp4_grouped_kernel;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(info->smem_attr_set & (1ull << 63))) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GC::SMEM_BYTES) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            info->smem_attr_set |= (1ull << 63);
        }
    }
    const long long units = (long long)G * prm.tiles_n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<long long>(units, info->num_sms), 1, 1);
    cfg.blockDim = dim3(nvfp4::kGroupedThreads, 1, 1);
    cfg.dynamicSmemBytes = GC::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmB, tmA, tmSB, tmSA, prm);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

nvfp4_status nvfp4_get_device_error(void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, nvfp4::g_error_word, sizeof(v)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(nvfp4::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    return (v & nvfp4::kErrTimeout) ? NVFP4_ERR_TIMEOUT : NVFP4_OK;
}

nvfp4_status nvfp4_debug_wait_timeout(uint64_t timeout_ns, void* stream_) {
    if (timeout_ns < 1000ull || timeout_ns > 5000000000ull) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    nvfp4::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_)>>>(timeout_ns);
    g_launches++;
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_quantize_scaled(const void* X, int x_is_bf16, int rows, int K, float g, void* codes,
                                   void* scales, void* stream_) {
    if (rows < 0 || K <= 0 || (x_is_bf16 != 0 && x_is_bf16 != 1)) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!(g > 0.0f) || !std::isfinite(g)) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0) return NVFP4_OK;
    if (!X || !codes || !scales || !aligned(X, 16) || !aligned(codes, 8)) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    const long long nb = (long long)rows * (K / 16);
    const int threads = 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((nb + threads - 1) / threads), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream_);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e =
        x_is_bf16 ? cudaLaunchKernelEx(&cfg, nvfp4::quantize_scaled_kernel<true>, X, nb, g, static_cast<uint8_t*>(codes),
                                       static_cast<uint8_t*>(scales))
                  : cudaLaunchKernelEx(&cfg, nvfp4::quantize_scaled_kernel<false>, X, nb, g,
                                       static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

nvfp4_status nvfp4_gemm_bf16a(const void* A, float gA, const void* B, const void* sB, float alpha, void* D, int M,
                              int N, int K, void* stream_) {
    if (M < 0 || N < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!(gA > 0.0f) || !std::isfinite(gA)) return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!A || !B || !sB || !D || !aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sB, 4))
        return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool sfr = (K % 256 == 0) && aligned(sB, 16);
    const Plan plan = make_plan(M, N, K, info, sfr);
    // The GEMM can quantize its activation tiles itself, but every CTA of a
    // weight-tile column then repeats the same conversion (IEEE divisions on
    // the critical path): measured 13.8 against 7.4 us per 768x6144 layer at
    // M = 1 in a dependent chain.  So the separate one-launch quantizer,
    // spread over all SMs and overlapped by programmatic dependent launch, is
    // the default; NVFP4_GEMM_FUSE_QUANT=1 selects the in-kernel form, for
    // the tensor-core shapes (token rows that the CUDA-core kernel takes are
    // always quantized first).
    const char* fuse_env = std::getenv("NVFP4_GEMM_FUSE_QUANT");
    const bool fuse = fuse_env && fuse_env[0] == '1' && !use_gemv(M, N, K);
    if (fuse && sfr && plan.swap && (plan.bq == 16 || plan.bq == 32)) {
        // Fused: the GEMM quantizes its activation tiles in shared memory.
        Maps maps;
        if (!make_operand_map(&maps.p, B, N, K / 2, 128) || !make_bf16_map(&maps.q, A, M, K, plan.bq) ||
            !make_scale_map(&maps.sp, sB, N, K / 16, 128))
            return NVFP4_ERR_CUDA;
        maps.sq = maps.sp;   // unused: the Q scales are computed in the kernel
        GemmParams prm{};
        prm.D = static_cast<__nv_bfloat16*>(D);
        prm.alpha = alpha;
        prm.rows_p = N;
        prm.rows_q = M;
        prm.K = K;
        prm.ldd = N;
        prm.k_tiles = plan.k_tiles;
        prm.tiles_q = plan.tiles_q;
        prm.gq = gA;
        if ((st = splitk_ws(dev, stream, plan, nullptr, 0, &prm.ws)) != NVFP4_OK) return st;
        const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
        const int sk = plan.splits > 1 ? 1 : 0;
        if (plan.bq == 16)
            return sk ? launch_gemm_kernel<16, true, true, true, true>(info, 1ull << 40, maps, prm, grid, stream)
                      : launch_gemm_kernel<16, true, false, true, true>(info, 1ull << 41, maps, prm, grid, stream);
        return sk ? launch_gemm_kernel<32, true, true, true, true>(info, 1ull << 42, maps, prm, grid, stream)
                  : launch_gemm_kernel<32, true, false, true, true>(info, 1ull << 43, maps, prm, grid, stream);
    }
    // Quantize into per-stream scratch, then the GEMM (two launches, chained
    // by programmatic dependent launch).
    const size_t codes_bytes = (size_t)M * (K / 2), off_s = align_up(codes_bytes, 256);
    uint8_t* ws = nullptr;
    if ((st = get_scratch(dev, stream, off_s + (size_t)M * (K / 16), &ws, kScratchAct)) != NVFP4_OK) return st;
    if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((st = nvfp4_quantize_scaled(A, 1, M, K, gA, ws, ws + off_s, stream_)) != NVFP4_OK) return st;
    return nvfp4_gemm(ws, ws + off_s, B, sB, alpha, D, M, N, K, stream_);
}

nvfp4_status nvfp4_fp4_peak_probe(int pair, long long steps, int* ctas_out, void* stream_) {
    if ((pair != 0 && pair != 1) || steps < 1 || steps > 100000000ll || !ctas_out) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    auto kern = pair ? nvfp4::fp4_peak_kernel<true> : nvfp4::fp4_peak_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, nvfp4::kPeakSmem) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(nvfp4::kPeakThreads, 1, 1);
    cfg.dynamicSmemBytes = nvfp4::kPeakSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    int ctas = info->num_sms;
    if (pair) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(2, 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        ctas = 2 * std::min(n, info->num_sms / 2);
    }
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, steps);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    *ctas_out = ctas;
    return NVFP4_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// 2:4-sparse weights (nvfp4_gemm_sparse24).
// ---------------------------------------------------------------------------
extern "C" nvfp4_status nvfp4_gemm_sparse24(const void* A, const void* sA, const void* Bv, const void* Bm,
                                            const void* sB, float alpha, void* D, int M, int N, int K,
                                            unsigned flags, void* stream_) {
    if (flags & ~NVFP4_GEMM_B_CONSTANT) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!A || !sA || !Bv || !Bm || !sB || !D) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(Bv, 16) || !aligned(D, 16) || !aligned(sA, 4) || !aligned(sB, 4) ||
        !aligned(Bm, 4))
        return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (M <= sp24_gemv_max_m()) {
        nvfp4::GemvSp24Params prm{};
        prm.A = static_cast<const uint8_t*>(A);
        prm.sA = static_cast<const uint8_t*>(sA);
        prm.Bv = static_cast<const uint8_t*>(Bv);
        prm.Bm = static_cast<const uint8_t*>(Bm);
        prm.sB = static_cast<const uint8_t*>(sB);
        prm.D = static_cast<__nv_bfloat16*>(D);
        prm.alpha = alpha;
        prm.M = M;
        prm.N = N;
        prm.K = K;
        prm.prefetch_b = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
        int rw = M == 1 ? (N >= 2048 ? 4 : 1) : 2;
        const bool areg = use_gemv_areg(M, K);
        if (areg) rw = N >= 4096 ? 4 : (M == 1 ? (N >= 2048 ? 2 : 1) : (N <= 256 ? 1 : 2));
        if (const char* e = std::getenv("NVFP4_GEMM_GEMV_RW")) {
            const int v = std::atoi(e);
            if (v == 1 || v == 2 || v == 4) rw = v;
        }
        if (areg) return gemv_sp24_areg_gemm(info, rw, prm, stream);
        if (M <= 1) return launch_gemv_sp24_rw<1>(info, rw, prm, stream);
        if (M <= 2) return launch_gemv_sp24_rw<2>(info, rw, prm, stream);
        if (M <= 4) return launch_gemv_sp24_rw<4>(info, rw, prm, stream);
        if (M <= 8) return launch_gemv_sp24_rw<8>(info, rw, prm, stream);
        return launch_gemv_sp24_rw<16>(info, rw, prm, stream);
    }
    // Dense codes in the operand scratch (ordered on the stream before the
    // GEMM that reads them; the GEMM gets no constant-B flag, since its B is
    // written right before it).
    const size_t dense_bytes = (size_t)N * (size_t)(K / 2);
    uint8_t* dense = nullptr;
    if ((st = get_scratch(dev, stream, dense_bytes, &dense, kScratchAct)) != NVFP4_OK) return st;
    const long long items = (long long)N * (K / 16);
    const int threads = 256;
    const int blocks = (int)std::min<long long>((items + threads - 1) / threads, (long long)info->num_sms * 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max(blocks, 1), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, nvfp4::sparse24_expand_kernel, static_cast<const uint8_t*>(Bv),
                                             static_cast<const uint8_t*>(Bm), items, dense);
    g_launches++;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return nvfp4_gemm_ex(A, sA, dense, sB, alpha, D, M, N, K, 0u, stream_);
}

// ---------------------------------------------------------------------------
// GEMM without any device allocation (nvfp4_gemm_noalloc).
//
// For callers that may not allocate device memory at call time: hosts that
// own every byte of device memory themselves (a serving runtime with its own
// pool, a plugin inside another framework), code with a fixed memory budget,
// or callers that must not trigger a driver allocation on the launch path.
// nvfp4_gemm may cudaMalloc per-stream scratch on its first call of a shape;
// this variant never does.  Its only scratch -- the scales re-laid out for
// the tensor cores -- lives in the file-scope device array below, which every
// GPU that loads this library holds for the life of the process.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
std::map<int, uint8_t*> g_noalloc_addr;   // device -> device address of g_noalloc_scratch

// The array's name in host code is only a host-side handle; the device
// address has to be looked up, once per device, with that device current.
nvfp4_status noalloc_scratch_address(int dev, uint8_t** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_addr.find(dev);
    if (it == g_noalloc_addr.end()) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        it = g_noalloc_addr.emplace(dev, static_cast<uint8_t*>(p)).first;
    }
    *out = it->second;
    return NVFP4_OK;
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm_noalloc(const void* A, const void* sA, const void* B, const void* sB, float alpha, void* D,
                                int M, int N, int K, void* stream_) {
    nvfp4_status st = check_gemm_args(A, sA, B, sB, D, M, N, K);
    if (st != NVFP4_OK || M == 0 || N == 0) return st;
    int dev;
    DeviceInfo* info;
    if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // A few token rows: the CUDA-core kernel, which uses no scratch at all.
    if (use_gemv(M, N, K)) return gemv_gemm(info, A, sA, B, sB, alpha, D, M, N, K, 0u, stream);
    // Row-major scales that TMA can load (K % 256 == 0, 16-byte aligned): the
    // tensor-core kernels lay them out on chip; the static scratch holds at
    // most the split-K partials (or the plan runs without a K split).  The
    // CTA-pair kernel, which needs its scales re-laid out first, is not used;
    // its shapes run on the single-CTA persistent kernel.
    const bool sfr = (K % 256 == 0) && aligned(sA, 16) && aligned(sB, 16);
    uint8_t* scratch = nullptr;
    if (sfr) {
        if ((st = noalloc_scratch_address(dev, &scratch)) != NVFP4_OK) return st;
        return sfr_gemm(dev, info, make_plan(M, N, K, info, true), A, sA, B, sB, alpha, D, M, N, K, 0u, stream,
                        scratch, kNoAllocScratchBytes);
    }
    // Otherwise the scales of both operands are re-laid out into the static
    // scratch, which they must fit (the split-K partials follow them there,
    // or the plan runs without a K split).
    const size_t sfa_bytes = nvfp4_swizzled_scale_bytes(M, K);
    const size_t sfb_bytes = nvfp4_swizzled_scale_bytes(N, K);
    if (align_up(sfa_bytes, 256) + sfb_bytes > kNoAllocScratchBytes) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((st = noalloc_scratch_address(dev, &scratch)) != NVFP4_OK) return st;

    Plan plan = make_plan(M, N, K, info, /*sfr=*/false);
    const size_t ws_off = align_up(align_up(sfa_bytes, 256) + sfb_bytes, 256);
    if (ws_off + splitk_ws_bytes(plan) > kNoAllocScratchBytes) plan = make_plan(M, N, K, info, false, 1);
    const void* P = plan.swap ? B : A;
    const void* Q = plan.swap ? A : B;
    const void* sP = plan.swap ? sB : sA;
    const void* sQ = plan.swap ? sA : sB;
    const int rows_p = plan.swap ? N : M;
    const int rows_q = plan.swap ? M : N;
    uint8_t* sfp = scratch;
    uint8_t* sfq = scratch + align_up(nvfp4_swizzled_scale_bytes(rows_p, K), 256);
    // Every byte the kernel reads is rewritten by these two passes (padding
    // rows included), so nothing left by an earlier call needs clearing.
    if ((st = launch_swizzle(sP, rows_p, K, sfp, stream)) != NVFP4_OK) return st;
    if ((st = launch_swizzle(sQ, rows_q, K, sfq, stream)) != NVFP4_OK) return st;

    Maps maps;
    if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq))
        return NVFP4_ERR_CUDA;
    maps.sp = maps.p;
    maps.sq = maps.q;
    GemmParams prm{};
    prm.sfp = sfp;
    prm.sfq = sfq;
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.rows_p = rows_p;
    prm.rows_q = rows_q;
    prm.K = K;
    prm.ldd = N;
    prm.k_tiles = plan.k_tiles;
    prm.tiles_q = plan.tiles_q;
    prm.prefetch_b = 0;
    if ((st = splitk_ws(dev, stream, plan, scratch + ws_off, kNoAllocScratchBytes - ws_off, &prm.ws)) != NVFP4_OK)
        return st;
    const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
    return launch_mode<false>(plan, info, maps, prm, grid, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// MXFP4 GEMM (nvfp4_gemm_mxfp4).
// ---------------------------------------------------------------------------
extern "C" nvfp4_status nvfp4_gemm_mxfp4(const void* A, const void* sA, const void* B, const void* sB, float alpha,
                                         void* D, int M, int N, int K, unsigned flags, void* stream_) {
    if (flags & ~NVFP4_GEMM_B_CONSTANT) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!A || !sA || !B || !sB || !D) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16)) return NVFP4_ERR_INVALID_ARG;
    int dev;
    DeviceInfo* info;
    nvfp4_status st = current_device(&dev, &info);
    if (st != NVFP4_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // One to four token rows: the CUDA-core kernel (NVFP4_GEMM_GEMV sets the
    // row limit here too, 0 turning it off).
    int gemv_rows = 4;
    if (const char* e = std::getenv("NVFP4_GEMM_GEMV")) gemv_rows = std::min(4, std::max(0, std::atoi(e)));
    if (M <= gemv_rows) {
        nvfp4::GemvMxParams prm{};
        prm.A = static_cast<const uint8_t*>(A);
        prm.sA = static_cast<const uint8_t*>(sA);
        prm.B = static_cast<const uint8_t*>(B);
        prm.sB = static_cast<const uint8_t*>(sB);
        prm.D = static_cast<__nv_bfloat16*>(D);
        prm.alpha = alpha;
        prm.M = M;
        prm.N = N;
        prm.K = K;
        prm.prefetch_b = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
        if (use_gemv_areg(M, K)) {
            int rw = N >= 4096 ? 4 : (M == 1 ? (N >= 2048 ? 2 : 1) : (N <= 256 ? 1 : 2));
            if (const char* e = std::getenv("NVFP4_GEMM_GEMV_RW")) {
                const int v = std::atoi(e);
                if (v == 1 || v == 2 || v == 4) rw = v;
            }
            const int cpt = (K / 32 + nvfp4::kGemvThreads - 1) / nvfp4::kGemvThreads;
            if (M == 1) {
                if (cpt <= 1) return launch_gemv_mx_areg_rw<1, 1>(info, rw, prm, stream);
                if (cpt <= 2) return launch_gemv_mx_areg_rw<1, 2>(info, rw, prm, stream);
                return launch_gemv_mx_areg_rw<1, 4>(info, rw, prm, stream);
            }
            if (cpt <= 1) return launch_gemv_mx_areg_rw<2, 1>(info, rw, prm, stream);
            return launch_gemv_mx_areg_rw<2, 2>(info, rw, prm, stream);
        }
        const int rw = M == 1 ? (N >= 2048 ? 4 : 1) : 2;
        if (M == 1) return rw == 4 ? launch_gemv_mx_kernel<1, 4>(info, prm, stream) : launch_gemv_mx_kernel<1, 1>(info, prm, stream);
        if (M == 2) return launch_gemv_mx_kernel<2, 2>(info, prm, stream);
        return launch_gemv_mx_kernel<4, 2>(info, prm, stream);
    }
    // The tensor cores.  Row-major scales that TMA can load (K % 512 == 0, so
    // that a row of K/32 scale bytes is a multiple of 16; 16-byte aligned):
    // the tiled kernel lays them out on chip, as for NVFP4.  Otherwise both
    // operands' scales are first re-laid out into atoms in per-stream scratch.
    const bool sfr = (K % 512 == 0) && aligned(sA, 16) && aligned(sB, 16) && !std::getenv("NVFP4_GEMM_MX_ATOMS");
    if (sfr) {
        const Plan plan = make_plan(M, N, K, info, /*sfr=*/true);
        const void* P = plan.swap ? B : A;
        const void* Q = plan.swap ? A : B;
        const void* sP = plan.swap ? sB : sA;
        const void* sQ = plan.swap ? sA : sB;
        const int rows_p = plan.swap ? N : M;
        const int rows_q = plan.swap ? M : N;
        Maps maps;
        if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq) ||
            !make_scale_map(&maps.sp, sP, rows_p, K / 32, 128) || !make_scale_map(&maps.sq, sQ, rows_q, K / 32, plan.bq))
            return NVFP4_ERR_CUDA;
        GemmParams prm{};
        prm.D = static_cast<__nv_bfloat16*>(D);
        prm.alpha = alpha;
        prm.rows_p = rows_p;
        prm.rows_q = rows_q;
        prm.K = K;
        prm.ldd = N;
        prm.k_tiles = plan.k_tiles;
        prm.tiles_q = plan.tiles_q;
        prm.prefetch_b = (flags & NVFP4_GEMM_B_CONSTANT) ? 1 : 0;
        if ((st = splitk_ws(dev, stream, plan, nullptr, 0, &prm.ws)) != NVFP4_OK) return st;
        const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
        if (plan.swap)
            return plan.splits > 1 ? launch_mx_sfr_by_bq<true, true>(plan.bq, info, maps, prm, grid, stream)
                                   : launch_mx_sfr_by_bq<true, false>(plan.bq, info, maps, prm, grid, stream);
        return plan.splits > 1 ? launch_mx_sfr_by_bq<false, true>(plan.bq, info, maps, prm, grid, stream)
                               : launch_mx_sfr_by_bq<false, false>(plan.bq, info, maps, prm, grid, stream);
    }
    const Plan plan = make_plan(M, N, K, info, /*sfr=*/false);
    const void* P = plan.swap ? B : A;
    const void* Q = plan.swap ? A : B;
    const void* sP = plan.swap ? sB : sA;
    const void* sQ = plan.swap ? sA : sB;
    const int rows_p = plan.swap ? N : M;
    const int rows_q = plan.swap ? M : N;
    const size_t off_sfq = align_up(mx_atom_bytes(rows_p, K), 256);
    uint8_t* ws = nullptr;
    if ((st = get_scratch(dev, stream, off_sfq + mx_atom_bytes(rows_q, K), &ws)) != NVFP4_OK) return st;
    Maps maps;
    if (!make_operand_map(&maps.p, P, rows_p, K / 2, 128) || !make_operand_map(&maps.q, Q, rows_q, K / 2, plan.bq))
        return NVFP4_ERR_CUDA;
    if ((st = launch_swizzle_mx(sP, rows_p, K, ws, stream)) != NVFP4_OK) return st;
    if ((st = launch_swizzle_mx(sQ, rows_q, K, ws + off_sfq, stream)) != NVFP4_OK) return st;
    maps.sp = maps.p;
    maps.sq = maps.q;
    GemmParams prm{};
    prm.sfp = ws;
    prm.sfq = ws + off_sfq;
    prm.D = static_cast<__nv_bfloat16*>(D);
    prm.alpha = alpha;
    prm.rows_p = rows_p;
    prm.rows_q = rows_q;
    prm.K = K;
    prm.ldd = N;
    prm.k_tiles = plan.k_tiles;
    prm.tiles_q = plan.tiles_q;
    if ((st = splitk_ws(dev, stream, plan, nullptr, 0, &prm.ws)) != NVFP4_OK) return st;
    const dim3 grid(plan.splits, plan.tiles_q * plan.tiles_p, 1);
    if (plan.swap)
        return plan.splits > 1 ? launch_mx_by_bq<true, true>(plan.bq, info, maps, prm, grid, stream)
                               : launch_mx_by_bq<true, false>(plan.bq, info, maps, prm, grid, stream);
    return plan.splits > 1 ? launch_mx_by_bq<false, true>(plan.bq, info, maps, prm, grid, stream)
                           : launch_mx_by_bq<false, false>(plan.bq, info, maps, prm, grid, stream);
}
