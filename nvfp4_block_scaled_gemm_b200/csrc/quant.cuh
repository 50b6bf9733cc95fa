// The block steps of quantize-and-pack, shared by the quantize kernels and
// the GEMM that quantizes its BF16 activations on the fly: one E4M3 scale per
// 16 values, s = E4M3(amax_blk / (6 g)), codes = E2M1(x / (g * s)), both
// round-to-nearest-even with saturation, fp32 IEEE division and products
// ("The SM120 FP4 Kernel Disaster", section "Input Knowledge Required",
// item 3: two 4-bit values per byte with per-block scale factors).
#pragma once

#include <cstdint>

namespace nvfp4 {

__device__ __forceinline__ float global_scale_from_amax(float amax) {
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);   // 6 * 448
}

// Non-negative float -> E4M3, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_from_float(float t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xFFu;
}

// E4M3 byte (sign bit clear) -> its exact float value.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
    if (e == 0) return (float)m * 0.001953125f;                 // m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));     // (1 + m/8) 2^(e-7)
}

// Eight fp32 values -> eight E2M1 codes (RNE, saturating at 6), element 2i in
// the low nibble of byte i.  A code whose magnitude rounds to zero carries the
// sign of its input.
__device__ __forceinline__ uint32_t e2m1x8_from_float(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t nib = (r >> (4 * i)) & 0xFu;
        const uint32_t fixed = (nib & 7u) ? nib : (__float_as_uint(v[i]) >> 31) << 3;
        r = (r & ~(0xFu << (4 * i))) | (fixed << (4 * i));
    }
    return r;
}

// One 16-value block with the global scale g (six_g = 6 * g, rounded): the
// scale byte and the eight code bytes (element 2i in the low nibble of byte i).
__device__ __forceinline__ void quantize_block16(const float (&x)[16], float g, float six_g, uint32_t& scale,
                                                 uint32_t (&codes)[2]) {
    float amax_blk = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax_blk = fmaxf(amax_blk, fabsf(x[i]));
    scale = e4m3_from_float(__fdiv_rn(amax_blk, six_g));
    const float denom = __fmul_rn(g, e4m3_to_float(scale));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = denom == 0.0f ? x[8 * h + i] * 0.0f : __fdiv_rn(x[8 * h + i], denom);
        codes[h] = e2m1x8_from_float(v);
    }
}

}  // namespace nvfp4
