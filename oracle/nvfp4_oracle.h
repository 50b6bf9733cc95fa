/*
 * CPU oracle for the NVFP4 block-scaled GEMM.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * call it.  The product path never includes, links or executes anything in
 * this directory, and this directory shares no code with the CUDA library.
 *
 * What it computes (all citations are to the three source pages):
 *   - NVFP4 data: 4-bit E2M1 values packed two per byte, with a scale factor
 *     per block of values ("The SM120 FP4 Kernel Disaster", section "Input
 *     Knowledge Required", item 3).
 *   - One FP8 (E4M3) block scale per 16 elements along K, BF16 output; the
 *     byte model M*K/2 + K*N/2 + M*K/16 + K*N/16 + 2*M*N ("Peeling the Kernel
 *     Onion", section "The Benchmark Design").
 *   - A global fp32 scale alpha applied to the output ("Peeling the Kernel
 *     Onion", section "The Chain of Reasoning": the kernel needs alpha).
 *
 *   D[m][n] = bf16_rne( alpha * sum_k e2m1(A[m,k]) * e4m3(sA[m,k/16])
 *                                  * e2m1(B[n,k]) * e4m3(sB[n,k/16]) )
 *
 * The sum is formed exactly (128-bit integer fixed point in units of 2^-20,
 * cross-checked against fp64), alpha is applied exactly, and the result is
 * rounded once to BF16 with round-to-nearest-even.
 *
 * Parity status of every function is stated beside it; all are pinned by the
 * not-gpu tests (format tables, closed forms, brute force, invariants).
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Format tables. */
double oracle_e2m1_value(int code);          /* code 0..15, bit 3 = sign            */
double oracle_e4m3_value(int byte);          /* 0..255; NaN for 0x7F and 0xFF       */
int    oracle_e4m3_rne_satfinite(float v);   /* nearest E4M3, ties to even, |v|>448 -> 448 */
int    oracle_e2m1_rne_satfinite(float v);   /* nearest E2M1, ties to even, |v|>6 -> 6     */

/* Quantize fp32 X[rows][K] to packed codes [rows][K/2], scales [rows][K/16]
 * and one global scale g for the whole tensor.  Returns 0 on success, -1 on a
 * bad argument (K not a multiple of 16, NaN/Inf input). */
int oracle_quantize(const float* X, int rows, int K,
                    uint8_t* codes, uint8_t* scales, float* g_out);

/* The same block steps with the global scale g given by the caller (a scale
 * fixed in advance for a tensor, instead of one computed from its amax): the
 * configs' recipe after its first step.  Block scales that would exceed 448
 * saturate, and so do codes beyond 6.  Returns -1 for g not positive and
 * finite or a NaN/Inf input. */
int oracle_quantize_with_scale(const float* X, int rows, int K, float g,
                               uint8_t* codes, uint8_t* scales);

/* Exact value of one output: sets *exact (double rounding of the exact
 * value), *absdot = |alpha| * sum_k |a_k b_k| (fp64) and returns the BF16 bits
 * of the single RNE rounding of the exact value. */
uint16_t oracle_dot(const uint8_t* a_row, const uint8_t* sa_row,
                    const uint8_t* b_row, const uint8_t* sb_row,
                    int K, float alpha, double* exact, double* absdot);

/* Full GEMM.  A [M][K/2], sA [M][K/16], B [N][K/2], sB [N][K/16], all
 * row-major bytes.  D_bf16 [M][N] (may be NULL), ref [M][N] and absdot [M][N]
 * (either may be NULL).  Returns 0, or -1 on bad arguments. */
int oracle_gemm(const uint8_t* A, const uint8_t* sA,
                const uint8_t* B, const uint8_t* sB,
                float alpha, int M, int N, int K,
                uint16_t* D_bf16, double* ref, double* absdot);

/* Only the listed outputs (rows[i], cols[i]), i < count. */
int oracle_gemm_sampled(const uint8_t* A, const uint8_t* sA,
                        const uint8_t* B, const uint8_t* sB,
                        float alpha, int M, int N, int K,
                        const int32_t* rows, const int32_t* cols, int count,
                        uint16_t* D_bf16, double* ref, double* absdot);

/* Grouped GEMM: rows [off[g], off[g+1]) of A use B[g], sB[g] and alpha[g].
 * B [G][N][K/2], sB [G][N][K/16]. */
int oracle_grouped_gemm(const uint8_t* A, const uint8_t* sA,
                        const uint8_t* B, const uint8_t* sB,
                        const float* alpha, const int32_t* row_offsets, int G,
                        int M_total, int N, int K,
                        uint16_t* D_bf16, double* ref, double* absdot);

/* BF16 RNE of the exact value alpha * S * 2^-20 (S a signed 128-bit integer
 * given as hi:lo words).  Exposed for the rounding pins. */
uint16_t oracle_bf16_of_scaled(int64_t s_hi, uint64_t s_lo, float alpha);

/* Tensor-core scale-factor layout: row-major [rows][K/16] -> 512-byte atoms
 * of 128 rows x 4 scale blocks, atoms ordered K-fastest within each 128-row
 * block; padding rows are zero.  Writes oracle_swizzled_bytes() bytes. */
long oracle_swizzled_bytes(int rows, int K);
int  oracle_swizzle_scales(const uint8_t* s_rowmajor, int rows, int K, uint8_t* out);

/* 2:4 structured sparsity over packed bytes.  The pages name FP4 structured
 * sparsity as a way to cut what small-batch decode demands ("Peeling the
 * Kernel Onion", sections "Assumptions Embedded in the Benchmark" and
 * "Knowledge Created and Its Impact") and give no layout; the reading here:
 * in every group of 4 consecutive packed bytes of a row (8 values along K,
 * the bytes being pairs of E2M1 values 2p, 2p+1) at most 2 bytes are
 * non-zero.  A row of K values is stored as
 *   values [K/4]:  the 2 kept bytes of each group, lower position first;
 *   meta   [K/16]: per group a nibble p0 | p1 << 2 (positions 0..3, p0 < p1),
 *                  the even group in the low nibble of each byte;
 *   scales [K/16]: the dense E4M3 block scales, one per 16 values.
 * A group with fewer than 2 non-zero bytes keeps its non-zero byte (if any)
 * and the lowest zero bytes.  K must be a multiple of 16.
 *
 * compress returns -1 when a group has more than 2 non-zero bytes;
 * decompress writes dense codes [rows][K/2] (dropped bytes 0x00) and returns
 * -1 for a position pair that is not p0 < p1.  Parity: pinned by a worked
 * layout example, round trips, and the pruning quantizer's reduction to the
 * dense quantizer (tests/test_oracle_sparse24.py). */
int oracle_sparse24_compress(const uint8_t* codes, int rows, int K, uint8_t* values, uint8_t* meta);
int oracle_sparse24_decompress(const uint8_t* values, const uint8_t* meta, int rows, int K, uint8_t* codes);

/* Prune fp32 X[rows][K] to the pattern above -- in each group of 4 value
 * pairs keep the 2 pairs with the largest max(|x_2p|, |x_2p+1|), ties to the
 * lower position -- and quantize the pruned tensor like oracle_quantize.
 * Every group keeps its largest value, so block scales and g equal those of
 * the unpruned tensor and kept codes equal its dense codes. */
int oracle_quantize_sparse24(const float* X, int rows, int K,
                             uint8_t* values, uint8_t* meta, uint8_t* scales, float* g_out);

/* D = A (dense) times the 2:4-sparse B (values, meta, scales) transposed:
 * by definition the dense GEMM of A and the decompressed B. */
int oracle_gemm_sparse24(const uint8_t* A, const uint8_t* sA,
                         const uint8_t* Bv, const uint8_t* Bm, const uint8_t* sB,
                         float alpha, int M, int N, int K,
                         uint16_t* D_bf16, double* ref, double* absdot);

/* MXFP4 (the other block-scaled FP4 format of the same tensor-core
 * instruction family; the pages do not use it): E2M1 values with one E8M0
 * scale -- a power of two 2^(byte - 127), byte 255 NaN -- per 32 values
 * along K, scales [rows][K/32].
 *   oracle_quantize_mxfp4: per block X = 2^(floor(log2 amax) - 2), clamped to
 *   2^-127 .. 2^127; codes E2M1(x / X) nearest even, saturating at 6, zero
 *   codes keep the sign of x; an all-zero block gets scale byte 0 and zero
 *   codes.  -1 for K % 32 != 0 or a non-finite input.
 *   oracle_gemm_mxfp4: D = bf16_rne(alpha * sum_k e2m1(A) 2^(sA-127)
 *   e2m1(B) 2^(sB-127)), the sum exact in a 768-bit integer (products span
 *   2^-256 .. 2^256), alpha applied exactly, one rounding; ref and absdot as
 *   for oracle_gemm.  -1 for a NaN scale (255), K % 32 != 0 or a non-finite
 *   alpha.
 * Parity: pinned by the E8M0 closed form, hand-worked quantizer blocks, brute
 * force with exact rationals, and the reduction to oracle_gemm when every
 * scale is 1 (tests/test_oracle_mxfp4.py). */
double oracle_e8m0_value(int byte);
int oracle_quantize_mxfp4(const float* X, int rows, int K, uint8_t* codes, uint8_t* scales);
int oracle_gemm_mxfp4(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB,
                      float alpha, int M, int N, int K, uint16_t* D_bf16, double* ref, double* absdot);

#ifdef __cplusplus
}
#endif
#endif
