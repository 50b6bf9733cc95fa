/*
 * CPU oracle for the NVFP4 block-scaled GEMM -- plain, slow, obviously
 * correct.  TEST INFRASTRUCTURE ONLY (see nvfp4_oracle.h): the CUDA library
 * never includes or links this file, and this file includes nothing of it.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction and IEEE float semantics are part of the quantizer's
 * definition, since its integer codes are compared bit for bit).
 *
 * Sources (the three pages):
 *   [P1] "The SM120 FP4 Kernel Disaster", section "Input Knowledge Required",
 *        item 3: FP4 packs two 4-bit values per byte, with per-block scales.
 *   [P3] "Peeling the Kernel Onion", section "The Benchmark Design": FP8 scale
 *        factors one per 16 elements, BF16 output, bytes
 *        M*K/2 + K*N/2 + M*K/16 + K*N/16 + 2*M*N.
 *   [P3c] "Peeling the Kernel Onion", section "The Chain of Reasoning": the
 *        FP4 GEMM takes a global alpha and writes an out tensor.
 * The element format (E2M1: 1 sign, 2 exponent, 1 mantissa bit, values
 * {0,0.5,1,1.5,2,3,4,6}) and the scale format (E4M3: bias 7, no infinities,
 * NaN at S.1111.111) are the standard NVFP4 definitions these pages use.
 */
#include "nvfp4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef __int128 i128;
typedef unsigned __int128 u128;

/* ------------------------------------------------------------------------ */
/* Format tables                                                            */
/* ------------------------------------------------------------------------ */

/* E2M1 magnitudes, code bits 2..0 (exponent bits 2..1, mantissa bit 0). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code) {
    code &= 0xF;
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 (bias 7): exponent field e = bits 6..3, mantissa m = bits 2..0.
 * e == 0: subnormal m * 2^-9;  otherwise (1 + m/8) * 2^(e-7);
 * e == 15 && m == 7: NaN.  No infinities. */
double oracle_e4m3_value(int byte) {
    byte &= 0xFF;
    int s = byte >> 7, e = (byte >> 3) & 0xF, m = byte & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Integer forms used by the exact accumulation.
 * e2m1 magnitude in units of 1/2; e4m3 magnitude in units of 2^-9. */
static int e2m1_half_units(int code) { return (int)(E2M1_MAG[code & 7] * 2.0); }
static int e4m3_units(int byte) { return (int)ldexp(fabs(oracle_e4m3_value(byte)), 9); }

/* Round-to-nearest, ties to the even code, over a monotone table of
 * non-negative values val[0..n-1]; values at or above val[n-1] saturate to
 * code n-1 (the "satfinite" behaviour). */
static int round_nearest_even(double v, const double* val, int n) {
    if (v >= val[n - 1]) return n - 1;
    int c = 0;
    while (c + 1 < n && val[c + 1] <= v) c++;      /* val[c] <= v < val[c+1] */
    double mid = (val[c] + val[c + 1]) * 0.5;       /* exact: few significant bits */
    if (v < mid) return c;
    if (v > mid) return c + 1;
    return (c & 1) ? c + 1 : c;                     /* tie: even code */
}

static double E4M3_POS[127];   /* codes 0x00..0x7E */
static int e4m3_pos_ready = 0;
static void init_e4m3_pos(void) {
    if (e4m3_pos_ready) return;
    for (int c = 0; c < 127; c++) E4M3_POS[c] = oracle_e4m3_value(c);
    e4m3_pos_ready = 1;
}

int oracle_e4m3_rne_satfinite(float v) {
    init_e4m3_pos();
    if (isnan(v)) return 0x7F;
    int sign = signbit(v) ? 0x80 : 0;
    return sign | round_nearest_even(fabs((double)v), E4M3_POS, 127);
}

int oracle_e2m1_rne_satfinite(float v) {
    if (isnan(v)) return -1;
    int sign = signbit(v) ? 8 : 0;
    return sign | round_nearest_even(fabs((double)v), E2M1_MAG, 8);
}

/* ------------------------------------------------------------------------ */
/* Quantize-and-pack                                                        */
/* ------------------------------------------------------------------------ */

/* Per tensor: g = amax / (6 * 448).  Per 16-element K block:
 * s = E4M3_rne_satfinite(amax_blk / (6 * g)); each element
 * q = E2M1_rne_satfinite(x / (g * decode(s))), packed two per byte with the
 * even-k element in the low nibble.  All arithmetic in IEEE fp32. */
/* The per-block steps of the quantizer for a given global scale g: block
 * scale s = E4M3(amax_blk / (6 g)), codes = E2M1(x / (g * E4M3(s))), both
 * round-to-nearest-even with saturation, fp32 IEEE arithmetic. */
static void quantize_blocks(const float* X, int rows, int K, float g_in, uint8_t* codes, uint8_t* scales) {
    volatile float g = g_in;
    volatile float six_g = 6.0f * g;
    for (int r = 0; r < rows; r++) {
        const float* x = X + (long)r * K;
        uint8_t* crow = codes + (long)r * (K / 2);
        uint8_t* srow = scales + (long)r * (K / 16);
        memset(crow, 0, (size_t)(K / 2));
        for (int b = 0; b < K / 16; b++) {
            float amax_blk = 0.0f;
            for (int i = 0; i < 16; i++) {
                float a = fabsf(x[b * 16 + i]);
                if (a > amax_blk) amax_blk = a;
            }
            volatile float t = amax_blk / six_g;
            int s = oracle_e4m3_rne_satfinite(t);
            srow[b] = (uint8_t)s;
            volatile float denom = g * (float)oracle_e4m3_value(s);
            for (int i = 0; i < 16; i++) {
                int k = b * 16 + i;
                int q;
                if (denom == 0.0f) {
                    q = signbit(x[k]) ? 8 : 0;   /* a zero scale carries zero codes */
                } else {
                    volatile float v = x[k] / denom;
                    q = oracle_e2m1_rne_satfinite(v);
                }
                crow[k / 2] |= (uint8_t)((k & 1) ? (q << 4) : q);
            }
        }
    }
}

int oracle_quantize(const float* X, int rows, int K,
                    uint8_t* codes, uint8_t* scales, float* g_out) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return -1;
    float amax = 0.0f;
    for (long i = 0; i < (long)rows * K; i++) {
        if (!isfinite(X[i])) return -1;
        float a = fabsf(X[i]);
        if (a > amax) amax = a;
    }
    /* An all-zero tensor has no scale to recover; g = 1 keeps every step finite. */
    volatile float g = (amax == 0.0f) ? 1.0f : amax / 2688.0f;
    quantize_blocks(X, rows, K, g, codes, scales);
    *g_out = g;
    return 0;
}

int oracle_quantize_with_scale(const float* X, int rows, int K, float g,
                               uint8_t* codes, uint8_t* scales) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return -1;
    if (!(g > 0.0f) || !isfinite(g)) return -1;
    for (long i = 0; i < (long)rows * K; i++)
        if (!isfinite(X[i])) return -1;
    quantize_blocks(X, rows, K, g, codes, scales);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Exact rounding of alpha * S * 2^-20 to BF16                              */
/* ------------------------------------------------------------------------ */

static int bitlen_u128(u128 x) {
    int n = 0;
    while (x) { n++; x >>= 1; }
    return n;
}

/* BF16: 8 significant bits, exponent bias 127, subnormals in steps of 2^-133. */
static uint16_t bf16_rne_of(i128 S, float alpha) {
    uint32_t ab;
    memcpy(&ab, &alpha, 4);
    int sign_a = (int)(ab >> 31), ea = (int)((ab >> 23) & 0xFF);
    uint32_t fa = ab & 0x7FFFFF;
    if (ea == 0xFF) {                       /* alpha is inf or NaN */
        if (fa || S == 0) return 0x7FC0;
        return (uint16_t)((((S < 0) ^ sign_a) << 15) | 0x7F80);
    }
    uint32_t ma = ea ? (fa | 0x800000u) : fa;
    int E = (ea ? ea - 150 : -149) - 20;    /* value = |S| * ma * 2^E */
    if (S == 0 || ma == 0) return 0x0000;   /* an exact zero is reported as +0 */
    int sign = (S < 0) ^ sign_a;
    u128 P = (u128)(S < 0 ? -S : S) * (u128)ma;
    int nb = bitlen_u128(P);
    int ev = nb - 1 + E;                    /* 2^ev <= value < 2^(ev+1) */
    int shift = (ev >= -126) ? nb - 8 : (-133 - E);
    u128 q;
    if (shift > 0) {
        q = P >> shift;
        u128 rem = P - (q << shift), half = (u128)1 << (shift - 1);
        if (rem > half || (rem == half && (q & 1))) q++;
    } else {
        q = P << (-shift);
    }
    int eq = E + shift;                     /* value ~= q * 2^eq */
    if (q == 256) { q = 128; eq += 1; }
    uint16_t bits;
    if (q >= 128) {
        int biased = eq + 7 + 127;
        if (biased >= 255) bits = 0x7F80;   /* overflow rounds to infinity */
        else bits = (uint16_t)((biased << 7) | (int)(q - 128));
    } else {
        bits = (uint16_t)q;                 /* subnormal (eq == -133) or zero */
    }
    return (uint16_t)((sign << 15) | bits);
}

uint16_t oracle_bf16_of_scaled(int64_t s_hi, uint64_t s_lo, float alpha) {
    i128 S = (i128)(((u128)(uint64_t)s_hi << 64) | (u128)s_lo);
    return bf16_rne_of(S, alpha);
}

/* ------------------------------------------------------------------------ */
/* The GEMM                                                                 */
/* ------------------------------------------------------------------------ */

static int scales_valid(const uint8_t* s, long n) {
    for (long i = 0; i < n; i++)
        if ((s[i] & 0x80) || s[i] == 0x7F) return 0;   /* unsigned, non-NaN */
    return 1;
}

/* Decode one packed row into signed integers a_k in units of 2^-10:
 * a_k = e2m1(code_k) * e4m3(scale_{k/16}); code_k is the low nibble of
 * byte k/2 for even k and the high nibble for odd k. */
static void decode_row(const uint8_t* codes, const uint8_t* scales, int K, int32_t* out) {
    for (int k = 0; k < K; k++) {
        int c = (k & 1) ? (codes[k / 2] >> 4) : (codes[k / 2] & 0xF);
        int v = e2m1_half_units(c) * e4m3_units(scales[k / 16]);
        out[k] = (c & 8) ? -v : v;
    }
}

/* Sum_k a_k b_k exactly (units 2^-20), with the fp64 sum in the same order as
 * a cross-check; returns the BF16 of alpha * sum and the fp64 views. */
static uint16_t dot_decoded(const int32_t* a, const int32_t* b, int K, float alpha,
                            double* exact, double* absdot) {
    i128 S = 0, A = 0;
    double Sd = 0.0;
    for (int k = 0; k < K; k++) {
        int64_t t = (int64_t)a[k] * (int64_t)b[k];
        S += t;
        A += (t < 0 ? -t : t);
        Sd += (double)t;
    }
    /* fp64 is exact while every partial sum stays below 2^53 units. */
    if (A < ((i128)1 << 53) && (i128)Sd != S) abort();
    if (exact) *exact = ldexp((double)S, -20) * (double)alpha;
    if (absdot) *absdot = ldexp((double)A, -20) * fabs((double)alpha);
    return bf16_rne_of(S, alpha);
}

uint16_t oracle_dot(const uint8_t* a_row, const uint8_t* sa_row,
                    const uint8_t* b_row, const uint8_t* sb_row,
                    int K, float alpha, double* exact, double* absdot) {
    int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
    int32_t* b = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
    decode_row(a_row, sa_row, K, a);
    decode_row(b_row, sb_row, K, b);
    uint16_t r = dot_decoded(a, b, K, alpha, exact, absdot);
    free(a);
    free(b);
    return r;
}

static int gemm_args_ok(int M, int N, int K) {
    return M >= 0 && N >= 0 && K > 0 && K % 16 == 0 && K <= (1 << 20);
}

int oracle_gemm(const uint8_t* A, const uint8_t* sA,
                const uint8_t* B, const uint8_t* sB,
                float alpha, int M, int N, int K,
                uint16_t* D_bf16, double* ref, double* absdot) {
    if (!gemm_args_ok(M, N, K)) return -1;
    if (!scales_valid(sA, (long)M * (K / 16)) || !scales_valid(sB, (long)N * (K / 16))) return -1;
    int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
    int32_t* bdec = (int32_t*)malloc(sizeof(int32_t) * (size_t)K * (size_t)(N > 0 ? N : 1));
    for (int n = 0; n < N; n++)
        decode_row(B + (long)n * (K / 2), sB + (long)n * (K / 16), K, bdec + (long)n * K);
    for (int m = 0; m < M; m++) {
        decode_row(A + (long)m * (K / 2), sA + (long)m * (K / 16), K, a);
        for (int n = 0; n < N; n++) {
            double e, ad;
            uint16_t d = dot_decoded(a, bdec + (long)n * K, K, alpha, &e, &ad);
            long o = (long)m * N + n;
            if (D_bf16) D_bf16[o] = d;
            if (ref) ref[o] = e;
            if (absdot) absdot[o] = ad;
        }
    }
    free(a);
    free(bdec);
    return 0;
}

int oracle_gemm_sampled(const uint8_t* A, const uint8_t* sA,
                        const uint8_t* B, const uint8_t* sB,
                        float alpha, int M, int N, int K,
                        const int32_t* rows, const int32_t* cols, int count,
                        uint16_t* D_bf16, double* ref, double* absdot) {
    if (!gemm_args_ok(M, N, K) || count < 0) return -1;
    for (int i = 0; i < count; i++) {
        int m = rows[i], n = cols[i];
        if (m < 0 || m >= M || n < 0 || n >= N) return -1;
        if (!scales_valid(sA + (long)m * (K / 16), K / 16) ||
            !scales_valid(sB + (long)n * (K / 16), K / 16)) return -1;
        double e, ad;
        uint16_t d = oracle_dot(A + (long)m * (K / 2), sA + (long)m * (K / 16),
                                B + (long)n * (K / 2), sB + (long)n * (K / 16),
                                K, alpha, &e, &ad);
        if (D_bf16) D_bf16[i] = d;
        if (ref) ref[i] = e;
        if (absdot) absdot[i] = ad;
    }
    return 0;
}

int oracle_grouped_gemm(const uint8_t* A, const uint8_t* sA,
                        const uint8_t* B, const uint8_t* sB,
                        const float* alpha, const int32_t* row_offsets, int G,
                        int M_total, int N, int K,
                        uint16_t* D_bf16, double* ref, double* absdot) {
    if (!gemm_args_ok(M_total, N, K) || G < 0) return -1;
    if (row_offsets[0] != 0 || row_offsets[G] != M_total) return -1;
    for (int g = 0; g < G; g++)
        if (row_offsets[g + 1] < row_offsets[g]) return -1;
    for (int g = 0; g < G; g++) {
        int r0 = row_offsets[g], rows = row_offsets[g + 1] - r0;
        if (rows == 0) continue;
        long o = (long)r0 * N;
        int rc = oracle_gemm(A + (long)r0 * (K / 2), sA + (long)r0 * (K / 16),
                             B + (long)g * N * (K / 2), sB + (long)g * N * (K / 16),
                             alpha[g], rows, N, K,
                             D_bf16 ? D_bf16 + o : NULL, ref ? ref + o : NULL,
                             absdot ? absdot + o : NULL);
        if (rc) return rc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Scale-factor layout for the tensor cores                                 */
/* ------------------------------------------------------------------------ */

/* One 512-byte atom holds 128 rows x 4 consecutive scale blocks (one MMA K
 * step of 64 elements): row r, block j of the atom sits at byte
 * 16*(r%32) + 4*(r/32) + j.  Atoms follow each other along K, then along
 * 128-row blocks. */
long oracle_swizzled_bytes(int rows, int K) {
    if (rows < 0 || K <= 0 || K % 64 != 0) return -1;
    long row_blocks = (rows + 127) / 128;
    return row_blocks * (K / 64) * 512L;
}

int oracle_swizzle_scales(const uint8_t* s, int rows, int K, uint8_t* out) {
    long bytes = oracle_swizzled_bytes(rows, K);
    if (bytes < 0) return -1;
    int kb_per_row = K / 16, steps = K / 64;
    long row_blocks = (rows + 127) / 128;
    for (long r = 0; r < row_blocks * 128; r++) {
        for (int kb = 0; kb < kb_per_row; kb++) {
            uint8_t v = (r < rows) ? s[r * kb_per_row + kb] : 0;
            long rb = r / 128, rr = r % 128, step = kb / 4, j = kb % 4;
            long off = (rb * steps + step) * 512 + 16 * (rr % 32) + 4 * (rr / 32) + j;
            out[off] = v;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 2:4 structured sparsity over packed bytes                                */
/* ------------------------------------------------------------------------ */

/* A packed byte (a pair of E2M1 values) is zero when both values are +-0. */
static int pair_is_zero(uint8_t b) { return (b & 0x77) == 0; }

/* The two positions (0..3) a group of four packed bytes keeps: its non-zero
 * bytes, then the lowest zero bytes until there are two.  -1 when more than
 * two are non-zero. */
static int group_positions(const uint8_t* g4, int* i0, int* i1) {
    int pos[4], n = 0;
    for (int i = 0; i < 4; i++)
        if (!pair_is_zero(g4[i])) pos[n++] = i;
    if (n > 2) return -1;
    for (int i = 0; i < 4 && n < 2; i++)
        if (pair_is_zero(g4[i])) pos[n++] = i;
    if (pos[0] > pos[1]) { int t = pos[0]; pos[0] = pos[1]; pos[1] = t; }
    *i0 = pos[0];
    *i1 = pos[1];
    return 0;
}

static void put_group(uint8_t* values, uint8_t* meta, long grp, const uint8_t* g4, int i0, int i1) {
    values[2 * grp] = g4[i0];
    values[2 * grp + 1] = g4[i1];
    uint8_t nib = (uint8_t)(i0 | (i1 << 2));
    if (grp & 1) meta[grp / 2] = (uint8_t)((meta[grp / 2] & 0x0F) | (nib << 4));
    else meta[grp / 2] = (uint8_t)((meta[grp / 2] & 0xF0) | nib);
}

int oracle_sparse24_compress(const uint8_t* codes, int rows, int K, uint8_t* values, uint8_t* meta) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return -1;
    long groups = (long)rows * (K / 8);
    memset(meta, 0, (size_t)((long)rows * (K / 16)));
    for (long grp = 0; grp < groups; grp++) {
        int i0, i1;
        if (group_positions(codes + 4 * grp, &i0, &i1)) return -1;
        put_group(values, meta, grp, codes + 4 * grp, i0, i1);
    }
    return 0;
}

int oracle_sparse24_decompress(const uint8_t* values, const uint8_t* meta, int rows, int K, uint8_t* codes) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return -1;
    long groups = (long)rows * (K / 8);
    for (long grp = 0; grp < groups; grp++) {
        uint8_t nib = (grp & 1) ? (uint8_t)(meta[grp / 2] >> 4) : (uint8_t)(meta[grp / 2] & 0x0F);
        int i0 = nib & 3, i1 = (nib >> 2) & 3;
        if (i0 >= i1) return -1;   /* not a valid position pair */
        uint8_t* g4 = codes + 4 * grp;
        g4[0] = g4[1] = g4[2] = g4[3] = 0;
        g4[i0] = values[2 * grp];
        g4[i1] = values[2 * grp + 1];
    }
    return 0;
}

/* Pruning: in each group of four value pairs (eight values along K) keep the
 * two pairs whose larger magnitude is largest (ties to the lower position),
 * set the others to zero, then quantize the pruned tensor as a dense one.
 * Each group keeps its largest value, so every 16-value block keeps its
 * amax: block scales and g are those of the unpruned tensor, and the kept
 * codes are the dense codes. */
int oracle_quantize_sparse24(const float* X, int rows, int K,
                             uint8_t* values, uint8_t* meta, uint8_t* scales, float* g_out) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return -1;
    for (long i = 0; i < (long)rows * K; i++)
        if (!isfinite(X[i])) return -1;
    float* P = (float*)malloc(sizeof(float) * (size_t)((long)rows * K > 0 ? (long)rows * K : 1));
    int* keep = (int*)malloc(sizeof(int) * (size_t)((long)rows * (K / 8) * 2 + 2));
    uint8_t* codes = (uint8_t*)malloc((size_t)((long)rows * (K / 2) + 1));
    if (!P || !keep || !codes) { free(P); free(keep); free(codes); return -1; }
    long groups = (long)rows * (K / 8);
    for (long grp = 0; grp < groups; grp++) {
        const float* x = X + 8 * grp;
        float key[4];
        for (int p = 0; p < 4; p++) {
            float a = fabsf(x[2 * p]), b = fabsf(x[2 * p + 1]);
            key[p] = a > b ? a : b;
        }
        /* the two largest keys; a later position wins only when strictly larger */
        int first = 0;
        for (int p = 1; p < 4; p++) if (key[p] > key[first]) first = p;
        int second = -1;
        for (int p = 0; p < 4; p++) {
            if (p == first) continue;
            if (second < 0 || key[p] > key[second]) second = p;
        }
        int i0 = first < second ? first : second, i1 = first < second ? second : first;
        keep[2 * grp] = i0;
        keep[2 * grp + 1] = i1;
        for (int p = 0; p < 4; p++) {
            int kept = (p == i0 || p == i1);
            P[8 * grp + 2 * p] = kept ? x[2 * p] : 0.0f;
            P[8 * grp + 2 * p + 1] = kept ? x[2 * p + 1] : 0.0f;
        }
    }
    int rc = oracle_quantize(P, rows, K, codes, scales, g_out);
    if (rc == 0) {
        memset(meta, 0, (size_t)((long)rows * (K / 16)));
        for (long grp = 0; grp < groups; grp++)
            put_group(values, meta, grp, codes + 4 * grp, keep[2 * grp], keep[2 * grp + 1]);
    }
    free(P);
    free(keep);
    free(codes);
    return rc;
}

int oracle_gemm_sparse24(const uint8_t* A, const uint8_t* sA,
                         const uint8_t* Bv, const uint8_t* Bm, const uint8_t* sB,
                         float alpha, int M, int N, int K,
                         uint16_t* D_bf16, double* ref, double* absdot) {
    if (!gemm_args_ok(M, N, K)) return -1;
    uint8_t* B = (uint8_t*)malloc((size_t)((long)N * (K / 2) + 1));
    if (!B) return -1;
    int rc = oracle_sparse24_decompress(Bv, Bm, N, K, B);
    if (rc == 0) rc = oracle_gemm(A, sA, B, sB, alpha, M, N, K, D_bf16, ref, absdot);
    free(B);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* MXFP4: E2M1 values, one E8M0 (power of two) scale per 32 values          */
/* ------------------------------------------------------------------------ */

double oracle_e8m0_value(int byte) {
    if (byte < 0 || byte > 255) return NAN;
    if (byte == 255) return NAN;
    return ldexp(1.0, byte - 127);
}

/* Per block of 32: X = 2^(floor(log2 amax) - 2) (2 = the exponent of E2M1's
 * largest value, 6 = 1.5 * 2^2), clamped to 2^-127 .. 2^127 and stored as
 * the byte log2(X) + 127; codes = E2M1(x / X), nearest even, saturating at 6,
 * keeping the sign of a value that rounds to zero.  An all-zero block gets
 * the byte 0 and zero codes. */
int oracle_quantize_mxfp4(const float* X, int rows, int K, uint8_t* codes, uint8_t* scales) {
    if (rows < 0 || K <= 0 || K % 32 != 0) return -1;
    for (long i = 0; i < (long)rows * K; i++)
        if (!isfinite(X[i])) return -1;
    for (int r = 0; r < rows; r++) {
        const float* x = X + (long)r * K;
        uint8_t* crow = codes + (long)r * (K / 2);
        memset(crow, 0, (size_t)(K / 2));
        for (int b = 0; b < K / 32; b++) {
            float amax = 0.0f;
            for (int i = 0; i < 32; i++) {
                float a = fabsf(x[32 * b + i]);
                if (a > amax) amax = a;
            }
            int shared = -127;
            if (amax > 0.0f) {
                int e;
                frexpf(amax, &e);               /* amax = f * 2^e, f in [0.5, 1) */
                shared = (e - 1) - 2;
                if (shared < -127) shared = -127;
                if (shared > 127) shared = 127;
            }
            scales[(long)r * (K / 32) + b] = (uint8_t)(amax > 0.0f ? shared + 127 : 0);
            volatile float Xs = ldexpf(1.0f, shared);
            for (int i = 0; i < 32; i++) {
                int k = 32 * b + i;
                int q;
                if (amax == 0.0f) {
                    q = signbit(x[k]) ? 8 : 0;
                } else {
                    volatile float v = x[k] / Xs;
                    q = oracle_e2m1_rne_satfinite(v);
                }
                crow[k / 2] |= (uint8_t)((k & 1) ? (q << 4) : q);
            }
        }
    }
    return 0;
}

/* Unsigned big integers, 32-bit limbs, little endian: the exact sums of MX
 * products span 2^-256 .. 2^267 (scales 2^-127 .. 2^127 on each side). */
#define BIG_LIMBS 24
typedef struct { uint32_t w[BIG_LIMBS]; } big_t;

static void big_add_shifted(big_t* x, uint64_t v, int shift) {
    int limb = shift / 32, bit = shift % 32;
    u128 carry = (u128)v << bit;
    for (int i = limb; i < BIG_LIMBS && carry; i++) {
        carry += x->w[i];
        x->w[i] = (uint32_t)carry;
        carry >>= 32;
    }
}

static int big_cmp(const big_t* a, const big_t* b) {
    for (int i = BIG_LIMBS - 1; i >= 0; i--)
        if (a->w[i] != b->w[i]) return a->w[i] < b->w[i] ? -1 : 1;
    return 0;
}

static void big_sub(big_t* a, const big_t* b) {   /* a -= b, a >= b */
    int64_t borrow = 0;
    for (int i = 0; i < BIG_LIMBS; i++) {
        int64_t d = (int64_t)a->w[i] - (int64_t)b->w[i] - borrow;
        borrow = d < 0;
        a->w[i] = (uint32_t)(d + (borrow ? ((int64_t)1 << 32) : 0));
    }
}

static void big_mul_small(big_t* a, uint32_t m) {
    uint64_t carry = 0;
    for (int i = 0; i < BIG_LIMBS; i++) {
        uint64_t t = (uint64_t)a->w[i] * m + carry;
        a->w[i] = (uint32_t)t;
        carry = t >> 32;
    }
}

static int big_bitlen(const big_t* a) {
    for (int i = BIG_LIMBS - 1; i >= 0; i--)
        if (a->w[i]) {
            int n = 32;
            while (!(a->w[i] >> (n - 1))) n--;
            return 32 * i + n;
        }
    return 0;
}

static int big_bit(const big_t* a, int i) { return i < 0 ? 0 : (int)((a->w[i / 32] >> (i % 32)) & 1u); }

static int big_any_below(const big_t* a, int i) {   /* any bit at index < i */
    for (int j = 0; j < i; j++)
        if (big_bit(a, j)) return 1;
    return 0;
}

static uint64_t big_shr_small(const big_t* a, int s) {   /* a >> s, known to fit 64 bits */
    uint64_t r = 0;
    for (int j = 0; j < 64; j++) r |= (uint64_t)big_bit(a, s + j) << j;
    return r;
}

/* BF16 (round to nearest even) of sign * P * 2^E, P a big integer. */
static uint16_t bf16_rne_big(int sign, const big_t* P, int E) {
    int nb = big_bitlen(P);
    if (nb == 0) return 0x0000;                 /* an exact zero is reported as +0 */
    int ev = nb - 1 + E;                        /* 2^ev <= value < 2^(ev+1) */
    int shift = (ev >= -126) ? nb - 8 : (-133 - E);
    uint64_t q;
    if (shift > 0) {
        q = big_shr_small(P, shift);
        int half = big_bit(P, shift - 1), sticky = big_any_below(P, shift - 1);
        if (half && (sticky || (q & 1))) q++;
    } else {
        q = big_shr_small(P, 0) << (-shift);
    }
    int eq = E + shift;
    if (q == 256) { q = 128; eq += 1; }
    uint16_t bits;
    if (q >= 128) {
        int biased = eq + 7 + 127;
        if (biased >= 255) bits = 0x7F80;
        else bits = (uint16_t)((biased << 7) | (int)(q - 128));
    } else {
        bits = (uint16_t)q;
    }
    return (uint16_t)((sign << 15) | bits);
}

static double big_to_double(const big_t* P, int E) {
    int nb = big_bitlen(P);
    if (nb == 0) return 0.0;
    int s = nb > 64 ? nb - 64 : 0;
    return ldexp((double)big_shr_small(P, s), s + E);
}

/* One exact MX dot product of K values (K % 32 == 0). */
static uint16_t mx_dot(const uint8_t* a, const uint8_t* sa, const uint8_t* b, const uint8_t* sb, int K,
                       float alpha, double* exact, double* absdot) {
    big_t pos, neg;
    memset(&pos, 0, sizeof pos);
    memset(&neg, 0, sizeof neg);
    double ad = 0.0;
    for (int blk = 0; blk < K / 32; blk++) {
        long s = 0, sabs = 0;                   /* quarter units: e2m1 half units squared */
        for (int i = 0; i < 32; i++) {
            int k = 32 * blk + i;
            int ca = (k & 1) ? (a[k / 2] >> 4) : (a[k / 2] & 0xF);
            int cb = (k & 1) ? (b[k / 2] >> 4) : (b[k / 2] & 0xF);
            long t = (long)e2m1_half_units(ca) * e2m1_half_units(cb);
            if ((ca ^ cb) & 8) t = -t;
            s += t;
            sabs += t < 0 ? -t : t;
        }
        int E = ((int)sa[blk] - 127) + ((int)sb[blk] - 127) - 2;   /* value = s * 2^E */
        if (s > 0) big_add_shifted(&pos, (uint64_t)s, E + 256);
        if (s < 0) big_add_shifted(&neg, (uint64_t)(-s), E + 256);
        ad += ldexp((double)sabs, E);
    }
    int sign = 0;
    if (big_cmp(&pos, &neg) >= 0) {
        big_sub(&pos, &neg);
    } else {
        big_sub(&neg, &pos);
        pos = neg;
        sign = 1;
    }
    /* alpha = +-ma * 2^ea2 exactly */
    uint32_t abits;
    memcpy(&abits, &alpha, 4);
    int sign_a = (int)(abits >> 31), ea = (int)((abits >> 23) & 0xFF);
    uint32_t ma = ea ? ((abits & 0x7FFFFF) | 0x800000u) : (abits & 0x7FFFFF);
    int ea2 = ea ? ea - 150 : -149;
    double mag = big_to_double(&pos, -256);
    if (exact) *exact = (sign ? -mag : mag) * (double)alpha;
    if (absdot) *absdot = ad * fabs((double)alpha);
    big_mul_small(&pos, ma);
    return bf16_rne_big(sign ^ sign_a, &pos, -256 + ea2);
}

int oracle_gemm_mxfp4(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB,
                      float alpha, int M, int N, int K, uint16_t* D_bf16, double* ref, double* absdot) {
    if (M < 0 || N < 0 || K <= 0 || K % 32 != 0 || K > (1 << 20) || !isfinite(alpha)) return -1;
    for (long i = 0; i < (long)M * (K / 32); i++) if (sA[i] == 0xFF) return -1;
    for (long i = 0; i < (long)N * (K / 32); i++) if (sB[i] == 0xFF) return -1;
    for (int m = 0; m < M; m++)
        for (int n = 0; n < N; n++) {
            double e, ad;
            uint16_t d = mx_dot(A + (long)m * (K / 2), sA + (long)m * (K / 32), B + (long)n * (K / 2),
                                sB + (long)n * (K / 32), K, alpha, &e, &ad);
            long o = (long)m * N + n;
            if (D_bf16) D_bf16[o] = d;
            if (ref) ref[o] = e;
            if (absdot) absdot[o] = ad;
        }
    return 0;
}
