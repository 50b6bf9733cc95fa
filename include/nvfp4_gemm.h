/*
 * nvfp4_gemm.h -- C ABI of the B200 (sm_100a) NVFP4 block-scaled GEMM library
 * (libnvfp4gemm.so).
 *
 * The operation (one GEMM):
 *
 *   D[m][n] = bf16_rne( alpha * sum_k  e2m1(A[m,k]) * e4m3(sA[m, k/16])
 *                                     * e2m1(B[n,k]) * e4m3(sB[n, k/16]) )
 *
 * Sources: NVFP4 packs two 4-bit values per byte with per-block scale factors
 * ("The SM120 FP4 Kernel Disaster", section "Input Knowledge Required",
 * item 3); one FP8 scale per 16 elements and a BF16 output, with the byte
 * model M*K/2 + K*N/2 + M*K/16 + K*N/16 + 2*M*N ("Peeling the Kernel Onion",
 * section "The Benchmark Design"); the call takes a global alpha and an
 * output tensor ("Peeling the Kernel Onion", section "The Chain of
 * Reasoning"); packed-K shapes must agree between operands ("The SM120 FP4
 * Kernel Disaster", section "The Bash Command").
 *
 * Data layout at the ABI (all row-major, K the contiguous dimension):
 *   A   uint8 [M][K/2]   E2M1 codes, element k of a row in byte k/2, the even
 *                        k in the low nibble (bits 3..0), bit 3 of a code is
 *                        its sign.
 *   sA  uint8 [M][K/16]  E4M3 block scales (bias 7), one per 16 elements of a
 *                        row.  Must be non-negative and not NaN (0x7F); this
 *                        is not checked.
 *   B   uint8 [N][K/2],  sB uint8 [N][K/16]   the same for the N operand ("TN").
 *   D   bf16  [M][N].
 * Any re-layout of the scales for the tensor cores happens on the device
 * inside these calls.
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers (cudaMalloc'd or equivalent) on the current
 *     device unless a parameter says otherwise; the caller owns them and they
 *     must stay valid until the work on `stream` has finished.  The library
 *     never frees caller memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous: they enqueue work and return without
 *     synchronising, except nvfp4_get_device_error.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns a status and launches nothing.  No exception or
 *     abort crosses this boundary.
 *   - The library owns per-device, per-stream scratch (scales re-laid out for
 *     the tensor cores, when a call needs that) and a 4 KB block of counters
 *     per stream for the grouped GEMM's run-time work hand-out, which it
 *     allocates on first need; scratch grows with the shapes.  The first call
 *     of a new, larger shape on a stream may therefore call cudaMalloc, so
 *     make it before capturing that stream into a CUDA graph.  Calls on
 *     different streams use different scratch and counters and may overlap;
 *     calls on one stream run in stream order.
 *   - Device-side waits are bounded; a wait that runs out records
 *     NVFP4_ERR_TIMEOUT in a device error word read by nvfp4_get_device_error.
 *   - Requires an sm_100 device (B200/GB200); others get
 *     NVFP4_ERR_UNSUPPORTED_DEVICE.  There is no fallback path.
 */
#ifndef NVFP4_GEMM_H
#define NVFP4_GEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, misaligned pointer */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 64 != 0, N % 8 != 0, size limits */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 3, /* not compute capability 10.0 */
    NVFP4_ERR_CUDA = 4,               /* a CUDA runtime/driver call failed */
    NVFP4_ERR_TIMEOUT = 5,            /* a bounded device-side wait ran out */
    NVFP4_ERR_NO_MEMORY = 6           /* scratch allocation failed */
} nvfp4_status;

/*
 * nvfp4_gemm -- single NVFP4 GEMM, D = alpha * A * B^T (see the top of this
 * file for the formula and layouts).
 *   A [M][K/2], sA [M][K/16], B [N][K/2], sB [N][K/16]: device, read only.
 *   alpha: fp32 global scale (for quantised inputs, gA * gB).
 *   D [M][N] bf16: device, written.
 *   Requirements: M >= 0, N >= 0, K > 0; K % 64 == 0; N % 8 == 0; A, B, D
 *   16-byte aligned; sA, sB 4-byte aligned.  M == 0 or N == 0 is a no-op.
 * One or two token rows (up to four for small N, K >= 4096 beyond one) run
 * on the CUDA cores: a matrix-vector kernel that streams B straight into
 * registers, whose block sums are exact and whose fp32 sum over the K/16
 * blocks is the only rounding before alpha and the BF16 store.  Other small
 * M uses the weight-streaming tensor-core kernel (B rows on the MMA's M side,
 * split-K over a thread-block cluster); large M uses 128- or 256-row output
 * tiles, on CTA pairs for the largest shapes.  Environment switches, for
 * tuning and tests: NVFP4_GEMM_GEMV=0 keeps every M on the tensor cores and
 * NVFP4_GEMM_GEMV=<n> sends every M <= n (at most 16) to the CUDA cores;
 * NVFP4_GEMM_PAIR=0 keeps large shapes off the CTA-pair kernel.
 */
nvfp4_status nvfp4_gemm(const void* A, const void* sA,
                        const void* B, const void* sB,
                        float alpha, void* D,
                        int M, int N, int K, void* stream);

/*
 * nvfp4_gemm_ex -- nvfp4_gemm with flags (0 gives exactly nvfp4_gemm).
 *   NVFP4_GEMM_B_CONSTANT: the caller guarantees that B and sB are not written
 *   by any work enqueued earlier on `stream` that may still be running (model
 *   weights).  The kernel then starts loading B before the previous kernel
 *   on the stream has finished (it still waits for it before reading A or sA
 *   and before writing D), which hides the memory latency of back-to-back
 *   weight-streaming GEMMs.  A, sA and D get no such relaxation.
 *   Other bits: NVFP4_ERR_INVALID_ARG.
 */
#define NVFP4_GEMM_B_CONSTANT 1u
nvfp4_status nvfp4_gemm_ex(const void* A, const void* sA,
                           const void* B, const void* sB,
                           float alpha, void* D,
                           int M, int N, int K, unsigned flags, void* stream);

/*
 * nvfp4_grouped_gemm -- MoE-style grouped GEMM: G independent problems that
 * share N and K.  Rows [row_offsets[g], row_offsets[g+1]) of A are multiplied
 * by B[g] and scaled by alpha[g]:
 *   D[m][n] = bf16_rne(alpha[g] * sum_k A[m,k] sA[m,k/16] B[g][n,k] sB[g][n,k/16]).
 *   A [M_total][K/2], sA [M_total][K/16]  rows grouped by g (device).
 *   B [G][N][K/2],    sB [G][N][K/16]     one weight matrix per group (device).
 *   alpha [G] fp32 (device), row_offsets [G+1] int32 (device): row_offsets[0]
 *   must be 0, row_offsets[G] must be M_total and the sequence non-decreasing
 *   (this is not checked on the device; violating it is undefined).
 *   D [M_total][N] bf16 (device).
 *   Groups with no rows cost nothing and their B is never read.
 *   Requirements: as nvfp4_gemm, and G >= 1, K % 256 == 0, sA and sB 16-byte
 *   aligned (the kernel loads 256-element K tiles of row-major scales with
 *   TMA); otherwise NVFP4_ERR_UNSUPPORTED_SHAPE / NVFP4_ERR_INVALID_ARG.
 * Sources: MoE routing gives each expert about 16 rows ("Peeling the Kernel
 * Onion", section "The Critical Connection to Real Inference"); persistent
 * grouped GEMM kernels amortise small per-expert problems (same page, section
 * "Knowledge Created and Its Impact").
 */
nvfp4_status nvfp4_grouped_gemm(const void* A, const void* sA,
                                const void* B, const void* sB,
                                const float* alpha, const int32_t* row_offsets,
                                int G, void* D,
                                int M_total, int N, int K, void* stream);

/*
 * nvfp4_quantize -- fp32 X [rows][K] (device) to NVFP4:
 *   g = amax(|X|) / (6 * 448)  (one global scale for the whole tensor; 1.0 if
 *   X is all zero), per 16-element block s = E4M3_rne_satfinite(amax_blk /
 *   (6 g)), per element q = E2M1_rne_satfinite(x / (g * s)); a zero scale
 *   gives zero codes.  All steps IEEE fp32 with round-to-nearest-even, so the
 *   output is bit-reproducible.  The sign of x is kept in the code, also when
 *   it rounds to zero.
 *   codes [rows][K/2] uint8, scales [rows][K/16] uint8, g_out [1] fp32: device,
 *   written.  X must be finite (not checked).  K % 16 == 0, X 16-byte aligned.
 */
nvfp4_status nvfp4_quantize(const float* X, int rows, int K,
                            void* codes, void* scales, float* g_out, void* stream);

/*
 * nvfp4_swizzle_scales -- re-lay row-major E4M3 scales [rows][K/16] into the
 * tensor-core scale-factor layout the GEMM kernels feed to tcgen05.cp:
 * 512-byte atoms of 128 rows x 4 scale blocks (one 64-element MMA K step),
 * row r, block j of an atom at byte 16*(r%32) + 4*(r/32) + j, atoms ordered
 * along K within each 128-row block, padding rows zero.
 *   s_rowmajor (device, read), s_swizzled (device, nvfp4_swizzled_scale_bytes
 *   bytes, written).  K % 64 == 0; both pointers 4-byte aligned.
 */
nvfp4_status nvfp4_swizzle_scales(const void* s_rowmajor, int rows, int K,
                                  void* s_swizzled, void* stream);

/* Bytes nvfp4_swizzle_scales writes: ceil(rows/128) * (K/64) * 512, or 0 for
 * invalid arguments. */
size_t nvfp4_swizzled_scale_bytes(int rows, int K);

/*
 * nvfp4_get_device_error -- synchronise `stream`, then read and clear the
 * current device's error word.  Returns NVFP4_ERR_TIMEOUT if a device-side
 * wait ran out since the last call, NVFP4_ERR_CUDA if the synchronisation
 * failed, else NVFP4_OK.
 */
nvfp4_status nvfp4_get_device_error(void* stream);

/* Human-readable name of a status (static storage, never NULL). */
const char* nvfp4_status_string(nvfp4_status status);

/*
 * nvfp4_debug_wait_timeout -- diagnostics for the bounded-wait machinery:
 * launches one block whose thread waits on a shared-memory barrier that
 * nothing ever arrives on, using the same bounded wait as the GEMM kernels
 * with a limit of `timeout_ns` nanoseconds (1e3 .. 5e9).  The kernel then
 * records NVFP4_ERR_TIMEOUT in the device error word and returns normally, so
 * a following nvfp4_get_device_error reports NVFP4_ERR_TIMEOUT and the
 * context stays usable.
 */
nvfp4_status nvfp4_debug_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * nvfp4_quantize_scaled -- quantize-and-pack with the global scale given:
 * the activation-side step that feeds the GEMM in decode, where a tensor's
 * global scale is fixed in advance rather than taken from its own amax
 * ("Peeling the Kernel Onion", section "The Critical Connection to Real
 * Inference": activations are quantized upstream of each GEMM).
 *   X       rows x K values, row-major: fp32 (x_is_bf16 = 0) or BF16
 *           (x_is_bf16 = 1); 16-byte aligned.  K a multiple of 16.
 *   g       global scale, positive and finite.
 *   codes   out: packed E2M1 [rows][K/2] (8-byte aligned), low nibble = even k.
 *   scales  out: E4M3 block scales [rows][K/16], s = E4M3(amax_blk / (6 g))
 *           round-to-nearest-even with saturation to 448; codes are
 *           E2M1(x / (g * s)) with the same rounding and saturation to 6.
 * Bit-exact with nvfp4_quantize's block steps for the same g (one launch
 * instead of three: no amax pass).  Launched with programmatic dependent
 * launch, so a following nvfp4_gemm on the stream starts its prologue while
 * this kernel runs.  Returns NVFP4_ERR_INVALID_ARG for bad pointers, g <= 0
 * or non-finite, NVFP4_ERR_UNSUPPORTED_SHAPE for K % 16 != 0.
 */
nvfp4_status nvfp4_quantize_scaled(const void* X, int x_is_bf16, int rows, int K, float g, void* codes,
                                   void* scales, void* stream);

/*
 * nvfp4_gemm_bf16a -- the GEMM with BF16 activations, quantized inside the
 * call with the given global scale gA (the quantize-and-pack of
 * nvfp4_quantize_scaled, then nvfp4_gemm), so that decode feeds the GEMM
 * straight from the previous layer's BF16 output ("Peeling the Kernel Onion",
 * section "The Critical Connection to Real Inference").
 *   A      BF16 [M][K], row-major, 16-byte aligned.
 *   gA     the activations' global scale, positive and finite.
 *   B, sB  the NVFP4 weights as for nvfp4_gemm; alpha = gA * gB as there.
 *   D      BF16 [M][N].
 * The activations are quantized into per-stream scratch by the one-launch
 * quantizer, then the GEMM runs (two launches, chained by programmatic
 * dependent launch).  With the environment variable NVFP4_GEMM_FUSE_QUANT=1,
 * for M <= 64 with K a multiple of 256 and 16-byte aligned sB, the GEMM
 * kernel instead quantizes each activation tile in shared memory (one launch;
 * slower on the attention shapes, where every CTA of a weight-tile column
 * repeats the conversion).  Either way the result equals
 * nvfp4_quantize_scaled followed by nvfp4_gemm on the same stream.  Errors as for nvfp4_gemm, plus
 * NVFP4_ERR_INVALID_ARG for gA not positive and finite.
 */
nvfp4_status nvfp4_gemm_bf16a(const void* A, float gA, const void* B, const void* sB, float alpha, void* D, int M,
                              int N, int K, void* stream);

/*
 * nvfp4_fp4_peak_probe -- calibration of the dense FP4 tensor-core rate (no
 * counterpart on the pages, which quote only a vendor-style peak for another
 * GPU, "Peeling the Kernel Onion", section "The Results").  Launches one CTA
 * per SM (pair = 0: tcgen05.mma.cta_group::1, 128 x 256 x 64 per instruction)
 * or one 2-CTA cluster per two SMs (pair = 1: cta_group::2, 256 x 256 x 64 per
 * instruction per pair), each issuing `steps` (1 .. 1e8) block-scaled
 * kind::mxf4nvf4 MMAs back to back on operands resident in shared memory and
 * scales resident in TMEM.  Writes the number of CTAs launched to *ctas_out.
 * The caller times the launch on `stream`; the work is
 * steps x ctas x 2 x 128 x 256 x 64 FLOPs in both forms.  The MMA results are
 * discarded.  Returns NVFP4_ERR_INVALID_ARG for arguments out of range.
 */
nvfp4_status nvfp4_fp4_peak_probe(int pair, long long steps, int* ctas_out, void* stream);

/*
 * nvfp4_gemm_noalloc -- the same GEMM as nvfp4_gemm (same arguments, layouts,
 * requirements and result), for callers that are not allowed to allocate
 * device memory during the call: runtimes that own and pool all device
 * memory themselves, code that runs under a fixed memory budget, or callers
 * that must keep driver allocations off their launch path.  nvfp4_gemm may
 * cudaMalloc scratch on its first call of a new shape; this entry point never
 * calls cudaMalloc, cudaFree or any allocating routine.  It has no counterpart
 * on the source pages; it is a deployment convenience of this library.
 *   Its scratch is a static device array of 8 MiB (8,388,608 bytes) that
 *   every GPU which loads the library keeps until the process exits.  A few
 *   token rows run on the CUDA cores and use none of it.  When K % 256 == 0
 *   and sA, sB are 16-byte aligned the tensor-core kernels read the
 *   row-major scales directly, and the array holds at most the fp32 partial
 *   tiles of a K split (problems large enough for nvfp4_gemm's CTA-pair
 *   kernel run on the single-CTA persistent kernel instead, as that kernel
 *   wants its scales re-laid out first).  The other problems (K % 256 != 0,
 *   or scales only 4-byte aligned) first have their scales re-laid out for
 *   the tensor cores into the array; such a problem whose scales need more,
 *   i.e. (ceil(M/128) + ceil(N/128)) * (K/64) * 512 bytes (plus up to 255
 *   bytes of alignment), is rejected with NVFP4_ERR_UNSUPPORTED_SHAPE before
 *   anything is launched.  Partial tiles that do not fit after the scales
 *   make the call run without a K split instead (slower, same result within
 *   the bound).
 *   The first call on a device that uses the array looks up its device
 *   address (cudaGetSymbolAddress, with that device current) and keeps it
 *   for the life of the process; make that first call before capturing the
 *   stream into a CUDA graph.  The kept address does not survive
 *   cudaDeviceReset (which unloads the library's device code): do not call
 *   this entry point on a device after resetting it.
 *   All calls share the one array, so calls whose work overlaps on the GPU
 *   (different streams, or different host threads) race on it: serialise
 *   them.  Each call rewrites every scratch byte it reads, so no clearing is
 *   needed between calls.
 */
nvfp4_status nvfp4_gemm_noalloc(const void* A, const void* sA,
                                const void* B, const void* sB,
                                float alpha, void* D,
                                int M, int N, int K, void* stream);

/*
 * nvfp4_gemm_sparse24 -- D = alpha * A * B^T with 2:4-sparse NVFP4 weights B.
 * The pages name FP4 structured sparsity as a way to cut what small-batch
 * decode demands ("Peeling the Kernel Onion", sections "Assumptions Embedded
 * in the Benchmark" and "Knowledge Created and Its Impact") and give no
 * layout; this library's layout: of every 4 consecutive packed bytes of a
 * row of B (pairs of E2M1 values) at most 2 are non-zero, stored as
 *   Bv [N][K/4]:  the 2 kept bytes of each group of 4, lower position first;
 *   Bm [N][K/16]: per group a nibble p0 | p1 << 2 (positions 0..3, p0 < p1),
 *                 the even group in the low nibble of each byte;
 *   sB [N][K/16]: the dense E4M3 block scales, as for nvfp4_gemm.
 * The result is nvfp4_gemm's on the dense B this describes (dropped bytes
 * zero).  A, sA, alpha, D and the flags are as for nvfp4_gemm_ex.
 *   Requirements: K % 64 == 0, N % 8 == 0; A, Bv, D 16-byte aligned; sA, Bm,
 *   sB 4-byte aligned.  Metadata nibbles with p0 >= p1 are not checked; they
 *   give an unspecified result but every access stays inside the arguments.
 *   Up to 8 token rows (NVFP4_GEMM_SP24_GEMV=<n> sets the limit, 0..16) run a
 *   CUDA-core kernel on the compressed weights, reading 6K/16 weight bytes
 *   per row instead of 9K/16.  Above it B is expanded to dense codes in
 *   per-stream scratch (may cudaMalloc on a stream's first use of a size, as
 *   nvfp4_gemm's scratch) and the dense GEMM runs.
 */
nvfp4_status nvfp4_gemm_sparse24(const void* A, const void* sA,
                                 const void* Bv, const void* Bm, const void* sB,
                                 float alpha, void* D,
                                 int M, int N, int K, unsigned flags, void* stream);

/*
 * nvfp4_gemm_mxfp4 -- D = alpha * A * B^T with MXFP4 operands, the OCP
 * microscaling format the same tensor-core instruction family takes
 * (tcgen05.mma kind::mxf4, block32): E2M1 codes packed as for nvfp4_gemm,
 * with one E8M0 scale per 32 values along K (byte e = 2^(e - 127); 255 is
 * NaN and must not occur).  The pages use NVFP4 only; this is the format's
 * sibling, exact up to the fp32 accumulation like nvfp4_gemm.
 *   A  [M][K/2], sA [M][K/32] (E8M0 bytes), B [N][K/2], sB [N][K/32];
 *   alpha fp32 (no global scales in this format; kept for the same call
 *   shape); D bf16 [M][N]; flags as for nvfp4_gemm_ex.
 *   Requirements: K % 64 == 0, N % 8 == 0; A, B, D 16-byte aligned (scales
 *   any alignment).  M == 0 or N == 0 is a no-op.
 *   Up to 4 token rows run on the CUDA cores (exact block sums, each scaled
 *   by 2^(ea + eb - 254) with ldexpf, fp32 sum); above that both operands'
 *   scales are re-laid out into per-stream scratch (may cudaMalloc on a
 *   stream's first use of a size) and the tensor-core kernel runs.  The
 *   partial sums are fp32, so products whose scales leave the fp32 range
 *   (about 2^-149 .. 2^127) under- or overflow.
 *   Errors: as for nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_mxfp4(const void* A, const void* sA,
                              const void* B, const void* sB,
                              float alpha, void* D,
                              int M, int N, int K, unsigned flags, void* stream);

/* Library version as major*10000 + minor*100 + patch. */
int nvfp4_version(void);

/* Number of kernels this library has enqueued in this process so far, on all
 * devices (a launch captured into a CUDA graph counts once, at capture). */
unsigned long long nvfp4_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_GEMM_H */
