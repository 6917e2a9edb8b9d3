/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 block quantization, dequantization
 * and the block-scaled FP4 GEMM on B200 (sm_100a).
 *
 * What the calls compute is defined by these pages (cited by title and
 * section / equation):
 *   [46] "Four Over Six: more accurate NVFP4 quantization with adaptive block
 *        scaling" (Chinese translation): §1 (Fig. 1, Table 1), §2.1 Eq. 1-3.
 *   [NV] Write-up of NVIDIA's "Pretraining LLMs with NVFP4": §一 format,
 *        §二 the four techniques (2D weight blocks, random Hadamard transform,
 *        stochastic rounding), §四 Blackwell tensor cores, §六 procedure,
 *        §七 ablations (SR on gradients only, 1D blocks for activations).
 *   [Q2] News write-up of Quartet II / MS-EDEN: §一 (MS-EDEN), §二 (recipe).
 *
 * Conventions shared by every call
 *   - All device pointers are caller-owned CUDA device memory; the library
 *     never allocates.  Scratch memory comes from the caller's workspace,
 *     except for nvfp4_quantize_noalloc, whose scratch is a fixed array
 *     inside the library (see that call).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Nothing synchronises the
 *     host; the tensor scale alpha stays on the device.
 *   - Errors the host can see (bad arguments, shapes, alignment, workspace
 *     too small) return before anything is launched.  Errors found on the
 *     device (non-finite input, a spin-wait that gave up) are written as a
 *     negative nvfp4_status_t to the optional device word `status`; that word
 *     is sticky: the library only ever writes error codes into it, the caller
 *     zeroes it.  Outputs are unspecified after a device-side error.
 *   - bf16 tensors are row-major with a row stride `ld` (elements); the base
 *     pointer must be 16-byte aligned and ld a multiple of 8.
 *   - Packed FP4 codes: two E2M1 codes per byte, element 2j in the low nibble
 *     of byte j; a code is sign (bit 3) + magnitude index (bits 0-2) into
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6} ([46] §1).
 *   - Block scales: one unsigned E4M3 byte (bias 7, max 448) per block.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_ARG = -1,        /* bad mode, flag combination or null pointer */
  NVFP4_ERR_SHAPE = -2,      /* a dimension breaks the block / tile rules   */
  NVFP4_ERR_ALIGN = -3,      /* a pointer or stride is not 16-byte aligned  */
  NVFP4_ERR_NONFINITE = -4,  /* device: the input holds a NaN or an Inf     */
  NVFP4_ERR_LAUNCH = -5,     /* a kernel could not be launched              */
  NVFP4_ERR_TIMEOUT = -6,    /* device: a bounded spin-wait gave up         */
  NVFP4_ERR_CUDA = -7,       /* a CUDA runtime call failed                  */
  NVFP4_ERR_WORKSPACE = -8   /* workspace missing or smaller than required  */
} nvfp4_status_t;

/* How a 16-element block is encoded. */
typedef enum {
  /* Eq. 2 scale rounded to nearest E4M3, Eq. 3 values rounded to nearest
   * ([46] §2.1, [NV] §六).  Block maximum mapped to 6. */
  NVFP4_RTN = 0,
  /* Four Over Six ([46] §1, [Q2] §二): encode the block with its maximum
   * mapped to 6 and to 4, keep the encoding with the lower squared error
   * measured after dequantization (ties keep 6). */
  NVFP4_FOUR_SIX = 1,
  /* Random Hadamard transform of each 16-block, scale rounded up to E4M3,
   * values stochastically rounded ([NV] §二, §七: for gradients). */
  NVFP4_RHT_SR = 2,
  /* MS-EDEN ([Q2] §一): rotate, round the values to nearest, and put the
   * randomness only on the E4M3 scale, stochastically rounded from the
   * unbiasing value ||r||^2 / (alpha <r, q>). */
  NVFP4_MS_EDEN = 3,
  /* As NVFP4_RHT_SR, with the values stochastically rounded by the sm_100a
   * convert instruction that takes caller random bits ([NV] §四 names
   * hardware stochastic rounding).  One Philox draw per block (tag 4,
   * unit = block index) gives one 32-bit word per group of four elements;
   * the instruction derives each element's 16-bit field from it.  Codes
   * differ from NVFP4_RHT_SR's draw for draw; both are unbiased.  Not
   * accepted with NVFP4_BLOCK2D. */
  NVFP4_RHT_SR_HW = 4
} nvfp4_mode_t;

/* nvfp4_quantize flags */
#define NVFP4_ROWWISE 0x1u          /* blocks along C (the contiguous axis)      */
#define NVFP4_COLWISE 0x2u          /* blocks along R; output is the transpose   */
#define NVFP4_BLOCK2D 0x4u          /* 16x16 blocks (weights, [NV] §二); RTN/4-6 */
#define NVFP4_SINGLE_PASS 0x8u      /* amax and quantize in one cooperative launch:
                                     * per-CTA maxima, a grid barrier (bounded:
                                     * 1 s, or the nanoseconds in the environment
                                     * variable NVFP4_BARRIER_TIMEOUT_NS read at
                                     * each call; then NVFP4_ERR_TIMEOUT in
                                     * *status and unspecified outputs), then
                                     * the encoding; results
                                     * identical to the two-pass call.  Needs 16
                                     * more workspace bytes (the barrier counter,
                                     * cleared by the call).  Pays off for small
                                     * tensors (one launch, the re-read from L2). */
#define NVFP4_ALPHA_PROVIDED 0x10u  /* use *alpha_in instead of Eq. 1            */
#define NVFP4_GEMM_SCALE_LAYOUT 0x20u /* write scales in nvfp4_gemm's layout     */
#define NVFP4_RHT 0x40u             /* rotate before RTN / FOUR_SIX encoding     */
#define NVFP4_HEADROOM 0x200u       /* alpha = amax / (4 * 448) instead of Eq. 1's
                                     * amax / (6 * 448): the M = 4 candidate of
                                     * Four Over Six then never saturates        */
#define NVFP4_VECTOR_SCALES 0x400u  /* one tensor scale per row of the quantized
                                     * operand ([NV] §九 names finer-than-tensor
                                     * global scales as the remedy for one global
                                     * amax; READING: Eq. 1 applied to each vector
                                     * on its own): alpha_i = amax_i / (6 * 448)
                                     * over row i of x (rowwise) or column i of x
                                     * (columnwise), rotated values in rotating
                                     * modes.  alpha_row then points to R floats,
                                     * alpha_col to C floats; amax_out receives
                                     * the largest vector amax per orientation.
                                     * 1D blocks only (not with BLOCK2D,
                                     * SINGLE_PASS or ALPHA_PROVIDED).  The
                                     * workspace holds the R + C vector maxima. */
#define NVFP4_AMAX_PROVIDED 0x800u  /* skip the amax pass: alpha_in points to
                                     * the three device floats nvfp4_amax
                                     * writes (plain, rotated rows, rotated
                                     * columns), from which alpha follows by
                                     * Eq. 1 exactly as in the two-pass path:
                                     * [0] without rotation, [1] for rotated
                                     * rows, [2] for rotated columns.  A
                                     * non-finite marker (0xFFFFFFFF) sets
                                     * NVFP4_ERR_NONFINITE.  Not with
                                     * ALPHA_PROVIDED, SINGLE_PASS or
                                     * VECTOR_SCALES; needs no workspace. */
/* nvfp4_dequantize flags (NVFP4_BLOCK2D and NVFP4_GEMM_SCALE_LAYOUT also apply) */
#define NVFP4_INVERSE_RHT 0x80u     /* undo the rotation after decoding          */
#define NVFP4_OUT_BF16 0x100u       /* write bf16 instead of fp32                */

/* nvfp4_gemm output types */
#define NVFP4_OUT_DTYPE_BF16 0
#define NVFP4_OUT_DTYPE_FP32 1

/* Outputs of nvfp4_quantize.  NULL members are not written; the row members
 * are required with NVFP4_ROWWISE, the column members with NVFP4_COLWISE.
 *   codes_row  [R, C/2] bytes            codes_col  [C, R/2] bytes
 *   scales_row [R, C/16]                 scales_col [C, R/16]
 *              BLOCK2D: [R/16, C/16]                BLOCK2D: [C/16, R/16]
 *              GEMM layout: see below               GEMM layout: see below
 *   alpha_row, alpha_col: one float each (device), the tensor scale of Eq. 1
 *   amax_out:  optional float[2] (device): amax seen by rows, by columns
 *   status:    optional sticky device error word (see conventions)
 * Column outputs hold the transpose: row c of codes_col / scales_col encodes
 * column c of x, so both outputs are K-major GEMM operands.
 *
 * GEMM scale layout (NVFP4_GEMM_SCALE_LAYOUT), for an operand with `rows`
 * rows and K columns (rows % 128 == 0, K % 64 == 0): the scale of (row m,
 * K-block j) sits at byte
 *     ((m / 128) * (K / 64) + j / 4) * 512 + (m % 32) * 16 + ((m / 32) % 4) * 4 + j % 4,
 * i.e. 512-byte atoms of 128 rows x 4 scales, in the order the tcgen05
 * block-scaled MMA reads them.  With BLOCK2D the 16x16 scale is written for
 * every one of its 16 rows (rows x K/16 bytes in total). */
typedef struct {
  uint8_t* codes_row;
  uint8_t* scales_row;
  float* alpha_row;
  uint8_t* codes_col;
  uint8_t* scales_col;
  float* alpha_col;
  float* amax_out;
  int32_t* status;
} nvfp4_qtensor_t;

/* Bytes of device workspace nvfp4_quantize needs for an R x C tensor and
 * these flags (0 if none).  The workspace is scratch: its contents on entry
 * do not matter, and one workspace must not be shared by calls that may run
 * at the same time. */
NVFP4_API size_t nvfp4_workspace_size(int64_t R, int64_t C, uint32_t flags);

/* Quantize the bf16 tensor x [R, C] (row stride ld) to NVFP4.
 *
 * Steps ([46] §2.1 Eq. 1-3; [NV] §六):
 *   1. amax = max |x| (max over the rotated values in rotating modes,
 *      separately per orientation); alpha = amax / (6 * 448)        (Eq. 1)
 *      -- skipped with NVFP4_ALPHA_PROVIDED (alpha = *alpha_in, device), or
 *      taken from amax values computed earlier with NVFP4_AMAX_PROVIDED.
 *   2. per block: Delta = E4M3(amax_block / (alpha * M))             (Eq. 2)
 *   3. per element: q = E2M1(x / (alpha * Delta)), computed as x times the
 *      correctly rounded reciprocal of alpha * Delta                 (Eq. 3)
 * with the mode choosing M, the rounding of Delta and q, and the 4/6 choice
 * (see nvfp4_mode_t).  Rotating modes (RHT_SR, MS_EDEN, RHT_SR_HW, or the
 * NVFP4_RHT flag) first replace each 16-block v by (1/4) H16 D v, D = diag of 16 random
 * signs drawn from `seed`; the same D serves every block and both
 * orientations, so two operands quantized with the same seed along their
 * shared K axis multiply to the unrotated product.
 *
 * Random bits come from Philox4x32-10 keyed by `seed`; `stream_id` (< 2^31)
 * separates the noise of tensors that share a seed.
 *
 * Shape rules: R, C >= 0; C % 16 == 0; R % 16 == 0 with NVFP4_COLWISE or
 * NVFP4_BLOCK2D (2D blocks: RTN / FOUR_SIX only, no rotation);
 * R * C / 16 < 2^31.  An empty tensor (R or C = 0) is a no-op.
 * Output pointers: 16-byte aligned.  `workspace` must hold
 * nvfp4_workspace_size(R, C, flags) bytes.  Arithmetic is IEEE binary32
 * without FMA contraction, so codes and scales are bit-exact with a plain
 * CPU restatement of these steps. */
NVFP4_API nvfp4_status_t nvfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld,
                              nvfp4_mode_t mode, uint32_t flags, uint64_t seed,
                              uint32_t stream_id, const float* alpha_in,
                              const nvfp4_qtensor_t* out, void* workspace,
                              size_t workspace_bytes, void* stream);

/* The amax values of Eq. 1 ([46] §2.1 Eq. 1; [NV] §六 step 1) of the bf16
 * tensor x [R, C] (row stride ld), for later nvfp4_quantize calls with
 * NVFP4_AMAX_PROVIDED: one read of x gives
 *   amax_out[0] = max |x|                               (plain)
 *   amax_out[1] = max |(1/4) H16 D v| over the 16-element row blocks v
 *                 (with NVFP4_ROWWISE | NVFP4_RHT)
 *   amax_out[2] = the same over the 16-element column blocks
 *                 (with NVFP4_COLWISE | NVFP4_RHT; R % 16 == 0)
 * with D the sign diagonal drawn from `seed` (as nvfp4_quantize rotates).
 * A tensor whose plain, row or column maxima several quantize calls need is
 * read once instead of once per call: pass amax_out as each call's alpha_in
 * with NVFP4_AMAX_PROVIDED.  Entries not requested are 0.
 * Each value is a device float (bit pattern 0xFFFFFFFF if a NaN or Inf was
 * read, and then NVFP4_ERR_NONFINITE in *status when status is not NULL).
 * x 16-byte aligned, ld % 8 == 0, C % 16 == 0; amax_out 4-byte aligned (3
 * floats, written through the stream; no workspace). */
NVFP4_API nvfp4_status_t nvfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags,
                                    uint64_t seed, float* amax_out, int32_t* status, void* stream);

/* nvfp4_quantize for callers that may not allocate device memory while they
 * run (no page defines this; it has no counterpart in the method): a plugin
 * inside another runtime that owns all device memory, or a program whose
 * memory plan is fixed at start-up.  Same arguments and results as
 * nvfp4_quantize, minus the workspace: the scratch (the amax pass's per-CTA
 * partials and, with NVFP4_SINGLE_PASS, the grid barrier's counter) lives in
 * an 8192-byte array compiled into the library, which every GPU that loads
 * the library holds until the process exits.  A call that would need more
 * scratch than that returns NVFP4_ERR_WORKSPACE.  Arguments are checked
 * first; the first accepted call on each device (with that device current)
 * then looks up the array's device address: make it before any stream
 * capture starts, and do not reset the device (cudaDeviceReset) between
 * calls, since the address is kept.  All calls on a device share the array,
 * so calls whose kernels may overlap on the GPU race and can give wrong
 * results or a barrier timeout: order them on one stream.  The partials need
 * no clearing; the barrier counter is cleared by each single-pass call with a
 * stream-ordered memset.  The function itself allocates nothing. */
NVFP4_API nvfp4_status_t nvfp4_quantize_noalloc(const void* x, int64_t R, int64_t C, int64_t ld,
                                                nvfp4_mode_t mode, uint32_t flags, uint64_t seed,
                                                uint32_t stream_id, const float* alpha_in,
                                                const nvfp4_qtensor_t* out, void* stream);

/* Decode packed codes [R, C/2] with scales ([R, C/16]; BLOCK2D [R/16, C/16];
 * or the GEMM layout with NVFP4_GEMM_SCALE_LAYOUT) and the device tensor
 * scale *alpha:  y = q * (alpha * Delta)  (the inverse of Eq. 3), optionally
 * followed by the inverse rotation x = D (1/4) H16 y (NVFP4_INVERSE_RHT, key
 * `seed`).  y is fp32 [R, C], or bf16 with NVFP4_OUT_BF16 (rounded to
 * nearest even), row-major, contiguous. */
NVFP4_API nvfp4_status_t nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                                const float* alpha, int64_t R, int64_t C,
                                uint32_t flags, uint64_t seed, void* y,
                                void* stream);

/* Block-scaled NVFP4 GEMM on the tcgen05 tensor cores ([NV] §四):
 *     D[m, n] = alphaA * alphaB * sum_k (qA[m,k] DeltaA[m,k/16]) (qB[n,k] DeltaB[n,k/16])
 * A: codes [M, K/2], B: codes [N, K/2] (both K-major, "TN"); sA, sB: scales
 * in the GEMM layout above (as written by nvfp4_quantize with
 * NVFP4_GEMM_SCALE_LAYOUT); alphaA, alphaB: device floats.  Products are
 * accumulated in FP32; D is bf16 (NVFP4_OUT_DTYPE_BF16) or fp32, row-major
 * with row stride ldd elements.  M % 128 == 0, N % 128 == 0, K % 128 == 0;
 * A, B, sA, sB, D 16-byte aligned.  The GEMM needs no scratch memory: the
 * workspace is optional (NULL, 0); when given (>= 4 bytes) its first int32 is
 * used as the sticky device status word (NVFP4_ERR_TIMEOUT if a bounded
 * pipeline wait gave up). */
NVFP4_API nvfp4_status_t nvfp4_gemm(const uint8_t* A, const uint8_t* sA, const float* alphaA,
                          const uint8_t* B, const uint8_t* sB, const float* alphaB,
                          int64_t M, int64_t N, int64_t K, void* D, int out_dtype,
                          int64_t ldd, void* workspace, size_t workspace_bytes,
                          void* stream);

/* nvfp4_gemm for operands quantized with NVFP4_VECTOR_SCALES (one tensor
 * scale per operand row; [NV] §九, READING as at that flag):
 *     D[m, n] = alphaA[m] * alphaB[n] * sum_k (qA DeltaA)(qB DeltaB)
 * alphaA: device floats [M] (the alpha_row vector of A's quantization, or
 * alpha_col when A is a column-orientation output), alphaB: [N] likewise.
 * D = RN(RN(acc * alphaA[m]) * alphaB[n]) in FP32, then bf16 or fp32 as for
 * nvfp4_gemm.  M % 256 == 0, N % 256 == 0, K % 128 == 0; operands and D
 * 16-byte aligned.  The workspace is optional as for nvfp4_gemm. */
NVFP4_API nvfp4_status_t nvfp4_gemm_vector_scales(const uint8_t* A, const uint8_t* sA, const float* alphaA,
                                                  const uint8_t* B, const uint8_t* sB, const float* alphaB,
                                                  int64_t M, int64_t N, int64_t K, void* D, int out_dtype,
                                                  int64_t ldd, void* workspace, size_t workspace_bytes,
                                                  void* stream);

/* nvfp4_gemm whose epilogue also quantizes the output for the next layer
 * ([NV] §九 counts the separate amax and quantize passes over an activation
 * as overhead; here the output is encoded while it is still in registers):
 *   D_bf16 = the bf16 result nvfp4_gemm would write (same arithmetic);
 *   codes [M, N/2], scales: exactly what
 *     nvfp4_quantize(D_bf16, mode, NVFP4_ROWWISE | NVFP4_ALPHA_PROVIDED | flags,
 *                    alpha_in = alpha_out)
 *     writes (16-element blocks along N; mode NVFP4_RTN or NVFP4_FOUR_SIX;
 *     flags: 0 or NVFP4_GEMM_SCALE_LAYOUT, the scales then [M, N/16] row-major
 *     or in the GEMM layout);
 *   amax_out (optional device float): max |D_bf16| over the whole output,
 *     from which a caller forms the next call's tensor scale amax / 2688
 *     (delayed scaling: the pages' Eq. 1 applied one step late);
 *   D (optional, bf16, row stride ldd): written only when not NULL.
 * alpha_out is a device float (the tensor scale of Eq. 1 for this output).
 * M % 256 == 0, N % 256 == 0, K % 128 == 0; pointers 16-byte aligned.  The
 * workspace is optional as for nvfp4_gemm (status word). */
NVFP4_API nvfp4_status_t nvfp4_gemm_quantize(const uint8_t* A, const uint8_t* sA, const float* alphaA,
                                   const uint8_t* B, const uint8_t* sB, const float* alphaB,
                                   int64_t M, int64_t N, int64_t K, void* D, int64_t ldd,
                                   nvfp4_mode_t mode, uint32_t flags, const float* alpha_out,
                                   uint8_t* codes, uint8_t* scales, float* amax_out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * MXFP4 ([NV] §一 and §五 contrast it with NVFP4; the AMD MI355X write-up,
 * 01-02, trains in it with a fixed Hadamard rotation).  Blocks of 32
 * consecutive elements, one power-of-two scale per block stored as a UE8M0
 * byte (2^(byte - 127)), E2M1 values, no tensor scale.
 *
 * READING (the pages give the format, not how the scale is chosen): the
 * OCP microscaling rule.  Per block e = floor(log2(max |v|)) - 2 (2 being
 * the largest E2M1 exponent), clamped to [-127, 127]; an all-zero block has
 * e = -127.  The stored byte is e + 127 and q_i = E2M1(v_i / 2^e) rounded to
 * nearest even, saturating at +-6 (a block maximum in [6, 8) 2^e clips).
 * ------------------------------------------------------------------------ */

/* Quantize the bf16 tensor x [R, C] (row stride ld) to MXFP4 in one read.
 *   flags: NVFP4_ROWWISE and / or NVFP4_COLWISE, optionally NVFP4_RHT (each
 *     16-element half of a block is first rotated by (1/4) H16 D, D the sign
 *     diagonal drawn from `seed` exactly as for nvfp4_quantize; a fixed seed
 *     gives the fixed rotation) and NVFP4_GEMM_SCALE_LAYOUT (scales written
 *     in the GEMM layout described at NVFP4_GEMM_SCALE_LAYOUT, with K-blocks
 *     of 32 elements: one 512-byte atom per 128 rows x 128 K; R % 128 == 0
 *     and C % 128 == 0).
 *   rowwise: codes_row [R, C/2] (element 2j in the low nibble), scales_row
 *     [R, C/32] row-major.  columnwise (blocks of 32 rows of a column, stored
 *     transposed): codes_col [C, R/2], scales_col [C, R/32].
 *   status (optional device int32, sticky): NVFP4_ERR_NONFINITE when the
 *     input holds an Inf or a NaN (the outputs are then unspecified).
 * All pointers are device memory owned by the caller.  Shapes: C % 32 == 0
 * (rowwise), R % 32 == 0 (columnwise), C % 16 == 0, ld >= C, ld % 8 == 0;
 * x and the code buffers 16-byte aligned.  No workspace.  Asynchronous on
 * `stream` (a cudaStream_t, NULL = legacy default stream). */
NVFP4_API nvfp4_status_t mxfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags,
                                        uint64_t seed, uint8_t* codes_row, uint8_t* scales_row,
                                        uint8_t* codes_col, uint8_t* scales_col, int32_t* status,
                                        void* stream);

/* Block-scaled MXFP4 GEMM on the tcgen05 tensor cores:
 *     D[m, n] = sum_k (qA[m,k] 2^eA[m,k/32]) (qB[n,k] 2^eB[n,k/32])
 * A: codes [M, K/2], B: codes [N, K/2] (K-major, "TN"); sA, sB: UE8M0 scales
 * in the GEMM layout (mxfp4_quantize with NVFP4_GEMM_SCALE_LAYOUT).  No
 * tensor scales.  FP32 accumulation; D bf16 (NVFP4_OUT_DTYPE_BF16) or fp32,
 * row-major with row stride ldd elements.  M % 256 == 0, N % 256 == 0,
 * K % 128 == 0 (the CTA-pair kernel); A, B, sA, sB, D 16-byte aligned.  The
 * workspace is optional as for nvfp4_gemm (status word). */
NVFP4_API nvfp4_status_t mxfp4_gemm(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB,
                                    int64_t M, int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Decode MXFP4 codes [R, C/2] with scales [R, C/32]:  y = q * 2^(byte - 127),
 * optionally followed by the inverse rotation D (1/4) H16 of each 16-element
 * half (NVFP4_INVERSE_RHT, key `seed`).  y is fp32 [R, C], or bf16 with
 * NVFP4_OUT_BF16 (rounded to nearest even), row-major, contiguous.
 * C % 32 == 0; codes 8-byte and y 16-byte aligned. */
NVFP4_API nvfp4_status_t mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C,
                                          uint32_t flags, uint64_t seed, void* y, void* stream);

/* Number of kernels this library has launched in the calling process since
 * it was loaded (all devices, all streams).  Instrumentation for callers that
 * account for their launches; not a page-defined operation. */
NVFP4_API uint64_t nvfp4_launch_count(void);

/* Static description of a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status_t status);

/* Library version, major * 10000 + minor * 100 + patch. */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
