// nvfp4_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

#include "nvfp4.h"

namespace nvfp4 {

constexpr int kModeRTN = NVFP4_RTN;
constexpr int kModeFourSix = NVFP4_FOUR_SIX;
constexpr int kModeRhtSR = NVFP4_RHT_SR;
constexpr int kModeMsEden = NVFP4_MS_EDEN;
constexpr int kModeRhtSRHw = NVFP4_RHT_SR_HW;

constexpr uint32_t kRowwise = NVFP4_ROWWISE;
constexpr uint32_t kColwise = NVFP4_COLWISE;
constexpr uint32_t kBlock2D = NVFP4_BLOCK2D;
constexpr uint32_t kSinglePass = NVFP4_SINGLE_PASS;
constexpr uint32_t kHeadroom = NVFP4_HEADROOM;
constexpr uint32_t kVectorScales = NVFP4_VECTOR_SCALES;
constexpr uint32_t kAlphaProvided = NVFP4_ALPHA_PROVIDED;
constexpr uint32_t kAmaxProvided = NVFP4_AMAX_PROVIDED;
constexpr uint32_t kGemmScaleLayout = NVFP4_GEMM_SCALE_LAYOUT;
constexpr uint32_t kRht = NVFP4_RHT;
constexpr uint32_t kInverseRht = NVFP4_INVERSE_RHT;
constexpr uint32_t kOutBf16 = NVFP4_OUT_BF16;

constexpr int32_t kStatusArg = NVFP4_ERR_ARG;
constexpr int32_t kStatusNonFinite = NVFP4_ERR_NONFINITE;
constexpr int32_t kStatusTimeout = NVFP4_ERR_TIMEOUT;

struct QuantOutputs {
  uint8_t* codes_row;
  uint8_t* scales_row;
  float* alpha_row;
  uint8_t* codes_col;
  uint8_t* scales_col;
  float* alpha_col;
  float* amax_out;
  int32_t* status;
};

int sm_count();
void note_launch(int n = 1);  // count kernels launched by the library
size_t quant_workspace_bytes(int64_t R, int64_t C, uint32_t flags);

// Host-side checks of nvfp4_quantize's arguments, the workspace excepted.
// NVFP4_OK with *empty set when the tensor has no elements (nothing to do).
nvfp4_status_t check_quantize_args(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode_t mode,
                                   uint32_t flags, uint32_t stream_id, const float* alpha_in,
                                   const nvfp4_qtensor_t* out, bool* empty);

cudaError_t quantize_launch(const void* x, int64_t R, int64_t C, int64_t ld, int mode,
                            uint32_t flags, uint64_t seed, uint32_t stream_id,
                            const float* alpha_in, const QuantOutputs& out, void* workspace,
                            cudaStream_t st);

// nvfp4_amax (quantize.cu): amax_out[0..2] = plain, rotated rows, rotated columns.
cudaError_t amax_launch(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                        float* amax_out, int32_t* status, cudaStream_t st);

cudaError_t dequantize_launch(const uint8_t* codes, const uint8_t* scales, const float* alpha,
                              int64_t R, int64_t C, uint32_t flags, uint64_t seed, void* y,
                              cudaStream_t st);

cudaError_t gemm_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                        const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K,
                        void* D, int out_dtype, int64_t ldd, int32_t* status, cudaStream_t st);

// NVFP4 GEMM whose epilogue also quantizes the bf16 output rowwise (RTN or
// FOUR_SIX, tensor scale *alpha_out): codes [M, N/2], scales (row-major or
// GEMM layout), optional max |D| (amax_out, float).  D may be null.
// Requires M % 256 == 0 and N % 256 == 0 (the CTA-pair kernel).
cudaError_t gemm_quantize_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                                 const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K, void* D,
                                 int64_t ldd, int mode, bool gemm_layout, const float* alpha_out, uint8_t* codes,
                                 uint8_t* scales, float* amax_out, int32_t* status, cudaStream_t st);

// NVFP4 GEMM with one tensor scale per operand row: alphaA [M], alphaB [N]
// (the CTA-pair kernel; M % 256 == 0, N % 256 == 0, K % 128 == 0).
cudaError_t gemm_vs_launch(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                           const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K, void* D,
                           int out_dtype, int64_t ldd, int32_t* status, cudaStream_t st);

// MXFP4 GEMM (gemm.cu, the CTA-pair kernel with UE8M0 block-32 scales):
// D = sum_k (qA 2^eA)(qB 2^eB), scales in the GEMM layout with one 512-byte
// atom per 128 rows x 128 K.  M % 256 == 0, N % 256 == 0, K % 128 == 0.
cudaError_t mx_gemm_launch(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB, int64_t M,
                           int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd, int32_t* status, cudaStream_t st);

// MXFP4 (mx.cu): one tile kernel for rows and / or columns; dequantization.
cudaError_t mx_quantize_launch(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                               uint8_t* codes_row, uint8_t* scales_row, uint8_t* codes_col, uint8_t* scales_col,
                               int32_t* status, cudaStream_t st);
cudaError_t mx_dequantize_launch(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C, uint32_t flags,
                                 uint64_t seed, void* y, cudaStream_t st);

}  // namespace nvfp4
