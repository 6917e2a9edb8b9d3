// api.cu -- the C ABI of libnvfp4.so: argument checks, workspace sizing and
// dispatch.  Host-detectable errors return before anything is launched.
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "nvfp4.h"
#include "nvfp4_internal.h"

namespace {

constexpr uint32_t kQuantFlags = NVFP4_ROWWISE | NVFP4_COLWISE | NVFP4_BLOCK2D | NVFP4_SINGLE_PASS | NVFP4_HEADROOM |
                                 NVFP4_ALPHA_PROVIDED | NVFP4_GEMM_SCALE_LAYOUT | NVFP4_RHT | NVFP4_VECTOR_SCALES |
                                 NVFP4_AMAX_PROVIDED;
constexpr uint32_t kDequantFlags = NVFP4_BLOCK2D | NVFP4_GEMM_SCALE_LAYOUT | NVFP4_INVERSE_RHT | NVFP4_OUT_BF16;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

nvfp4_status_t launch_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  return (e == cudaErrorInvalidConfiguration || e == cudaErrorLaunchOutOfResources ||
          e == cudaErrorInvalidDeviceFunction || e == cudaErrorNoKernelImageForDevice ||
          e == cudaErrorCooperativeLaunchTooLarge)
             ? NVFP4_ERR_LAUNCH
             : NVFP4_ERR_CUDA;
}

std::atomic<uint64_t> g_launches{0};

}  // namespace

namespace nvfp4 {
void note_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

nvfp4_status_t check_quantize_args(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode_t mode,
                                   uint32_t flags, uint32_t stream_id, const float* alpha_in,
                                   const nvfp4_qtensor_t* out, bool* empty) {
  *empty = false;
  if (!out) return NVFP4_ERR_ARG;
  if (static_cast<int>(mode) < NVFP4_RTN || static_cast<int>(mode) > NVFP4_RHT_SR_HW) return NVFP4_ERR_ARG;
  if (flags & ~kQuantFlags) return NVFP4_ERR_ARG;
  const bool row = flags & NVFP4_ROWWISE, col = flags & NVFP4_COLWISE, two_d = flags & NVFP4_BLOCK2D;
  const bool gemm = flags & NVFP4_GEMM_SCALE_LAYOUT;
  if (!row && !col) return NVFP4_ERR_ARG;
  if (two_d && (mode == NVFP4_RHT_SR || mode == NVFP4_MS_EDEN || mode == NVFP4_RHT_SR_HW || (flags & NVFP4_RHT)))
    return NVFP4_ERR_ARG;
  if (stream_id >= 0x80000000u) return NVFP4_ERR_ARG;
  if ((flags & NVFP4_VECTOR_SCALES) && (flags & (NVFP4_BLOCK2D | NVFP4_SINGLE_PASS | NVFP4_ALPHA_PROVIDED)))
    return NVFP4_ERR_ARG;
  if ((flags & NVFP4_AMAX_PROVIDED) &&
      (flags & (NVFP4_ALPHA_PROVIDED | NVFP4_SINGLE_PASS | NVFP4_VECTOR_SCALES)))
    return NVFP4_ERR_ARG;
  if (R < 0 || C < 0 || ld < C) return NVFP4_ERR_SHAPE;
  if (C % 16) return NVFP4_ERR_SHAPE;
  if ((col || two_d) && R % 16) return NVFP4_ERR_SHAPE;
  if (R * (C / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (gemm) {
    if (row && (R % 128 || C % 64)) return NVFP4_ERR_SHAPE;
    if (col && (C % 128 || R % 64)) return NVFP4_ERR_SHAPE;
  }
  if (R == 0 || C == 0) {  // empty tensor: nothing to write
    *empty = true;
    return NVFP4_OK;
  }
  if ((flags & (NVFP4_ALPHA_PROVIDED | NVFP4_AMAX_PROVIDED)) && !alpha_in) return NVFP4_ERR_ARG;
  if ((flags & NVFP4_AMAX_PROVIDED) && !aligned(alpha_in, 4)) return NVFP4_ERR_ALIGN;
  if (row && (!out->codes_row || !out->scales_row || !out->alpha_row)) return NVFP4_ERR_ARG;
  if (col && (!out->codes_col || !out->scales_col || !out->alpha_col)) return NVFP4_ERR_ARG;
  if (!x) return NVFP4_ERR_ARG;
  if (!aligned(x, 16) || ld % 8) return NVFP4_ERR_ALIGN;
  if (row && !aligned(out->codes_row, 16)) return NVFP4_ERR_ALIGN;
  if (col && !aligned(out->codes_col, 16)) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}
}  // namespace nvfp4

extern "C" {

uint64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

nvfp4_status_t nvfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                          float* amax_out, int32_t* status, void* stream) {
  if (flags & ~(NVFP4_ROWWISE | NVFP4_COLWISE | NVFP4_RHT)) return NVFP4_ERR_ARG;
  if (!amax_out) return NVFP4_ERR_ARG;
  if (R < 0 || C < 0 || ld < C || C % 16) return NVFP4_ERR_SHAPE;
  if ((flags & NVFP4_RHT) && (flags & NVFP4_COLWISE) && R % 16) return NVFP4_ERR_SHAPE;
  if (R * (C / 8) >= (int64_t(1) << 32)) return NVFP4_ERR_SHAPE;
  if (!aligned(amax_out, 4) || (status && !aligned(status, 4))) return NVFP4_ERR_ALIGN;
  if (R > 0 && C > 0) {
    if (!x) return NVFP4_ERR_ARG;
    if (!aligned(x, 16) || ld % 8) return NVFP4_ERR_ALIGN;
  }
  return launch_status(nvfp4::amax_launch(x, R, C, ld, flags, seed, amax_out, status,
                                          static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t mxfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                              uint8_t* codes_row, uint8_t* scales_row, uint8_t* codes_col, uint8_t* scales_col,
                              int32_t* status, void* stream) {
  if (flags & ~(NVFP4_ROWWISE | NVFP4_COLWISE | NVFP4_RHT | NVFP4_GEMM_SCALE_LAYOUT)) return NVFP4_ERR_ARG;
  const bool row = flags & NVFP4_ROWWISE, col = flags & NVFP4_COLWISE;
  if (!row && !col) return NVFP4_ERR_ARG;
  if (R < 0 || C < 0 || ld < C) return NVFP4_ERR_SHAPE;
  if (C % 16 || (row && C % 32) || (col && R % 32)) return NVFP4_ERR_SHAPE;
  if ((flags & NVFP4_GEMM_SCALE_LAYOUT) && (R % 128 || C % 128)) return NVFP4_ERR_SHAPE;
  if (R * (C / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (R == 0 || C == 0) return NVFP4_OK;
  if (!x || (row && (!codes_row || !scales_row)) || (col && (!codes_col || !scales_col))) return NVFP4_ERR_ARG;
  if (!aligned(x, 16) || ld % 8) return NVFP4_ERR_ALIGN;
  if ((row && !aligned(codes_row, 16)) || (col && !aligned(codes_col, 16))) return NVFP4_ERR_ALIGN;
  return launch_status(nvfp4::mx_quantize_launch(x, R, C, ld, flags, seed, row ? codes_row : nullptr,
                                                 row ? scales_row : nullptr, col ? codes_col : nullptr,
                                                 col ? scales_col : nullptr, status,
                                                 static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t mxfp4_gemm(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB, int64_t M,
                          int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (out_dtype != NVFP4_OUT_DTYPE_BF16 && out_dtype != NVFP4_OUT_DTYPE_FP32) return NVFP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return NVFP4_ERR_SHAPE;
  if (M % 256 || N % 256 || K % 128 || ldd < N) return NVFP4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (!A || !sA || !B || !sB || !D) return NVFP4_ERR_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sA, 16) || !aligned(sB, 16) || !aligned(D, 16))
    return NVFP4_ERR_ALIGN;
  if ((ldd * (out_dtype == NVFP4_OUT_DTYPE_BF16 ? 2 : 4)) % 16) return NVFP4_ERR_ALIGN;
  int32_t* status = (workspace && workspace_bytes >= sizeof(int32_t) && aligned(workspace, 4))
                        ? static_cast<int32_t*>(workspace)
                        : nullptr;
  return launch_status(nvfp4::mx_gemm_launch(A, sA, B, sB, M, N, K, D, out_dtype, ldd, status,
                                             static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C, uint32_t flags,
                                uint64_t seed, void* y, void* stream) {
  if (flags & ~(NVFP4_INVERSE_RHT | NVFP4_OUT_BF16)) return NVFP4_ERR_ARG;
  if (R < 0 || C < 0 || C % 32) return NVFP4_ERR_SHAPE;
  if (R * (C / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (R == 0 || C == 0) return NVFP4_OK;
  if (!codes || !scales || !y) return NVFP4_ERR_ARG;
  if (!aligned(codes, 8) || !aligned(y, 16)) return NVFP4_ERR_ALIGN;
  return launch_status(nvfp4::mx_dequantize_launch(codes, scales, R, C, flags, seed, y,
                                                   static_cast<cudaStream_t>(stream)));
}

int nvfp4_version(void) { return 10000; }

const char* nvfp4_status_string(nvfp4_status_t s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_ARG: return "invalid argument (mode, flags or null pointer)";
    case NVFP4_ERR_SHAPE: return "shape breaks the block or tile rules";
    case NVFP4_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case NVFP4_ERR_NONFINITE: return "input holds a NaN or an infinity";
    case NVFP4_ERR_LAUNCH: return "kernel launch failed";
    case NVFP4_ERR_TIMEOUT: return "a bounded device wait gave up";
    case NVFP4_ERR_CUDA: return "CUDA runtime error";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

size_t nvfp4_workspace_size(int64_t R, int64_t C, uint32_t flags) {
  return nvfp4::quant_workspace_bytes(R, C, flags);
}

nvfp4_status_t nvfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode_t mode,
                              uint32_t flags, uint64_t seed, uint32_t stream_id,
                              const float* alpha_in, const nvfp4_qtensor_t* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  bool empty = false;
  const nvfp4_status_t chk = nvfp4::check_quantize_args(x, R, C, ld, mode, flags, stream_id, alpha_in, out, &empty);
  if (chk != NVFP4_OK || empty) return chk;
  const bool row = flags & NVFP4_ROWWISE, col = flags & NVFP4_COLWISE;
  const size_t need = nvfp4::quant_workspace_bytes(R, C, flags);
  if (need && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return NVFP4_ERR_WORKSPACE;
  nvfp4::QuantOutputs o{out->codes_row, out->scales_row, out->alpha_row, out->codes_col,
                        out->scales_col, out->alpha_col, out->amax_out, out->status};
  if (!row) o.codes_row = nullptr, o.scales_row = nullptr, o.alpha_row = nullptr;
  if (!col) o.codes_col = nullptr, o.scales_col = nullptr, o.alpha_col = nullptr;
  return launch_status(nvfp4::quantize_launch(x, R, C, ld, static_cast<int>(mode), flags, seed, stream_id,
                                              alpha_in, o, workspace, static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* alpha,
                                int64_t R, int64_t C, uint32_t flags, uint64_t seed, void* y,
                                void* stream) {
  if (flags & ~kDequantFlags) return NVFP4_ERR_ARG;
  const bool two_d = flags & NVFP4_BLOCK2D, gemm = flags & NVFP4_GEMM_SCALE_LAYOUT;
  if (two_d && (flags & NVFP4_INVERSE_RHT)) return NVFP4_ERR_ARG;
  if (two_d && gemm) return NVFP4_ERR_ARG;
  if (R < 0 || C < 0 || C % 16) return NVFP4_ERR_SHAPE;
  if (two_d && R % 16) return NVFP4_ERR_SHAPE;
  if (gemm && (R % 128 || C % 64)) return NVFP4_ERR_SHAPE;
  if (R * (C / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (R == 0 || C == 0) return NVFP4_OK;
  if (!codes || !scales || !alpha || !y) return NVFP4_ERR_ARG;
  if (!aligned(codes, 8) || !aligned(y, 16)) return NVFP4_ERR_ALIGN;
  return launch_status(nvfp4::dequantize_launch(codes, scales, alpha, R, C, flags, seed, y,
                                                static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t nvfp4_gemm(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                          const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K,
                          void* D, int out_dtype, int64_t ldd, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (out_dtype != NVFP4_OUT_DTYPE_BF16 && out_dtype != NVFP4_OUT_DTYPE_FP32) return NVFP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return NVFP4_ERR_SHAPE;
  if (M % 128 || N % 128 || K % 128 || ldd < N) return NVFP4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (!A || !sA || !alphaA || !B || !sB || !alphaB || !D) return NVFP4_ERR_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sA, 16) || !aligned(sB, 16) || !aligned(D, 16))
    return NVFP4_ERR_ALIGN;
  if ((ldd * (out_dtype == NVFP4_OUT_DTYPE_BF16 ? 2 : 4)) % 16) return NVFP4_ERR_ALIGN;
  int32_t* status = (workspace && workspace_bytes >= sizeof(int32_t) && aligned(workspace, 4))
                        ? static_cast<int32_t*>(workspace)
                        : nullptr;
  return launch_status(nvfp4::gemm_launch(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status,
                                          static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t nvfp4_gemm_vector_scales(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                                        const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K,
                                        void* D, int out_dtype, int64_t ldd, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  if (out_dtype != NVFP4_OUT_DTYPE_BF16 && out_dtype != NVFP4_OUT_DTYPE_FP32) return NVFP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return NVFP4_ERR_SHAPE;
  if (M % 256 || N % 256 || K % 128 || ldd < N) return NVFP4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (!A || !sA || !alphaA || !B || !sB || !alphaB || !D) return NVFP4_ERR_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sA, 16) || !aligned(sB, 16) || !aligned(D, 16))
    return NVFP4_ERR_ALIGN;
  if (!aligned(alphaA, 4) || !aligned(alphaB, 4)) return NVFP4_ERR_ALIGN;
  if ((ldd * (out_dtype == NVFP4_OUT_DTYPE_BF16 ? 2 : 4)) % 16) return NVFP4_ERR_ALIGN;
  int32_t* status = (workspace && workspace_bytes >= sizeof(int32_t) && aligned(workspace, 4))
                        ? static_cast<int32_t*>(workspace)
                        : nullptr;
  return launch_status(nvfp4::gemm_vs_launch(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, status,
                                             static_cast<cudaStream_t>(stream)));
}

nvfp4_status_t nvfp4_gemm_quantize(const uint8_t* A, const uint8_t* sA, const float* alphaA, const uint8_t* B,
                                   const uint8_t* sB, const float* alphaB, int64_t M, int64_t N, int64_t K, void* D,
                                   int64_t ldd, nvfp4_mode_t mode, uint32_t flags, const float* alpha_out,
                                   uint8_t* codes, uint8_t* scales, float* amax_out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (mode != NVFP4_RTN && mode != NVFP4_FOUR_SIX) return NVFP4_ERR_ARG;
  if (flags & ~NVFP4_GEMM_SCALE_LAYOUT) return NVFP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return NVFP4_ERR_SHAPE;
  if (M % 256 || N % 256 || K % 128) return NVFP4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (M * (N / 16) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
  if (D && ldd < N) return NVFP4_ERR_SHAPE;
  if (!A || !sA || !alphaA || !B || !sB || !alphaB || !alpha_out || !codes || !scales) return NVFP4_ERR_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sA, 16) || !aligned(sB, 16) || !aligned(codes, 16))
    return NVFP4_ERR_ALIGN;
  if (D && (!aligned(D, 16) || (ldd * 2) % 16)) return NVFP4_ERR_ALIGN;
  if (amax_out && !aligned(amax_out, 4)) return NVFP4_ERR_ALIGN;
  int32_t* status = (workspace && workspace_bytes >= sizeof(int32_t) && aligned(workspace, 4))
                        ? static_cast<int32_t*>(workspace)
                        : nullptr;
  return launch_status(nvfp4::gemm_quantize_launch(A, sA, alphaA, B, sB, alphaB, M, N, K, D, ldd,
                                                   static_cast<int>(mode), (flags & NVFP4_GEMM_SCALE_LAYOUT) != 0,
                                                   alpha_out, codes, scales, amax_out, status,
                                                   static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
