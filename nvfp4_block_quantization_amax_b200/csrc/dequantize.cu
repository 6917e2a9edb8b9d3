// dequantize.cu -- decode NVFP4 codes back to fp32 / bf16 (the inverse of
// Eq. 3 of Four Over Six §2.1: x_hat = q * (alpha * Delta)), optionally
// undoing the 16-wide Hadamard rotation.  One thread per 16-element block;
// 8-byte code loads, 64-byte (fp32) or 32-byte (bf16) stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>

#include "nvfp4_device.cuh"
#include "launch.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

template <bool INV, bool BF16, int SCALES /*0 plain, 1 2D, 2 GEMM layout*/>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ codes,
                                                      const uint8_t* __restrict__ scales,
                                                      const float* __restrict__ alpha_p,
                                                      int64_t R, int64_t C, FastDiv nb,
                                                      uint64_t seed, void* __restrict__ y) {
  pdl_entry();
  const float alpha = __ldg(alpha_p);
  uint32_t signs = 0;
  if constexpr (INV) signs = philox(philox_keys(seed), 0u, 0u, 0u, kTagSigns).x & 0xFFFFu;
  const uint32_t total = static_cast<uint32_t>(R) * nb.d;
  for (uint32_t k = blockIdx.x * blockDim.x + threadIdx.x; k < total; k += gridDim.x * blockDim.x) {
    const uint32_t r = fastdiv(k, nb), cb = k - r * nb.d;
    int64_t so;
    if constexpr (SCALES == 0) so = k;
    else if constexpr (SCALES == 1) so = static_cast<int64_t>(r / 16) * nb.d + cb;
    else so = ((static_cast<int64_t>(r) >> 7) * (nb.d >> 2) + (cb >> 2)) * 512 + (r & 31) * 16 +
              ((r >> 5) & 3) * 4 + (cb & 3);
    const float s = __fmul_rn(alpha, e4m3_value(__ldg(scales + so)));
    const uint2 p = __ldg(reinterpret_cast<const uint2*>(codes + static_cast<int64_t>(r) * (C / 2) + 8 * cb));
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t b = ((j < 4) ? (p.x >> (8 * j)) : (p.y >> (8 * (j - 4)))) & 0xFFu;
      float q0, q1;
      e2m1x2_values(b, q0, q1);
      v[2 * j] = __fmul_rn(q0, s);
      v[2 * j + 1] = __fmul_rn(q1, s);
    }
    if constexpr (INV) irht16(v, signs);
    const int64_t off = static_cast<int64_t>(r) * C + 16 * cb;
    if constexpr (BF16) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j + 1]));
        w[j] = lo | (hi << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + off);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + off);
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
}

template <bool INV, bool BF16>
static void launch_dq(int sc, dim3 g, const uint8_t* codes, const uint8_t* scales, const float* alpha,
                      int64_t R, int64_t C, FastDiv nb, uint64_t seed, void* y, cudaStream_t st) {
  if (sc == 0) { launch_k(dequant_kernel<INV, BF16, 0>, dim3(g), dim3(256), 0, st, 1u, codes, scales, alpha, R, C, nb, seed, y); note_launch(); }
  else if (sc == 1) { launch_k(dequant_kernel<INV, BF16, 1>, dim3(g), dim3(256), 0, st, 1u, codes, scales, alpha, R, C, nb, seed, y); note_launch(); }
  else { launch_k(dequant_kernel<INV, BF16, 2>, dim3(g), dim3(256), 0, st, 1u, codes, scales, alpha, R, C, nb, seed, y); note_launch(); }
}

cudaError_t dequantize_launch(const uint8_t* codes, const uint8_t* scales, const float* alpha,
                              int64_t R, int64_t C, uint32_t flags, uint64_t seed, void* y,
                              cudaStream_t st) {
  if (R == 0 || C == 0) return cudaSuccess;
  const FastDiv nb = make_fastdiv(static_cast<uint32_t>(C / 16));
  const int64_t total = R * (C / 16);
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(sm_count()) * 8));
  const dim3 g(blocks > 0 ? blocks : 1);
  const int sc = (flags & kGemmScaleLayout) ? 2 : ((flags & kBlock2D) ? 1 : 0);
  const bool inv = flags & kInverseRht, bf = flags & kOutBf16;
  if (inv) {
    if (bf) launch_dq<true, true>(sc, g, codes, scales, alpha, R, C, nb, seed, y, st);
    else launch_dq<true, false>(sc, g, codes, scales, alpha, R, C, nb, seed, y, st);
  } else {
    if (bf) launch_dq<false, true>(sc, g, codes, scales, alpha, R, C, nb, seed, y, st);
    else launch_dq<false, false>(sc, g, codes, scales, alpha, R, C, nb, seed, y, st);
  }
  return cudaGetLastError();
}

}  // namespace nvfp4
