// mx.cu -- MXFP4 quantization and dequantization kernels for sm_100a.
//
// MXFP4 (NVFP4 pretraining write-up §一 and §五; AMD MI355X write-up 01-02):
// blocks of 32 consecutive elements, one power-of-two scale per block stored
// as a UE8M0 byte, E2M1 values, no tensor scale.  The scale exponent is
// e = floor(log2(max |v|)) - 2 (2 = the largest E2M1 exponent), clamped to
// [-127, 127], -127 for an all-zero block; values are q = E2M1-RNE(v / 2^e)
// saturating at 6.  Dividing by a power of two is exact, so v / 2^e is
// v * 2^-e with one exact multiply (a result that underflows is far below
// the first rounding threshold 0.25 and encodes to zero either way).
//
// No tensor-wide pass: one read of the bf16 tensor produces the codes of
// both orientations.  The tensor streams through 64 x 128 tiles in a
// two-buffer cp.async ring (tile.cuh); per tile, thread t takes row block
// (t / 4, t % 4) and column block (t / 2, t % 2), the two 16-element halves
// of a block lane-paired in float2 registers.  With NVFP4_RHT each half is
// first rotated by (1/4) H16 D, D the seeded sign diagonal of the NVFP4 path
// (a fixed seed gives a fixed rotation).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>

#include "nvfp4_device.cuh"
#include "launch.cuh"
#include "nvfp4_internal.h"
#include "tile.cuh"

namespace nvfp4 {

struct MxArgs {
  const uint16_t* x;
  int64_t R, C, ld;
  uint64_t seed;
  uint8_t* codes_row;
  uint8_t* scales_row;
  uint8_t* codes_col;
  uint8_t* scales_col;
  int32_t* status;
  int gemm;                       // scales in the tcgen05 block-scale layout
  int64_t tiles_c;
  FastDiv tiles_c_div;
  uint32_t ntiles;
};

// Shared exponent from the block maximum m (non-negative, finite): for a
// normal m with biased exponent E, floor(log2 m) = E - 127, so e = E - 129;
// zero, subnormal and E = 1 maxima clamp to -127.
__device__ __forceinline__ int mx_exponent(float m) {
  const int E = static_cast<int>(__float_as_uint(m) >> 23);
  return max(E - 129, -127);
}

// 2^-e for e in [-127, 125] (a normal float: biased exponent 127 - e in [2, 254]).
__device__ __forceinline__ float mx_inv_scale(int e) { return __uint_as_float(static_cast<uint32_t>(127 - e) << 23); }

// 2^e for e in [-127, 127]; 2^-127 is subnormal.
__device__ __forceinline__ float mx_scale(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Encode one 32-block held as two lane-paired 16-halves (x: elements 0..15,
// y: 16..31), rotating first when ROT.  Returns the 16 code bytes and the
// scale byte.
template <bool ROT>
__device__ __forceinline__ uint4 mx_encode(float2* v, uint32_t& scale) {
  if constexpr (ROT) rht16x2_presigned(v);
  float ma, mb;
  max_abs16x2(v, ma, mb);
  const float m = fmaxf(ma, mb);
  const int e = mx_exponent(m);
  scale = static_cast<uint32_t>(e + 127);
  const float inv = mx_inv_scale(e);
  const float2 i2 = make_float2(inv, inv);
  float2 y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = mul2(v[i], i2);
  uint4 c;
  c.x = e2m1x8_rne(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x);
  c.y = e2m1x8_rne(y[8].x, y[9].x, y[10].x, y[11].x, y[12].x, y[13].x, y[14].x, y[15].x);
  c.z = e2m1x8_rne(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y);
  c.w = e2m1x8_rne(y[8].y, y[9].y, y[10].y, y[11].y, y[12].y, y[13].y, y[14].y, y[15].y);
  return c;
}

template <bool ROT, bool ROW, bool COL>
__global__ void __launch_bounds__(TNT, 3) mx_tile_kernel(const MxArgs a) {
  pdl_entry();
  extern __shared__ __align__(128) uint8_t mx_ring[];
  auto tiles = reinterpret_cast<uint4(*)[TR][TC / 8]>(mx_ring);
  SignMasks sm;
  if constexpr (ROT) {
    sm = sign_masks(philox(philox_keys(a.seed), 0u, 0u, 0u, kTagSigns).x & 0xFFFFu);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) sm.m[i] = 0u;
  }
  const int t = threadIdx.x;
  const int64_t R = a.R, C = a.C;
  uint32_t hin = 0;   // per-halfword max of the input magnitudes (Inf / NaN check)
  uint32_t tile = blockIdx.x;
  if (tile < a.ntiles) load_tile_async(tiles[0], a.x, R, C, a.ld, a.tiles_c_div, tile);
  else cp_async_commit();
  for (int buf = 0; tile < a.ntiles; tile += gridDim.x, buf ^= 1) {
    const uint32_t next = tile + gridDim.x;
    if (next < a.ntiles) load_tile_async(tiles[buf ^ 1], a.x, R, C, a.ld, a.tiles_c_div, next);
    else cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint4 (*s)[TC / 8] = tiles[buf];
    int64_t tr, tc;
    tile_coords(tile, a.tiles_c_div, tr, tc);
    const int64_t r0 = tr * TR, c0 = tc * TC;
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);

    if constexpr (ROW) {
      const int row = t >> 2, cb = t & 3;
      if (row < rows && 32 * cb < cols) {
        const uint4 u0 = s[row][tile_chunk(row, 4 * cb)], u1 = s[row][tile_chunk(row, 4 * cb + 1)];
        const uint4 u2 = s[row][tile_chunk(row, 4 * cb + 2)], u3 = s[row][tile_chunk(row, 4 * cb + 3)];
        const uint32_t w[16] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w,
                                u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
#pragma unroll
        for (int i = 0; i < 16; ++i) hin = __vmaxu2(hin, w[i] & 0x7FFF7FFFu);
        float2 v[16];
        unpack16x2_signed(u0, u1, u2, u3, sm, v);
        uint32_t sc;
        const uint4 c = mx_encode<ROT>(v, sc);
        const int64_t gr = r0 + row;
        *reinterpret_cast<uint4*>(a.codes_row + gr * (C / 2) + (c0 + 32 * cb) / 2) = c;
        const int64_t j = c0 / 32 + cb;
        a.scales_row[a.gemm ? gemm_scale_offset(gr, j, C / 32) : gr * (C / 32) + j] = static_cast<uint8_t>(sc);
      }
    }
    if constexpr (COL) {
      const int c = t >> 1, h = t & 1;
      if (c < cols && 32 * h < rows) {
        const int hi = c & 1;
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int ra = 32 * h + i, rb = ra + 16;
          const uint32_t wa = reinterpret_cast<const uint32_t*>(&s[ra][0])[tile_word(ra, c >> 1)];
          const uint32_t wb = reinterpret_cast<const uint32_t*>(&s[rb][0])[tile_word(rb, c >> 1)];
          hin = __vmaxu2(hin, wa & 0x7FFF7FFFu);   // the word's other column is in the tensor too
          hin = __vmaxu2(hin, wb & 0x7FFF7FFFu);
          const uint32_t ba = hi ? (wa & 0xFFFF0000u) : (wa << 16);
          const uint32_t bb = hi ? (wb & 0xFFFF0000u) : (wb << 16);
          v[i] = make_float2(__uint_as_float(ba ^ sm.m[i]), __uint_as_float(bb ^ sm.m[i]));
        }
        uint32_t sc;
        const uint4 q = mx_encode<ROT>(v, sc);
        const int64_t gc = c0 + c;
        *reinterpret_cast<uint4*>(a.codes_col + gc * (R / 2) + (r0 + 32 * h) / 2) = q;
        const int64_t j = r0 / 32 + h;
        a.scales_col[a.gemm ? gemm_scale_offset(gc, j, R / 32) : gc * (R / 32) + j] = static_cast<uint8_t>(sc);
      }
    }
    __syncthreads();   // the buffer is refilled by the next iteration's copies
  }
  cp_async_wait<0>();
  if (max(hin & 0xFFFFu, hin >> 16) >= 0x7F80u && a.status) *a.status = kStatusNonFinite;
}

// Dequantize: thread per 16-element half block; y = q 2^e, then with INV the
// inverse rotation D (1/4) H16.
template <bool INV, bool BF16>
__global__ void __launch_bounds__(256) mx_dequant_kernel(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales, int64_t R, int64_t C,
                                                         uint64_t seed, void* __restrict__ y) {
  pdl_entry();
  const int64_t halves = R * (C / 16);
  const uint32_t signs = INV ? (philox(philox_keys(seed), 0u, 0u, 0u, kTagSigns).x & 0xFFFFu) : 0u;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < halves;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = k / (C / 16), hb = k - r * (C / 16);
    const uint2 w = *reinterpret_cast<const uint2*>(codes + r * (C / 2) + 8 * hb);
    const float s = mx_scale(static_cast<int>(scales[r * (C / 32) + hb / 2]) - 127);
    float v[16];
    e2m1x8_values(w.x, v);
    e2m1x8_values(w.y, v + 8);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], s);
    if constexpr (INV) irht16(v, signs);
    if constexpr (BF16) {
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        o[i] = *reinterpret_cast<const uint32_t*>(&p);
      }
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + r * C + 16 * hb);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + r * C + 16 * hb);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
}

template <bool ROT, bool ROW, bool COL>
static cudaError_t launch_mx_tile(const MxArgs& a, cudaStream_t st) {
  const int smem = 2 * TR * TC * 2;   // 32 KB: within the default dynamic shared-memory limit
  auto fn = mx_tile_kernel<ROT, ROW, COL>;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, TNT, smem) != cudaSuccess || n <= 0) n = 1;
  const int grid = static_cast<int>(std::min<int64_t>(a.ntiles, static_cast<int64_t>(sm_count()) * n));
  launch_k(fn, dim3(grid), dim3(TNT), smem, st, 1u, a);
  note_launch();
  return cudaGetLastError();
}

template <bool ROT>
static cudaError_t dispatch_mx(const MxArgs& a, bool row, bool col, cudaStream_t st) {
  if (row && col) return launch_mx_tile<ROT, true, true>(a, st);
  if (row) return launch_mx_tile<ROT, true, false>(a, st);
  return launch_mx_tile<ROT, false, true>(a, st);
}

cudaError_t mx_quantize_launch(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                               uint8_t* codes_row, uint8_t* scales_row, uint8_t* codes_col, uint8_t* scales_col,
                               int32_t* status, cudaStream_t st) {
  MxArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.R = R;
  a.C = C;
  a.ld = ld;
  a.seed = seed;
  a.codes_row = codes_row;
  a.scales_row = scales_row;
  a.codes_col = codes_col;
  a.scales_col = scales_col;
  a.status = status;
  a.gemm = (flags & kGemmScaleLayout) ? 1 : 0;
  const int64_t tiles_r = (R + TR - 1) / TR;
  a.tiles_c = (C + TC - 1) / TC;
  a.tiles_c_div = make_fastdiv(static_cast<uint32_t>(a.tiles_c > 0 ? a.tiles_c : 1));
  a.ntiles = static_cast<uint32_t>(tiles_r * a.tiles_c);
  if (a.ntiles == 0) return cudaSuccess;
  const bool row = flags & kRowwise, col = flags & kColwise;
  return (flags & kRht) ? dispatch_mx<true>(a, row, col, st) : dispatch_mx<false>(a, row, col, st);
}

cudaError_t mx_dequantize_launch(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C, uint32_t flags,
                                 uint64_t seed, void* y, cudaStream_t st) {
  const int64_t halves = R * (C / 16);
  if (halves == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((halves + 255) / 256, static_cast<int64_t>(sm_count()) * 8));
  const bool inv = flags & kInverseRht, bf16 = flags & kOutBf16;
  if (inv && bf16) launch_k(mx_dequant_kernel<true, true>, dim3(blocks), dim3(256), 0, st, 1u, codes, scales, R, C, seed, y);
  else if (inv) launch_k(mx_dequant_kernel<true, false>, dim3(blocks), dim3(256), 0, st, 1u, codes, scales, R, C, seed, y);
  else if (bf16) launch_k(mx_dequant_kernel<false, true>, dim3(blocks), dim3(256), 0, st, 1u, codes, scales, R, C, seed, y);
  else launch_k(mx_dequant_kernel<false, false>, dim3(blocks), dim3(256), 0, st, 1u, codes, scales, R, C, seed, y);
  note_launch();
  return cudaGetLastError();
}

}  // namespace nvfp4
