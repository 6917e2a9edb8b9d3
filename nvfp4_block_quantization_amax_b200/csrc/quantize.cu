// quantize.cu -- NVFP4 quantization kernels for sm_100a.
//
// Two-pass path (Four Over Six §2.1 Eq. 1 needs the tensor amax before any
// block can be scaled; the NVFP4 pretraining write-up §九 notes this extra
// pass over memory):
//   1. an amax kernel reads the bf16 tensor once and leaves one partial
//      maximum per CTA in the workspace (no atomics, no zero-fill needed);
//   2. a quantize kernel reduces those partials to amax and alpha in its
//      prologue, then encodes every block.
// Rowwise-only work streams straight from HBM into registers (128-bit loads,
// two consecutive 16-element blocks per thread).  Column, dual (row + column
// from one read) and 2D 16x16 work stream 64 x 128 tiles through a two-buffer
// cp.async ring in shared memory, swizzled so both orientations are read
// without bank conflicts; transposed outputs are written in full 32-byte
// sectors.  Every kernel holds two independent blocks per thread in float2
// registers and runs the element-wise steps with packed f32x2 instructions.
// Single pass (NVFP4_SINGLE_PASS): the amax and quantize bodies run in one
// cooperative launch separated by a bounded grid barrier.
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>
#include <cstdlib>

#include "nvfp4_device.cuh"
#include "launch.cuh"
#include "nvfp4_internal.h"
#include "tile.cuh"

namespace nvfp4 {

// ---------------------------------------------------------------------------
// Shared parameter block of the quantize kernels.
// ---------------------------------------------------------------------------
struct QuantArgs {
  const uint16_t* x;
  int64_t R, C, ld;
  uint64_t seed;
  uint32_t stream_id;
  uint32_t flags;
  const float* alpha_in;          // device, used with NVFP4_ALPHA_PROVIDED
  const uint32_t* partials;       // row-orientation maxima (float bits), one per amax CTA
  const uint32_t* partials_col;   // column-orientation maxima (== partials when not rotated)
  int npart;
  uint8_t* codes_row;
  uint8_t* scales_row;
  float* alpha_row;
  uint8_t* codes_col;
  uint8_t* scales_col;
  float* alpha_col;
  float* amax_out;
  int32_t* status;
  FastDiv nb_row;                 // C / 16
  int64_t tiles_r, tiles_c;       // tile grid (tile kernels)
  FastDiv tiles_c_div;            // divides a tile index by tiles_c
  FastDiv chunks_row;             // C / 8: 16-byte chunks per row (plain amax)
  uint32_t* vmax_r;               // NVFP4_VECTOR_SCALES: per-row maxima [R] (float bits)
  uint32_t* vmax_c;               // and per-column maxima [C]
  int amax_rot;                   // NVFP4_AMAX_PROVIDED: rotated (per-orientation amax values)
};

// Tensor scale of one vector from its maximum (Eq. 1 per vector; the
// headroom form with NVFP4_HEADROOM).
__device__ __forceinline__ float vector_alpha(const QuantArgs& a, const uint32_t* vmax, int64_t i) {
  const float den = (a.flags & kHeadroom) ? 1792.0f : 2688.0f;
  return __fdiv_rn(__uint_as_float(__ldcg(vmax + i)), den);
}

constexpr uint32_t kNonFinite = 0xFFFFFFFFu;   // partial marker: a NaN / Inf was read

__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

// Block-wide max of a uint32 (all threads get the result).
template <int NT>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < NT / 32) ? red[l] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Reduce the amax partials of one orientation (all threads of the CTA).
template <int NT>
__device__ __forceinline__ uint32_t reduce_partials(const uint32_t* p, int n, uint32_t* red) {
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n; i += NT) m = max(m, __ldcg(p + i));
  return block_max_u32<NT>(m, red);
}

// Tensor scales of both orientations from the partials (or the caller's
// alpha).  need_* select what is computed, pub_* what is published; CTA 0
// publishes alpha, amax and a device-side error.
template <int NT>
__device__ __forceinline__ void resolve_alpha(const QuantArgs& a, bool need_r, bool need_c,
                                              bool pub_r, bool pub_c, float& alpha_r,
                                              float& alpha_c, uint32_t* red, uint32_t cta) {
  if (a.flags & kAlphaProvided) {
    const float al = __ldg(a.alpha_in);
    alpha_r = alpha_c = al;
    if (cta == 0 && threadIdx.x == 0) {
      if (!(al >= 0.0f && al <= 3.402823466e38f) && a.status) *a.status = kStatusArg;
      if (pub_r && a.alpha_row) *a.alpha_row = al;
      if (pub_c && a.alpha_col) *a.alpha_col = al;
    }
    return;
  }
  uint32_t mr = 0, mc = 0;
  if (a.flags & kAmaxProvided) {
    // amax values of an earlier amax pass (nvfp4_amax's [plain, rotated
    // rows, rotated columns]): the plain one without rotation
    const uint32_t* am = reinterpret_cast<const uint32_t*>(a.alpha_in);
    if (need_r) mr = __ldg(am + (a.amax_rot ? 1 : 0));
    if (need_c) mc = __ldg(am + (a.amax_rot ? 2 : 0));
  } else {
    if (need_r) mr = reduce_partials<NT>(a.partials, a.npart, red);
    if (need_c) mc = reduce_partials<NT>(a.partials_col, a.npart, red);
  }
  // Eq. 1: alpha = amax / (6 * 448); with NVFP4_HEADROOM amax / (4 * 448)
  const float amax_r = __uint_as_float(mr == kNonFinite ? 0u : mr);
  const float amax_c = __uint_as_float(mc == kNonFinite ? 0u : mc);
  const float den = (a.flags & kHeadroom) ? 1792.0f : 2688.0f;
  alpha_r = __fdiv_rn(amax_r, den);
  alpha_c = __fdiv_rn(amax_c, den);
  if (cta == 0 && threadIdx.x == 0) {
    if ((mr == kNonFinite || mc == kNonFinite) && a.status) *a.status = kStatusNonFinite;
    if (pub_r && a.alpha_row) *a.alpha_row = alpha_r;
    if (pub_c && a.alpha_col) *a.alpha_col = alpha_c;
    if (a.amax_out) {
      if (pub_r) a.amax_out[0] = amax_r;
      if (pub_c) a.amax_out[1] = amax_c;
    }
  }
}

__device__ __forceinline__ uint32_t sign_bits(const PhiloxKeys& K) {
  return philox(K, 0u, 0u, 0u, kTagSigns).x & 0xFFFFu;
}

// ===========================================================================
// amax kernels.  Each CTA leaves one partial maximum (float bits, or
// kNonFinite) per orientation; the quantize kernels reduce them.
// ===========================================================================
// Plain amax: max |x| over the tensor in 16-byte chunks, four loads in
// flight per thread.  bf16 magnitudes order like their bit patterns with the
// sign cleared, so two are compared at once with a per-halfword unsigned
// max; a pattern >= 0x7F80 is an Inf or a NaN.
template <int NT>
// With atomic_out the CTA's maximum is folded into atomic_out[0] (zeroed by
// the launcher) instead of being stored as a partial.
__device__ __forceinline__ void amax_plain_body(const uint16_t* __restrict__ x, int64_t R, int64_t ld, FastDiv cpr,
                                                uint32_t* __restrict__ partial, uint32_t cta, uint32_t ncta,
                                                uint32_t* red, uint32_t* atomic_out = nullptr,
                                                int32_t* status = nullptr) {
  const uint32_t total = static_cast<uint32_t>(R) * cpr.d;   // chunks of 8 values
  const uint32_t stride = ncta * NT;
  uint32_t hm = 0;
  auto chunk = [&](uint32_t k) {
    const uint32_t r = fastdiv(k, cpr), c = k - r * cpr.d;
    return __ldcs(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(r) * ld) + c);
  };
  uint32_t k = cta * NT + threadIdx.x;
  for (; k + 3 * stride < total; k += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = chunk(k + j * stride);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      hm = __vmaxu2(hm, u[j].x & 0x7FFF7FFFu);
      hm = __vmaxu2(hm, u[j].y & 0x7FFF7FFFu);
      hm = __vmaxu2(hm, u[j].z & 0x7FFF7FFFu);
      hm = __vmaxu2(hm, u[j].w & 0x7FFF7FFFu);
    }
  }
  for (; k < total; k += stride) {
    const uint4 u = chunk(k);
    hm = __vmaxu2(hm, u.x & 0x7FFF7FFFu);
    hm = __vmaxu2(hm, u.y & 0x7FFF7FFFu);
    hm = __vmaxu2(hm, u.z & 0x7FFF7FFFu);
    hm = __vmaxu2(hm, u.w & 0x7FFF7FFFu);
  }
  const uint32_t h = max(hm & 0xFFFFu, hm >> 16);
  uint32_t m = (h >= 0x7F80u) ? kNonFinite : (h << 16);
  m = block_max_u32<NT>(m, red);
  if (threadIdx.x == 0) {
    if (atomic_out) {
      atomicMax(atomic_out, m);
      if (m == kNonFinite && status) *status = kStatusNonFinite;
    } else {
      partial[cta] = m;
    }
  }
}

// Rotated maxima: rows (16-element blocks along a row) and / or columns
// (16-element blocks down a column), from one read of the tensor.  The
// butterfly runs on two blocks at once (lane-paired) and without its final
// 1/4: round-to-nearest multiplication is monotone, so the maximum of the
// scaled magnitudes is the scaled maximum, applied once per CTA.
// With atomic_out the CTA's maxima are folded into atomic_out[0] (plain
// max |x|, from the same per-halfword maximum the Inf / NaN check keeps),
// [1] (rotated rows) and [2] (rotated columns), zeroed by the launcher,
// instead of being stored as partials.
// NT threads per CTA (256 or 128): with 128 each thread takes two row pairs
// and two column units of every tile, so the per-tile work (tile walk,
// copies, barrier) is spread over twice the elements.
template <bool ROW, bool COL, int NT = TNT>
__device__ __forceinline__ void amax_tile_body(const uint16_t* __restrict__ x, int64_t R, int64_t C, int64_t ld,
                                               FastDiv tiles_c, uint32_t ntiles, uint64_t seed,
                                               uint32_t* __restrict__ part_r, uint32_t* __restrict__ part_c,
                                               uint32_t cta, uint32_t ncta, uint8_t* ring, uint32_t* red,
                                               uint32_t* atomic_out = nullptr, int32_t* status = nullptr) {
  auto tiles = reinterpret_cast<uint4(*)[TR][TC / 8]>(ring);   // two tile buffers
  const SignMasks sm = sign_masks(sign_bits(philox_keys(seed)));
  const int t = threadIdx.x;
  float mr = 0.0f, mc = 0.0f;
  uint32_t hin = 0;   // per-halfword max of the input magnitudes (Inf / NaN check)
  uint32_t tile = cta;
  int buf = 0;
  TileWalk cur(cta, ncta, tiles_c.d), nxt = cur;   // this tile and the next, without divisions
  static_assert(NT == 256 || NT == 128, "256 or 128 threads");
  constexpr int kReps = 256 / NT;   // row pairs and column units per thread and tile
  if (tile < ntiles) load_tile_at<false, NT>(tiles[0], x, R, C, ld, nxt.tr, nxt.tc);
  nxt.advance();
  for (; tile < ntiles; tile += ncta, buf ^= 1) {
    const uint32_t next = tile + ncta;
    if (next < ntiles) {
      load_tile_at<false, NT>(tiles[buf ^ 1], x, R, C, ld, nxt.tr, nxt.tc);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    nxt.advance();
    __syncthreads();
    const uint4 (*s)[TC / 8] = tiles[buf];
    const int64_t r0 = static_cast<int64_t>(cur.tr) * TR, c0 = static_cast<int64_t>(cur.tc) * TC;
    cur.advance();
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);
    if constexpr (ROW) {
#pragma unroll
      for (int rep = 0; rep < kReps; ++rep) {
      // blocks (row, cb) and (row + 32, cb)
      const int row = (t >> 3) + (NT / 8) * rep, cb = t & 7;
      const bool va = row < rows && 16 * cb < cols, vb = row + 32 < rows && 16 * cb < cols;
      const uint4 a0 = s[row][tile_chunk(row, 2 * cb)], a1 = s[row][tile_chunk(row, 2 * cb + 1)];
      const uint4 b0 = s[row + 32][tile_chunk(row + 32, 2 * cb)];
      const uint4 b1 = s[row + 32][tile_chunk(row + 32, 2 * cb + 1)];
      if (va) {
        hin = __vmaxu2(hin, a0.x & 0x7FFF7FFFu); hin = __vmaxu2(hin, a0.y & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, a0.z & 0x7FFF7FFFu); hin = __vmaxu2(hin, a0.w & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, a1.x & 0x7FFF7FFFu); hin = __vmaxu2(hin, a1.y & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, a1.z & 0x7FFF7FFFu); hin = __vmaxu2(hin, a1.w & 0x7FFF7FFFu);
      }
      if (vb) {
        hin = __vmaxu2(hin, b0.x & 0x7FFF7FFFu); hin = __vmaxu2(hin, b0.y & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, b0.z & 0x7FFF7FFFu); hin = __vmaxu2(hin, b0.w & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, b1.x & 0x7FFF7FFFu); hin = __vmaxu2(hin, b1.y & 0x7FFF7FFFu);
        hin = __vmaxu2(hin, b1.z & 0x7FFF7FFFu); hin = __vmaxu2(hin, b1.w & 0x7FFF7FFFu);
      }
      float2 v[16];
      unpack16x2_signed(a0, a1, b0, b1, sm, v);
      hadamard16x2(v);
      float ma, mb;
      max_abs16x2(v, ma, mb);
      if (va) mr = fmaxf(mr, ma);
      if (vb) mr = fmaxf(mr, mb);
      }
    }
    if constexpr (COL) {
#pragma unroll
      for (int rep = 0; rep < kReps; ++rep) {
      // columns (2 cp, 2 cp + 1) of row block rb: one 32-bit word per row
      const int cp = t & 63, rb = (t >> 6) + (NT / 64) * rep;
      if (16 * rb < rows && 2 * cp < cols) {
        const uint32_t* base = reinterpret_cast<const uint32_t*>(&s[16 * rb][0]);
        const int wofs = tile_word(16 * rb, cp);   // the same for all 16 rows of the block
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = base[i * (TC / 2) + wofs];
          if constexpr (!ROW) hin = __vmaxu2(hin, w & 0x7FFF7FFFu);
          v[i] = make_float2(bf16lo_flip(w, sm.m[i]), bf16hi_flip(w, sm.m[i]));
        }
        hadamard16x2(v);
        float ma, mb;
        max_abs16x2(v, ma, mb);
        mc = max3(mc, ma, mb);
      }
      }
    }
    __syncthreads();   // buf is refilled two iterations from now
  }
  const uint32_t h = max(hin & 0xFFFFu, hin >> 16);
  const bool bad = h >= 0x7F80u;
  if (atomic_out) {
    const uint32_t mp = block_max_u32<NT>(bad ? kNonFinite : (h << 16), red);
    if (t == 0) {
      atomicMax(atomic_out, mp);
      if (mp == kNonFinite && status) *status = kStatusNonFinite;
    }
  }
  if constexpr (ROW) {
    uint32_t m = bad ? kNonFinite : __float_as_uint(__fmul_rn(mr, 0.25f));
    m = block_max_u32<NT>(m, red);
    if (t == 0) {
      if (atomic_out) atomicMax(atomic_out + 1, m);
      else part_r[cta] = m;
    }
  }
  if constexpr (COL) {
    uint32_t m = bad ? kNonFinite : __float_as_uint(__fmul_rn(mc, 0.25f));
    m = block_max_u32<NT>(m, red);
    if (t == 0) {
      if (atomic_out) atomicMax(atomic_out + 2, m);
      else part_c[cta] = m;
    }
  }
}

constexpr int kColPitch = 48;   // bytes per staged column of codes (32 used; rows 16-byte aligned)

// ---------------------------------------------------------------------------
// One mode's quantization of two lane-paired 16-element blocks (x: block a,
// y: block b), the element-wise steps done two blocks at a time.  v holds the
// (rotated) values; a block's random streams are keyed by (seed,
// c2 = 2 stream_id + orientation, block index).
// ---------------------------------------------------------------------------
// MS-EDEN scale of one block from its sums and its random word.
__device__ __forceinline__ uint32_t eden_scale(float num, float den, uint32_t word) {
  const uint32_t sc = e4m3_sr(__fdiv_rn(num, den), word >> 8);   // a select, not a branch, on den == 0
  return (den == 0.0f) ? 0u : sc;
}

// have_words: MS-EDEN only - wa / wb already hold the blocks' scale-SR words.
// c: the tensor scale's table (s and 1 / s per scale byte) and the Eq. 2
// denominators.
template <int MODE, class S>
__device__ __forceinline__ void quantize_pair(const float2* v, const S& c, const PhiloxKeys& K, uint32_t c2,
                                              uint64_t blka, uint64_t blkb, Packed16& pa, Packed16& pb,
                                              uint32_t& sba, uint32_t& sbb, bool have_words = false,
                                              uint32_t wa = 0u, uint32_t wb = 0u) {
  if constexpr (MODE == kModeRTN || MODE == kModeFourSix) {
    quantize_pair_tab<MODE == kModeFourSix>(v, c, pa, pb, sba, sbb);
  } else if constexpr (MODE == kModeMsEden) {
    // RTN codes under the provisional scale (M = 6), then the unbiasing
    // scale sum(r^2) / (alpha sum(r q)), stochastically rounded to E4M3
    float ma, mb;
    max_abs16x2(v, ma, mb);
    const float2 d6 = c.d6();
    const uint32_t prov = e4m3x2_rne(scale_quot(ma, d6.x), scale_quot(mb, d6.y));
    const float2 ta = c.ent_a(prov & 0xFFu), tb = c.ent_b(prov >> 8);
    float2 q[16], rr[16], rq[16];
    encode_decode_x2(v, make_float2(ta.y, tb.y), pa, pb, q);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      rr[i] = mul2(v[i], v[i]);
      rq[i] = mul2(v[i], q[i]);
    }
    const float2 num = sum16x2<true>(rr);
    const float2 den = mul2(c.alpha2(), sum16x2<true>(rq));
    if (!have_words) {
      const uint64_t ua = blka >> 2, ub = blkb >> 2;
      const uint4 da = philox(K, static_cast<uint32_t>(ua), static_cast<uint32_t>(ua >> 32), c2, kTagScaleSR);
      const uint4 db =
          (ua == ub) ? da : philox(K, static_cast<uint32_t>(ub), static_cast<uint32_t>(ub >> 32), c2, kTagScaleSR);
      const uint32_t sa = static_cast<uint32_t>(blka & 3), sbw = static_cast<uint32_t>(blkb & 3);
      wa = sa == 0 ? da.x : (sa == 1 ? da.y : (sa == 2 ? da.z : da.w));
      wb = sbw == 0 ? db.x : (sbw == 1 ? db.y : (sbw == 2 ? db.z : db.w));
    }
    sba = eden_scale(num.x, den.x, wa);
    sbb = eden_scale(num.y, den.y, wb);
  } else if constexpr (MODE == kModeRhtSRHw) {
    // RHT + stochastic rounding by the convert instruction: ceil scales as
    // below; one draw per block (unit blk), word g rounds elements 4g..4g+3,
    // handed over last element first so that nibble j holds element 4g + j.
    float ma, mb;
    max_abs16x2(v, ma, mb);
    const float2 d6 = c.d6();
    e4m3x2_ceil(scale_quot(ma, d6.x), scale_quot(mb, d6.y), sba, sbb);
    const float2 r2 = make_float2(c.ent_a(sba).y, c.ent_b(sbb).y);
    const uint4 da = philox(K, static_cast<uint32_t>(blka), static_cast<uint32_t>(blka >> 32), c2, kTagValueSRHw);
    const uint4 db = philox(K, static_cast<uint32_t>(blkb), static_cast<uint32_t>(blkb >> 32), c2, kTagValueSRHw);
    const uint32_t wa4[4] = {da.x, da.y, da.z, da.w}, wb4[4] = {db.x, db.y, db.z, db.w};
    float2 y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = mul2(v[i], r2);
    uint32_t ca[4], cb[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      ca[g] = e2m1x4_sr_hw(y[4 * g + 3].x, y[4 * g + 2].x, y[4 * g + 1].x, y[4 * g].x, wa4[g]);
      cb[g] = e2m1x4_sr_hw(y[4 * g + 3].y, y[4 * g + 2].y, y[4 * g + 1].y, y[4 * g].y, wb4[g]);
    }
    // the sign nibble follows the input's sign bit, zeros included (a zero
    // reciprocal leaves magnitude 0 and the sign alone)
    const Packed16 sa = sign_codes16<false>(v), sb = sign_codes16<true>(v);
    pa.lo = (ca[0] | (ca[1] << 16)) | sa.lo;
    pa.hi = (ca[2] | (ca[3] << 16)) | sa.hi;
    pb.lo = (cb[0] | (cb[1] << 16)) | sb.lo;
    pb.hi = (cb[2] | (cb[3] << 16)) | sb.hi;
  } else {  // RHT + stochastic rounding of the values
    float ma, mb;
    max_abs16x2(v, ma, mb);
    const float2 d6 = c.d6();
    e4m3x2_ceil(scale_quot(ma, d6.x), scale_quot(mb, d6.y), sba, sbb);
    const float2 r2 = make_float2(c.ent_a(sba).y, c.ent_b(sbb).y);
    // element i uses half (i & 1) of word (i >> 1) & 3 of draw i >> 3 (unit 2 blk + draw)
    uint32_t wa8[8], wb8[8];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint64_t ua = 2 * blka + j, ub = 2 * blkb + j;
      const uint4 da = philox(K, static_cast<uint32_t>(ua), static_cast<uint32_t>(ua >> 32), c2, kTagValueSR);
      const uint4 db = philox(K, static_cast<uint32_t>(ub), static_cast<uint32_t>(ub >> 32), c2, kTagValueSR);
      wa8[4 * j] = da.x; wa8[4 * j + 1] = da.y; wa8[4 * j + 2] = da.z; wa8[4 * j + 3] = da.w;
      wb8[4 * j] = db.x; wb8[4 * j + 1] = db.y; wb8[4 * j + 2] = db.z; wb8[4 * j + 3] = db.w;
    }
    float qa[16], qb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = mul2(v[i], r2);
      const int w = ((i >> 3) << 2) | ((i >> 1) & 3), sh = 16 * (i & 1);
      qa[i] = e2m1_sr_value_nb(y.x, (wa8[w] >> sh) & 0xFFFFu);
      qb[i] = e2m1_sr_value_nb(y.y, (wb8[w] >> sh) & 0xFFFFu);
    }
    // the rounded values lie on the grid, so their encoding is exact (a zero
    // reciprocal gives signed zeros)
    pa.lo = e2m1x8_rne(qa[0], qa[1], qa[2], qa[3], qa[4], qa[5], qa[6], qa[7]);
    pa.hi = e2m1x8_rne(qa[8], qa[9], qa[10], qa[11], qa[12], qa[13], qa[14], qa[15]);
    pb.lo = e2m1x8_rne(qb[0], qb[1], qb[2], qb[3], qb[4], qb[5], qb[6], qb[7]);
    pb.hi = e2m1x8_rne(qb[8], qb[9], qb[10], qb[11], qb[12], qb[13], qb[14], qb[15]);
  }
}

// ===========================================================================
// Rowwise quantization, streamed: a thread takes the consecutive blocks 2k
// and 2k + 1 of the row-major block order (64 contiguous bytes when they
// share a row) and quantizes them lane-paired.  Both lie in MS-EDEN draw
// unit k / 2, so one draw serves the pair.
// ===========================================================================
template <int MODE, bool ROT, int NT, bool VEC = false>
__device__ __forceinline__ void quant_rows_body(const QuantArgs& a, uint32_t cta, uint32_t ncta, uint32_t* red,
                                                float2* tab) {
  float alpha = 0.0f, alpha_unused;
  if constexpr (!VEC) {
    resolve_alpha<NT>(a, true, false, true, false, alpha, alpha_unused, red, cta);
    build_scale_tab<NT>(tab, alpha);
    __syncthreads();
  }
  const TabScales sc = make_scale_ctx(tab, alpha);
  const PhiloxKeys K = philox_keys(a.seed);
  SignMasks sm;
  if constexpr (ROT) {
    sm = sign_masks(sign_bits(K));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) sm.m[i] = 0u;
  }
  const uint32_t c2 = a.stream_id * 2u;
  const uint32_t nb = a.nb_row.d;
  const uint32_t total = static_cast<uint32_t>(a.R) * nb;
  const uint32_t npairs = (total + 1) / 2;
  const uint32_t stride = ncta * NT;
  const bool gemm = (a.flags & kGemmScaleLayout) != 0;
  const bool check = (a.flags & kAlphaProvided) != 0;
  // Pair pk holds blocks 2 pk and 2 pk + 1 (64 contiguous bytes when they
  // share a row).  The next pair's loads are issued before this pair is
  // encoded, so every thread keeps a pair in flight while it computes.
  auto load_pair = [&](uint32_t pk, uint4& a0, uint4& a1, uint4& b0, uint4& b1) {
    const uint32_t ka = 2 * pk, kb = ka + 1 < total ? ka + 1 : ka;
    const uint32_t ra = fastdiv(ka, a.nb_row), cba = ka - ra * nb;
    const uint32_t rb = fastdiv(kb, a.nb_row), cbb = kb - rb * nb;
    const uint4* pa = reinterpret_cast<const uint4*>(a.x + static_cast<int64_t>(ra) * a.ld + 16 * cba);
    const uint4* pb = reinterpret_cast<const uint4*>(a.x + static_cast<int64_t>(rb) * a.ld + 16 * cbb);
    a0 = __ldcs(pa);
    a1 = __ldcs(pa + 1);
    b0 = __ldcs(pb);
    b1 = __ldcs(pb + 1);
  };
  uint32_t pk = cta * NT + threadIdx.x;
  uint4 n0, n1, n2, n3;
  if (pk < npairs) load_pair(pk, n0, n1, n2, n3);
  for (; pk < npairs; pk += stride) {
    const uint4 a0 = n0, a1 = n1, b0 = n2, b1 = n3;
    if (pk + stride < npairs) load_pair(pk + stride, n0, n1, n2, n3);
    const uint32_t ka = 2 * pk, kb = ka + 1;
    const bool vb = kb < total;
    const uint32_t ra = fastdiv(ka, a.nb_row), cba = ka - ra * nb;
    const uint32_t kk = vb ? kb : ka;
    const uint32_t rb = fastdiv(kk, a.nb_row), cbb = kk - rb * nb;
    if (check) {
      uint32_t hin = 0;
      const uint32_t w[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                              b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) hin = __vmaxu2(hin, w[i] & 0x7FFF7FFFu);
      if (max(hin & 0xFFFFu, hin >> 16) >= 0x7F80u && a.status) *a.status = kStatusNonFinite;
    }
    float2 v[16];
    unpack16x2_signed(a0, a1, b0, b1, sm, v);
    if constexpr (ROT) rht16x2_presigned(v);
    Packed16 qa, qb;
    uint32_t sa, sb;
    if constexpr (VEC) {
      // one tensor scale per row; the thread holding a row's first block
      // publishes it
      const float aa = vector_alpha(a, a.vmax_r, ra);
      const float ab = (rb == ra) ? aa : vector_alpha(a, a.vmax_r, rb);
      quantize_pair<MODE>(v, make_vec_scales(aa, ab), K, c2, ka, kb, qa, qb, sa, sb);
      if (cba == 0) a.alpha_row[ra] = aa;
      if (vb && cbb == 0) a.alpha_row[rb] = ab;
    } else {
      quantize_pair<MODE>(v, sc, K, c2, ka, kb, qa, qb, sa, sb);
    }
    uint8_t* ca = a.codes_row + static_cast<int64_t>(ra) * (a.C / 2) + 8 * cba;
    if (vb && rb == ra && (reinterpret_cast<uintptr_t>(ca) & 15u) == 0) {
      *reinterpret_cast<uint4*>(ca) = make_uint4(qa.lo, qa.hi, qb.lo, qb.hi);
    } else {
      *reinterpret_cast<uint2*>(ca) = make_uint2(qa.lo, qa.hi);
      if (vb)
        *reinterpret_cast<uint2*>(a.codes_row + static_cast<int64_t>(rb) * (a.C / 2) + 8 * cbb) =
            make_uint2(qb.lo, qb.hi);
    }
    if (a.scales_row) {
      // R * C / 16 < 2^32 blocks here, so 32-bit offsets suffice
      a.scales_row[gemm ? gemm_scale_offset32(ra, cba, nb) : ka] = static_cast<uint8_t>(sa);
      if (vb) a.scales_row[gemm ? gemm_scale_offset32(rb, cbb, nb) : kb] = static_cast<uint8_t>(sb);
    }
  }
}

// ===========================================================================
// Tiled 1D quantization (columns, or rows + columns from one read), two
// blocks per thread per orientation, lane-paired.
//   rows:    thread t takes row blocks (t / 8, t % 8) and (t / 8 + 32, t % 8)
//   columns: thread t takes columns 2 (t / 4), 2 (t / 4) + 1 of row block t % 4
// Column codes are staged transposed in shared memory and written as whole
// 32-byte rows of the column-major output.
// ===========================================================================
// Tiles stream through a ring of kTileStages shared-memory buffers (dynamic
// shared memory), so up to kTileStages - 1 tiles are in flight per CTA while
// one is processed.
constexpr int kTileStages = 2;
constexpr int kTileBytes = TR * TC * 2;

// Resident CTAs per SM the register budget is sized for: the kernels are
// bound by the latency of dependent arithmetic, so more warps help.
// Threads per CTA of the 1D tile kernels: RTN and hardware-SR run 128-thread
// CTAs (two units of each orientation per thread and tile, five CTAs per SM
// by shared memory), measured 3-4% faster; the modes with more arithmetic
// per block keep 256 threads, where the extra registers of two units cost
// more than the shared per-tile work saves (4/6 rows + columns +13%, RHT + SR
// +26% at 128).
template <int MODE>
constexpr int tile_1d_threads() { return (MODE == kModeRTN || MODE == kModeRhtSRHw) ? 128 : 256; }
template <int MODE>
constexpr int tile_1d_min_blocks() { return tile_1d_threads<MODE>() == 128 ? 5 : 3; }

// Shared memory of the tile kernels besides the tile ring.
struct TileStaging {
  uint8_t colcodes[TC][kColPitch];   // transposed column codes of one tile
  uint8_t colscale[TC][TR / 16];     // their scales (2D: unused)
  uint8_t scale2d[TR / 16][TC / 16]; // chosen 16x16 scales (2D)
  uint32_t red[TNT / 32];
  float2 tab_r[kScaleTab];           // {s, 1 / s} per scale byte, row orientation
  float2 tab_c[kScaleTab];           // the same for the column orientation
};

// NT threads per CTA (256 or 128): with 128 each thread takes two row pairs
// and two column pairs of every tile (kReps units of each).
template <int MODE, bool ROT, bool ROW, bool COL, bool VEC = false, int NT = TNT>
__device__ __forceinline__ void quant_tile_1d_body(const QuantArgs& a, uint32_t cta, uint32_t ncta, uint8_t* ring,
                                                   TileStaging& stg) {
  auto tiles = reinterpret_cast<uint4(*)[TR][TC / 8]>(ring);
  auto& colcodes = stg.colcodes;
  auto& colscale = stg.colscale;
  uint32_t* red = stg.red;
  float alpha_r = 0.0f, alpha_c = 0.0f;
  if constexpr (!VEC) {
    resolve_alpha<NT>(a, ROW, COL, ROW, COL, alpha_r, alpha_c, red, cta);
    if constexpr (ROW) build_scale_tab<NT>(stg.tab_r, alpha_r);
    if constexpr (COL) build_scale_tab<NT>(stg.tab_c, alpha_c);
    __syncthreads();
  }
  const TabScales scr = make_scale_ctx(stg.tab_r, alpha_r), scc = make_scale_ctx(stg.tab_c, alpha_c);
  const PhiloxKeys K = philox_keys(a.seed);
  SignMasks sm;
  if constexpr (ROT) {
    sm = sign_masks(sign_bits(K));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) sm.m[i] = 0u;
  }
  const uint32_t c2r = a.stream_id * 2u, c2c = a.stream_id * 2u + 1u;
  const bool gemm = (a.flags & kGemmScaleLayout) != 0;
  const bool check = (a.flags & kAlphaProvided) != 0;
  const int t = threadIdx.x;
  const int64_t R = a.R, C = a.C;
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  // MS-EDEN draws one 4-word number per 4 consecutive blocks.  The lanes
  // 4k .. 4k+3 of a warp hold the same two row-block units and the same two
  // column-block units of a tile (when C and R are multiples of 64, so units
  // never straddle a row or a column), each lane needing word (lane % 4) of
  // all four draws: each lane computes one draw, stores it in its warp's
  // slice of the column staging and reads its words back.
  const bool share = MODE == kModeMsEden && (!ROW || C % 64 == 0) && (!COL || R % 64 == 0);
  const int lane = t & 31, j4 = t & 3;
  static_assert(NT == 256 || NT == 128, "256 or 128 threads");
  constexpr int kReps = 256 / NT;
  // whole tiles write columns as 16-byte code pieces and 4-byte scale words
  // (R % 64 == 0 keeps both aligned)
  const bool col_words = R % 64 == 0 && (reinterpret_cast<uintptr_t>(a.scales_col) & 3u) == 0;

  // Per-thread parts of the block indices and offsets, fixed for the whole
  // kernel: rows t/8 and t/8 + 32 of block column t%8 (row orientation);
  // columns 2 (t/4), +1 of row block t%4 and, in the write-out, column t/2
  // (column orientation); unit k of kReps adds NT/8 rows, NT/4 column pairs
  // and NT/2 write-out columns.  A tile adds its own part once.
  const int64_t nbr = C / 16, nbc = R / 16;
  const int trow = t >> 3, tcb = t & 7, tcp = t >> 2, trb = t & 3;
  const int64_t rblk_thr = trow * nbr + tcb, rcode_thr = trow * (C / 2) + 8 * tcb;
  const int64_t cblk_thr = 2 * tcp * nbc + trb, ccode_thr = (t >> 1) * (R / 2) + 16 * (t & 1);
  const int64_t share_thr = (j4 < 2) ? (trow + 32 * j4) * nbr + (tcb & ~3) : (2 * tcp + (j4 - 2)) * nbc;
  const int64_t rep_rblk = (NT / 8) * nbr, rep_rcode = (NT / 8) * (C / 2), rep_cblk = 2 * (NT / 4) * nbc;
  const int64_t rep_share = (j4 < 2) ? rep_rblk : rep_cblk, rep_ccode = (NT / 2) * (R / 2);
  // this tile and the one kTileStages - 1 iterations ahead, walked without
  // divisions
  TileWalk cur(cta, ncta, static_cast<uint32_t>(a.tiles_c)), ahd = cur;

  // prologue: the first kTileStages - 1 tiles (an empty copy group when a
  // tile does not exist keeps the group count in step)
  uint32_t tile = cta;
#pragma unroll
  for (int k = 0; k < kTileStages - 1; ++k) {
    const uint32_t tk = tile + k * ncta;
    if (tk < ntiles) load_tile_at<false, NT>(tiles[k], a.x, R, C, a.ld, ahd.tr, ahd.tc);
    else cp_async_commit();
    ahd.advance();
  }
  int buf = 0;
  for (; tile < ntiles; tile += ncta, buf = (buf + 1 == kTileStages) ? 0 : buf + 1) {
    const uint32_t ahead = tile + (kTileStages - 1) * ncta;
    const int abuf = (buf == 0) ? kTileStages - 1 : buf - 1;   // (buf + kTileStages - 1) % kTileStages
    if (ahead < ntiles) load_tile_at<false, NT>(tiles[abuf], a.x, R, C, a.ld, ahd.tr, ahd.tc);
    else cp_async_commit();
    ahd.advance();
    cp_async_wait<kTileStages - 1>();   // this tile's group has landed
    __syncthreads();
    const uint4 (*s)[TC / 8] = tiles[buf];
    const uint32_t tr = cur.tr, tc = cur.tc;
    cur.advance();
    const int64_t r0 = static_cast<int64_t>(tr) * TR, c0 = static_cast<int64_t>(tc) * TC;
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);
    const int64_t rblk_tile = r0 * nbr + c0 / 16;   // first row block of the tile
    const int64_t cblk_tile = c0 * nbc + r0 / 16;   // first column block of the tile

    // scale-SR words of this thread's blocks: row a, row b, column 2cp, 2cp+1
    // (per unit)
    uint32_t w_ra[kReps] = {}, w_rb[kReps] = {}, w_ca[kReps] = {}, w_cb[kReps] = {};
    if (share) {
#pragma unroll
      for (int k = 0; k < kReps; ++k) {
        // row block units: row (t / 8) + 32 j4, blocks (t % 8) & ~3 ..;
        // column units: column 2 (t / 4) + (j4 - 2), row blocks r0/16 ..
        const uint64_t unit = static_cast<uint64_t>((j4 < 2 ? rblk_tile : cblk_tile) + share_thr + k * rep_share) >> 2;
        const uint32_t c2 = (j4 < 2) ? c2r : c2c;
        const uint4 d = philox(K, static_cast<uint32_t>(unit), static_cast<uint32_t>(unit >> 32), c2, kTagScaleSR);
        // warp w's slice for unit k: 512 bytes at the start of colcodes rows
        // 16 w + (NT / 2) k .., rows only warp w writes (column pass) and
        // reads (write-out) in this tile, free until its column pass; the
        // previous tile's write-out read them before the barrier at the top
        // of this iteration
        uint4* xs = reinterpret_cast<uint4*>(&colcodes[16 * (t >> 5) + (NT / 2) * k][0]);
        xs[lane] = d;
        __syncwarp();
        // word j4 of the draws of quad lanes 0..3
        const uint32_t* xw = reinterpret_cast<const uint32_t*>(xs + (lane & ~3)) + j4;
        w_ra[k] = xw[0];
        w_rb[k] = xw[4];
        w_ca[k] = xw[8];
        w_cb[k] = xw[12];
      }
      __syncwarp();   // every lane has read before the column pass rewrites the rows
    }

    if (check) {
      uint32_t hin = 0;
#pragma unroll
      for (int i = 0; i < (TR * TC / 8) / NT; ++i) {
        const int ch = t + NT * i;
        const int row = ch >> 4, cc = ch & 15;
        if (row < rows && 8 * cc < cols) {
          const uint4 u = s[row][tile_chunk(row, cc)];
          hin = __vmaxu2(hin, u.x & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.y & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.z & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.w & 0x7FFF7FFFu);
        }
      }
      if (max(hin & 0xFFFFu, hin >> 16) >= 0x7F80u && a.status) *a.status = kStatusNonFinite;
    }

    if constexpr (ROW) {
#pragma unroll
      for (int k = 0; k < kReps; ++k) {
      const int row = trow + (NT / 8) * k, cb = tcb;
      const bool va = row < rows && 16 * cb < cols, vb = row + 32 < rows && 16 * cb < cols;
      if (va || vb) {
        const uint4 a0 = s[row][tile_chunk(row, 2 * cb)], a1 = s[row][tile_chunk(row, 2 * cb + 1)];
        const uint4 b0 = s[row + 32][tile_chunk(row + 32, 2 * cb)];
        const uint4 b1 = s[row + 32][tile_chunk(row + 32, 2 * cb + 1)];
        float2 v[16];
        unpack16x2_signed(a0, a1, b0, b1, sm, v);
        if constexpr (ROT) rht16x2_presigned(v);
        const int64_t gra = r0 + row, grb = gra + 32;
        const uint64_t blka = static_cast<uint64_t>(rblk_tile + rblk_thr + k * rep_rblk);
        const uint64_t blkb = blka + static_cast<uint64_t>(32 * nbr);
        Packed16 pa, pb;
        uint32_t sa, sb;
        if constexpr (VEC) {
          // tensor scales of rows gra and grb; the tiles of the first tile
          // column publish them
          const float aa = va ? vector_alpha(a, a.vmax_r, gra) : 0.0f;
          const float ab = vb ? vector_alpha(a, a.vmax_r, grb) : aa;
          quantize_pair<MODE>(v, make_vec_scales(aa, ab), K, c2r, blka, blkb, pa, pb, sa, sb, share, w_ra[k], w_rb[k]);
          if (tc == 0 && cb == 0) {
            if (va) a.alpha_row[gra] = aa;
            if (vb) a.alpha_row[grb] = ab;
          }
        } else {
          quantize_pair<MODE>(v, scr, K, c2r, blka, blkb, pa, pb, sa, sb, share, w_ra[k], w_rb[k]);
        }
        // row gra's 8 code bytes, row grb's 32 rows further on; the scale
        // offsets split into a tile part and a thread part
        uint8_t* crow = a.codes_row + (r0 * (C / 2) + c0 / 2) + rcode_thr + k * rep_rcode;
        if (va) *reinterpret_cast<uint2*>(crow) = make_uint2(pa.lo, pa.hi);
        if (vb) *reinterpret_cast<uint2*>(crow + 32 * (C / 2)) = make_uint2(pb.lo, pb.hi);
        if (a.scales_row) {
          uint8_t* srow = a.scales_row + (gemm ? gemm_scale_tile_row(tr, tc, C / 16) + gemm_scale_thread_row(row, cb)
                                               : static_cast<int64_t>(blka));
          if (va) srow[0] = static_cast<uint8_t>(sa);
          if (vb) srow[gemm ? 4 : 32 * nbr] = static_cast<uint8_t>(sb);
        }
      }
      }
    }

    if constexpr (COL) {
#pragma unroll
      for (int k = 0; k < kReps; ++k) {
      const int cp = tcp + (NT / 4) * k, rb = trb;
      if (16 * rb < rows && 2 * cp < cols) {
        const uint32_t* base = reinterpret_cast<const uint32_t*>(&s[16 * rb][0]);
        const int wofs = tile_word(16 * rb, cp);   // the same for all 16 rows of the block
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = base[i * (TC / 2) + wofs];
          v[i] = make_float2(bf16lo_flip(w, sm.m[i]), bf16hi_flip(w, sm.m[i]));
        }
        if constexpr (ROT) rht16x2_presigned(v);
        const int64_t gc = c0 + 2 * cp;
        const uint64_t blka = static_cast<uint64_t>(cblk_tile + cblk_thr + k * rep_cblk);
        const uint64_t blkb = blka + static_cast<uint64_t>(nbc);
        Packed16 qa, qb;
        uint32_t sa, sb;
        if constexpr (VEC) {
          // tensor scales of columns gc, gc + 1; the first tile row publishes them
          const float aa = vector_alpha(a, a.vmax_c, gc), ab = vector_alpha(a, a.vmax_c, gc + 1);
          quantize_pair<MODE>(v, make_vec_scales(aa, ab), K, c2c, blka, blkb, qa, qb, sa, sb, share, w_ca[k], w_cb[k]);
          if (tr == 0 && rb == 0) {
            a.alpha_col[gc] = aa;
            a.alpha_col[gc + 1] = ab;
          }
        } else {
          quantize_pair<MODE>(v, scc, K, c2c, blka, blkb, qa, qb, sa, sb, share, w_ca[k], w_cb[k]);
        }
        *reinterpret_cast<uint2*>(&colcodes[2 * cp][8 * rb]) = make_uint2(qa.lo, qa.hi);
        *reinterpret_cast<uint2*>(&colcodes[2 * cp + 1][8 * rb]) = make_uint2(qb.lo, qb.hi);
        colscale[2 * cp][rb] = static_cast<uint8_t>(sa);
        colscale[2 * cp + 1][rb] = static_cast<uint8_t>(sb);
      }
      }
      __syncthreads();
      if (rows == TR && cols == TC && col_words) {
        // whole tile: thread t copies 16 code bytes of column t / 2 (+ NT / 2
        // per unit) and the 4-byte word of column t's (t + NT ..) four scales
#pragma unroll
        for (int k = 0; k < kReps; ++k) {
          const int c = (t >> 1) + (NT / 2) * k, h = t & 1;
          *reinterpret_cast<uint4*>(a.codes_col + (c0 * (R / 2) + r0 / 2) + ccode_thr + k * rep_ccode) =
              *reinterpret_cast<const uint4*>(&colcodes[c][16 * h]);
        }
        if (a.scales_col) {
          for (int c = t; c < TC; c += NT) {
            const int64_t off = gemm ? gemm_scale_tile_col(tr, tc, nbc) + gemm_scale_thread_col(c)
                                     : cblk_tile + c * nbc;
            *reinterpret_cast<uint32_t*>(a.scales_col + off) = *reinterpret_cast<const uint32_t*>(&colscale[c][0]);
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < kReps; ++k) {
          const int c = (t >> 1) + (NT / 2) * k, h = t & 1;
          const int nbytes = rows / 2;
          if (c < cols && 16 * h < nbytes) {
            uint8_t* dst = a.codes_col + (c0 + c) * (R / 2) + r0 / 2 + 16 * h;
            const uint2* src = reinterpret_cast<const uint2*>(&colcodes[c][16 * h]);
            reinterpret_cast<uint2*>(dst)[0] = src[0];
            if (16 * h + 8 < nbytes) reinterpret_cast<uint2*>(dst)[1] = src[1];
          }
        }
        if (a.scales_col) {
          for (int c = t >> 1; c < cols; c += NT / 2) {
            for (int rb2 = (t & 1); rb2 < rows / 16; rb2 += 2) {
              const int64_t gc = c0 + c, grb = r0 / 16 + rb2;
              const uint8_t sbyte = colscale[c][rb2];
              if (gemm) a.scales_col[gemm_scale_offset(gc, grb, R / 16)] = sbyte;
              else a.scales_col[gc * (R / 16) + grb] = sbyte;
            }
          }
        }
      }
    }
    // With the column pass no barrier is needed here: every read of this
    // tile's buffer happens before the barrier ahead of the write-out, and
    // every read of the staging before the next tile's first barrier, which
    // the next writes of the staging follow.
    if constexpr (!COL) __syncthreads();
  }
  cp_async_wait<0>();
}

// ===========================================================================
// Tiled 2D quantization: 16 x 16 blocks share one scale (rows of a 16-lane
// half-warp, one tile row each), two blocks per thread lane-paired:
// thread t takes row t % 16 of blocks (t / 128, (t / 16) % 8) and
// (t / 128 + 2, (t / 16) % 8) of the tile's 4 x 8 block grid.  The column
// orientation reuses the chosen block scales on the transposed blocks.
// ===========================================================================
template <int MODE, bool ROW, bool COL>
__device__ __forceinline__ void quant_tile_2d_body(const QuantArgs& a, uint32_t cta, uint32_t ncta, uint8_t* ring,
                                                   TileStaging& stg) {
  auto tiles = reinterpret_cast<uint4(*)[TR][TC / 8]>(ring);
  auto& colcodes = stg.colcodes;
  auto& scale2d = stg.scale2d;
  uint32_t* red = stg.red;
  float alpha, alpha_c;
  // one tensor scale for both orientations: the plain amax, whose partials
  // both orientations read (alpha_c == alpha; it is computed to publish it)
  resolve_alpha<TNT>(a, true, COL, ROW, COL, alpha, alpha_c, red, cta);
  build_scale_tab<TNT>(stg.tab_r, alpha);
  __syncthreads();
  const TabScales sc = make_scale_ctx(stg.tab_r, alpha);
  const bool gemm = (a.flags & kGemmScaleLayout) != 0;
  const bool check = (a.flags & kAlphaProvided) != 0;
  const int t = threadIdx.x;
  const int64_t R = a.R, C = a.C;
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  // whole tiles write columns as 16-byte code pieces and 4-byte scale words
  const bool col_words = R % 64 == 0 && (reinterpret_cast<uintptr_t>(a.scales_col) & 3u) == 0;

  // this tile and the one kTileStages - 1 iterations ahead, walked without
  // divisions
  TileWalk cur(cta, ncta, static_cast<uint32_t>(a.tiles_c)), ahd = cur;
  uint32_t tile = cta;
#pragma unroll
  for (int k = 0; k < kTileStages - 1; ++k) {
    const uint32_t tk = tile + k * ncta;
    if (tk < ntiles) load_tile_at<true>(tiles[k], a.x, R, C, a.ld, ahd.tr, ahd.tc);
    else cp_async_commit();
    ahd.advance();
  }
  int buf = 0;
  for (; tile < ntiles; tile += ncta, buf = (buf + 1 == kTileStages) ? 0 : buf + 1) {
    const uint32_t ahead = tile + (kTileStages - 1) * ncta;
    const int abuf = (buf == 0) ? kTileStages - 1 : buf - 1;
    if (ahead < ntiles) load_tile_at<true>(tiles[abuf], a.x, R, C, a.ld, ahd.tr, ahd.tc);
    else cp_async_commit();
    ahd.advance();
    cp_async_wait<kTileStages - 1>();
    __syncthreads();
    const uint4 (*s)[TC / 8] = tiles[buf];
    const uint32_t tr = cur.tr, tc = cur.tc;
    cur.advance();
    const int64_t r0 = static_cast<int64_t>(tr) * TR, c0 = static_cast<int64_t>(tc) * TC;
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);   // multiple of 16
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);   // multiple of 16

    if (check) {
      uint32_t hin = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ch = t + TNT * i;
        const int row = ch >> 4, cc = ch & 15;
        if (row < rows && 8 * cc < cols) {
          const uint4 u = s[row][tile_chunk_2d(row, cc)];
          hin = __vmaxu2(hin, u.x & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.y & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.z & 0x7FFF7FFFu);
          hin = __vmaxu2(hin, u.w & 0x7FFF7FFFu);
        }
      }
      if (max(hin & 0xFFFFu, hin >> 16) >= 0x7F80u && a.status) *a.status = kStatusNonFinite;
    }

    {
      const int rb = t >> 7, cbb = (t >> 4) & 7, lr = t & 15;
      const int rowa = 16 * rb + lr, rowb = rowa + 32;
      // uniform per half-warp (rows and cols are multiples of 16)
      const bool va = 16 * rb < rows && 16 * cbb < cols, vb = 16 * rb + 32 < rows && 16 * cbb < cols;
      const uint4 a0 = s[rowa][tile_chunk_2d(rowa, 2 * cbb)], a1 = s[rowa][tile_chunk_2d(rowa, 2 * cbb + 1)];
      const uint4 b0 = s[rowb][tile_chunk_2d(rowb, 2 * cbb)], b1 = s[rowb][tile_chunk_2d(rowb, 2 * cbb + 1)];
      SignMasks none;
#pragma unroll
      for (int i = 0; i < 16; ++i) none.m[i] = 0u;
      float2 v[16];
      unpack16x2_signed(a0, a1, b0, b1, none, v);
      if (!va) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i].x = 0.0f;
      }
      if (!vb) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i].y = 0.0f;
      }
      float ma, mb;
      max_abs16x2(v, ma, mb);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        ma = fmaxf(ma, __shfl_xor_sync(0xFFFFFFFFu, ma, o));
        mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
      }
      const uint32_t s6 = e4m3x2_rne(scale_quot(ma, sc.den6), scale_quot(mb, sc.den6));
      uint32_t sa = s6 & 0xFFu, sb = s6 >> 8;
      const float2 ta6 = sc.tab[sa], tb6 = sc.tab[sb];
      Packed16 pa, pb;
      if constexpr (MODE != kModeFourSix) encode_x2(v, make_float2(ta6.y, tb6.y), pa, pb);
      if constexpr (MODE == kModeFourSix) {
        // each candidate's grid values come out of its encoding
        float2 q[16];
        encode_decode_x2(v, make_float2(ta6.y, tb6.y), pa, pb, q);
        float2 e6 = sq_error_q(v, make_float2(ta6.x, tb6.x), q);
        const uint32_t s4 = e4m3x2_rne(scale_quot(ma, sc.den4), scale_quot(mb, sc.den4));
        const uint32_t sa4 = s4 & 0xFFu, sb4 = s4 >> 8;
        const float2 ta4 = sc.tab[sa4], tb4 = sc.tab[sb4];
        Packed16 pa4, pb4;
        encode_decode_x2(v, make_float2(ta4.y, tb4.y), pa4, pb4, q);
        float2 e4 = sq_error_q(v, make_float2(ta4.x, tb4.x), q);
        // block error = the half-warp's row errors summed in butterfly order
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          e6.x = __fadd_rn(e6.x, __shfl_xor_sync(0xFFFFFFFFu, e6.x, o));
          e6.y = __fadd_rn(e6.y, __shfl_xor_sync(0xFFFFFFFFu, e6.y, o));
          e4.x = __fadd_rn(e4.x, __shfl_xor_sync(0xFFFFFFFFu, e4.x, o));
          e4.y = __fadd_rn(e4.y, __shfl_xor_sync(0xFFFFFFFFu, e4.y, o));
        }
        if (e4.x < e6.x) {
          sa = sa4;
          pa = pa4;
        }
        if (e4.y < e6.y) {
          sb = sb4;
          pb = pb4;
        }
      }
      const int64_t gcb = c0 / 16 + cbb;
      if (lr == 0) {
        if (va) scale2d[rb][cbb] = static_cast<uint8_t>(sa);
        if (vb) scale2d[rb + 2][cbb] = static_cast<uint8_t>(sb);
      }
      if constexpr (ROW) {
        // row rowa's 8 code bytes, row rowb = rowa + 32 further on; in the
        // GEMM layout every row of a 2D block carries its scale (rowa < 32:
        // tile part + thread part, rowb 4 bytes further on), in the plain
        // layout one byte per 16 x 16 block
        uint8_t* crow = a.codes_row + (r0 + rowa) * (C / 2) + 8 * gcb;
        if (va) *reinterpret_cast<uint2*>(crow) = make_uint2(pa.lo, pa.hi);
        if (vb) *reinterpret_cast<uint2*>(crow + 32 * (C / 2)) = make_uint2(pb.lo, pb.hi);
        if (a.scales_row && (gemm || lr == 0)) {
          uint8_t* srow = a.scales_row + (gemm ? gemm_scale_tile_row(tr, tc, C / 16) + gemm_scale_thread_row(rowa, cbb)
                                               : (r0 / 16 + rb) * (C / 16) + gcb);
          if (va) srow[0] = static_cast<uint8_t>(sa);
          if (vb) srow[gemm ? 4 : 2 * (C / 16)] = static_cast<uint8_t>(sb);
        }
      }
    }

    if constexpr (COL) {
      __syncthreads();   // scale2d complete
      // columns (2 cp, 2 cp + 1) of row block rb, both in 16-column block cp / 8
      const int cp = t & 63, rb = t >> 6;
      if (16 * rb < rows && 2 * cp < cols) {
        const uint32_t* base = reinterpret_cast<const uint32_t*>(&s[16 * rb][0]);
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = base[i * (TC / 2) + tile_word_2d(i, cp)];   // row 16 rb + i: (16 rb + i) & 7 == i & 7
          v[i] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
        }
        const uint32_t sbyte = scale2d[rb][cp >> 3];
        Packed16 qa, qb;
        const float r = sc.tab[sbyte].y;
        encode_x2(v, make_float2(r, r), qa, qb);
        *reinterpret_cast<uint2*>(&colcodes[2 * cp][8 * rb]) = make_uint2(qa.lo, qa.hi);
        *reinterpret_cast<uint2*>(&colcodes[2 * cp + 1][8 * rb]) = make_uint2(qb.lo, qb.hi);
      }
      __syncthreads();
      if (rows == TR && cols == TC && col_words) {
        // whole tile: 16 code bytes per thread; in the GEMM layout threads
        // 0..127 write column t's four scale bytes as one word
        const int c = t >> 1, h = t & 1;
        *reinterpret_cast<uint4*>(a.codes_col + (c0 + c) * (R / 2) + r0 / 2 + 16 * h) =
            *reinterpret_cast<const uint4*>(&colcodes[c][16 * h]);
        if (a.scales_col && t < TC) {
          const int cb = t >> 4;
          if (gemm) {
            const uint32_t w = static_cast<uint32_t>(scale2d[0][cb]) | (static_cast<uint32_t>(scale2d[1][cb]) << 8) |
                               (static_cast<uint32_t>(scale2d[2][cb]) << 16) |
                               (static_cast<uint32_t>(scale2d[3][cb]) << 24);
            *reinterpret_cast<uint32_t*>(a.scales_col + gemm_scale_tile_col(tr, tc, R / 16) +
                                         gemm_scale_thread_col(t)) = w;
          } else if ((t & 15) == 0) {
            for (int rb2 = 0; rb2 < 4; ++rb2) a.scales_col[((c0 + t) / 16) * (R / 16) + r0 / 16 + rb2] = scale2d[rb2][cb];
          }
        }
      } else {
        {
          const int c = t >> 1, h = t & 1;
          const int nbytes = rows / 2;
          if (c < cols && 16 * h < nbytes) {
            uint8_t* dst = a.codes_col + (c0 + c) * (R / 2) + r0 / 2 + 16 * h;
            const uint2* src = reinterpret_cast<const uint2*>(&colcodes[c][16 * h]);
            reinterpret_cast<uint2*>(dst)[0] = src[0];
            if (16 * h + 8 < nbytes) reinterpret_cast<uint2*>(dst)[1] = src[1];
          }
        }
        if (a.scales_col) {
          const int c = t >> 1;
          if (c < cols) {
            for (int rb2 = (t & 1); rb2 < rows / 16; rb2 += 2) {
              const int64_t gc = c0 + c, grb = r0 / 16 + rb2;
              const uint8_t sbyte = scale2d[rb2][c >> 4];
              if (gemm) a.scales_col[gemm_scale_offset(gc, grb, R / 16)] = sbyte;
              else if ((c & 15) == 0) a.scales_col[(gc / 16) * (R / 16) + grb] = sbyte;
            }
          }
        }
      }
    }
    __syncthreads();   // buf, scale2d and the staging are reused
  }
  cp_async_wait<0>();
}

// ===========================================================================
// Kernels.  Each wraps one body above with its own shared memory; the
// single-pass kernel runs an amax body and a quantize body in one launch.
// ===========================================================================
template <int NT>
__global__ void __launch_bounds__(NT) amax_plain_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t ld,
                                                        FastDiv cpr, uint32_t* __restrict__ partial) {
  pdl_entry();
  __shared__ uint32_t red[NT / 32];
  amax_plain_body<NT>(x, R, ld, cpr, partial, blockIdx.x, gridDim.x, red);
}

// The amax pass of nvfp4_amax: maxima folded into out[0..2] (zeroed first).
template <int NT>
__global__ void __launch_bounds__(NT) amax_plain_atomic_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t ld,
                                                               FastDiv cpr, uint32_t* __restrict__ out,
                                                               int32_t* status) {
  pdl_entry();
  __shared__ uint32_t red[NT / 32];
  amax_plain_body<NT>(x, R, ld, cpr, nullptr, blockIdx.x, gridDim.x, red, out, status);
}

// Threads per CTA of the rotated amax kernels (two units per thread and tile).
constexpr int kAmaxNT = 128;

template <bool ROW, bool COL>
__global__ void __launch_bounds__(kAmaxNT) amax_tile_atomic_kernel(const uint16_t* __restrict__ x, int64_t R,
                                                                   int64_t C, int64_t ld, FastDiv tiles_c,
                                                                   uint32_t ntiles, uint64_t seed,
                                                                   uint32_t* __restrict__ out, int32_t* status) {
  pdl_entry();
  __shared__ __align__(16) uint8_t ring[2 * kTileBytes];
  __shared__ uint32_t red[kAmaxNT / 32];
  amax_tile_body<ROW, COL, kAmaxNT>(x, R, C, ld, tiles_c, ntiles, seed, nullptr, nullptr, blockIdx.x, gridDim.x, ring, red,
                           out, status);
}

template <bool ROW, bool COL>
__global__ void __launch_bounds__(kAmaxNT) amax_tile_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                            int64_t ld, FastDiv tiles_c, uint32_t ntiles,
                                                            uint64_t seed, uint32_t* __restrict__ part_r,
                                                            uint32_t* __restrict__ part_c) {
  pdl_entry();
  __shared__ __align__(16) uint8_t ring[2 * kTileBytes];
  __shared__ uint32_t red[kAmaxNT / 32];
  amax_tile_body<ROW, COL, kAmaxNT>(x, R, C, ld, tiles_c, ntiles, seed, part_r, part_c, blockIdx.x, gridDim.x, ring, red);
}

template <int MODE, bool ROT, int NT, bool VEC>
__global__ void __launch_bounds__(NT) quant_rows_kernel(const QuantArgs a) {
  pdl_entry();
  __shared__ uint32_t red[NT / 32];
  __shared__ float2 tab[kScaleTab];
  quant_rows_body<MODE, ROT, NT, VEC>(a, blockIdx.x, gridDim.x, red, tab);
}

template <int MODE, bool ROT, bool ROW, bool COL, bool VEC>
__global__ void __launch_bounds__(tile_1d_threads<MODE>(), tile_1d_min_blocks<MODE>())
    quant_tile_1d_kernel(const QuantArgs a) {
  pdl_entry();
  extern __shared__ __align__(16) uint8_t tile_ring[];
  __shared__ __align__(16) TileStaging stg;
  quant_tile_1d_body<MODE, ROT, ROW, COL, VEC, tile_1d_threads<MODE>()>(a, blockIdx.x, gridDim.x, tile_ring, stg);
}

// Per-vector maxima for NVFP4_VECTOR_SCALES: max |x| (over rotated 16-blocks
// with ROT, scaled by the transform's 1/4 at the end, which commutes with
// the maximum) of every row (ROW) and / or column (COL), folded into
// vmax_r / vmax_c (float bits, zeroed by the launcher) with atomicMax; the
// largest of each orientation goes to amax_out[0] / [1] the same way.  An
// Inf or NaN sets NVFP4_ERR_NONFINITE.
template <bool ROW, bool COL, bool ROT>
__global__ void __launch_bounds__(TNT) amax_vec_kernel(const QuantArgs a) {
  pdl_entry();
  __shared__ __align__(16) uint8_t ring[2 * kTileBytes];
  __shared__ uint32_t colmax[TC];
  __shared__ uint32_t red[TNT / 32];
  auto tiles = reinterpret_cast<uint4(*)[TR][TC / 8]>(ring);
  SignMasks sm;
  if constexpr (ROT) {
    sm = sign_masks(sign_bits(philox_keys(a.seed)));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) sm.m[i] = 0u;
  }
  const float post = ROT ? 0.25f : 1.0f;
  const int t = threadIdx.x;
  const int64_t R = a.R, C = a.C;
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  const uint32_t ncta = gridDim.x;
  uint32_t hin = 0, trmax = 0, tcmax = 0;
  if (COL && t < TC) colmax[t] = 0u;
  uint32_t tile = blockIdx.x;
  int buf = 0;
  if (tile < ntiles) load_tile_async(tiles[0], a.x, R, C, a.ld, a.tiles_c_div, tile);
  for (; tile < ntiles; tile += ncta, buf ^= 1) {
    const uint32_t next = tile + ncta;
    if (next < ntiles) {
      load_tile_async(tiles[buf ^ 1], a.x, R, C, a.ld, a.tiles_c_div, next);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint4 (*sv)[TC / 8] = tiles[buf];
    int64_t tr, tc;
    tile_coords(tile, a.tiles_c_div, tr, tc);
    const int64_t r0 = tr * TR, c0 = tc * TC;
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);
    if constexpr (ROW) {
      // blocks (row, cb) and (row + 32, cb); the 8 lanes of a row then combine
      const int row = t >> 3, cb = t & 7;
      const bool va = row < rows && 16 * cb < cols, vb = row + 32 < rows && 16 * cb < cols;
      const uint4 a0 = sv[row][tile_chunk(row, 2 * cb)], a1 = sv[row][tile_chunk(row, 2 * cb + 1)];
      const uint4 b0 = sv[row + 32][tile_chunk(row + 32, 2 * cb)];
      const uint4 b1 = sv[row + 32][tile_chunk(row + 32, 2 * cb + 1)];
      const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (va) hin = __vmaxu2(hin, wa[i] & 0x7FFF7FFFu);
        if (vb) hin = __vmaxu2(hin, wb[i] & 0x7FFF7FFFu);
      }
      float2 v[16];
      unpack16x2_signed(a0, a1, b0, b1, sm, v);
      if constexpr (ROT) hadamard16x2(v);
      float ma, mb;
      max_abs16x2(v, ma, mb);
      if (!va) ma = 0.0f;
      if (!vb) mb = 0.0f;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        ma = fmaxf(ma, __shfl_xor_sync(0xFFFFFFFFu, ma, o));
        mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
      }
      const uint32_t ba = __float_as_uint(__fmul_rn(ma, post)), bb = __float_as_uint(__fmul_rn(mb, post));
      if (cb == 0) {
        if (row < rows) atomicMax(a.vmax_r + r0 + row, ba);
        if (row + 32 < rows) atomicMax(a.vmax_r + r0 + row + 32, bb);
      }
      trmax = max(trmax, max(ba, bb));
    }
    if constexpr (COL) {
      // columns (2 cp, 2 cp + 1) of row block rb, combined in shared memory
      const int cp = t & 63, rb = t >> 6;
      if (16 * rb < rows && 2 * cp < cols) {
        const uint32_t* base = reinterpret_cast<const uint32_t*>(&sv[16 * rb][0]);
        const int wofs = tile_word(16 * rb, cp);
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = base[i * (TC / 2) + wofs];
          if constexpr (!ROW) hin = __vmaxu2(hin, w & 0x7FFF7FFFu);
          v[i] = make_float2(bf16lo_flip(w, sm.m[i]), bf16hi_flip(w, sm.m[i]));
        }
        if constexpr (ROT) hadamard16x2(v);
        float mx = 0.0f, my = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          mx = fmaxf(mx, fabsf(v[i].x));
          my = fmaxf(my, fabsf(v[i].y));
        }
        atomicMax(&colmax[2 * cp], __float_as_uint(__fmul_rn(mx, post)));
        atomicMax(&colmax[2 * cp + 1], __float_as_uint(__fmul_rn(my, post)));
      }
      __syncthreads();
      if (t < TC) {
        const uint32_t m = colmax[t];
        if (t < cols) {
          atomicMax(a.vmax_c + c0 + t, m);
          tcmax = max(tcmax, m);
        }
        colmax[t] = 0u;
      }
    }
    __syncthreads();   // buf and colmax are reused
  }
  if (max(hin & 0xFFFFu, hin >> 16) >= 0x7F80u && a.status) *a.status = kStatusNonFinite;
  if (a.amax_out) {
    if constexpr (ROW) {
      const uint32_t m = block_max_u32<TNT>(trmax, red);
      if (t == 0) atomicMax(reinterpret_cast<uint32_t*>(a.amax_out), m);
    }
    if constexpr (COL) {
      const uint32_t m = block_max_u32<TNT>(tcmax, red);
      if (t == 0) atomicMax(reinterpret_cast<uint32_t*>(a.amax_out) + 1, m);
    }
  }
}

template <int MODE, bool ROW, bool COL>
__global__ void __launch_bounds__(TNT, 3) quant_tile_2d_kernel(const QuantArgs a) {
  pdl_entry();
  extern __shared__ __align__(16) uint8_t tile_ring[];
  __shared__ __align__(16) TileStaging stg;
  quant_tile_2d_body<MODE, ROW, COL>(a, blockIdx.x, gridDim.x, tile_ring, stg);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t load_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Default limit of the single-pass grid barrier's wait: 1 s.  The
// environment variable NVFP4_BARRIER_TIMEOUT_NS, read at every single-pass
// call, replaces it (the tests set it to 0 to make the wait run out).
constexpr uint64_t kBarrierTimeoutNs = 1000000000ull;

// Grid-wide barrier of a cooperative launch: every CTA's thread 0 releases
// its writes, counts itself in, and waits (at most timeout_ns) until all `n`
// CTAs are in.  The counter starts at 0 (the launcher clears it).  Returns
// false, with NVFP4_ERR_TIMEOUT in the status word, if the wait ran out; the
// caller then returns without touching its outputs (its own copies have all
// landed: every amax body ends with no cp.async group outstanding).
__device__ __forceinline__ bool grid_barrier(uint32_t* counter, uint32_t n, uint64_t timeout_ns, int32_t* status,
                                             uint32_t* ok_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(counter, 1u);
    const uint64_t t0 = global_ns();
    uint32_t ok = 1;
    while (load_acquire_gpu(counter) < n) {
      if (global_ns() - t0 >= timeout_ns) {
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    if (!ok && status) *status = kStatusTimeout;
    *ok_smem = ok;
  }
  __syncthreads();
  return *ok_smem != 0;
}

// Single pass: amax partials (one per CTA), a grid barrier, then the
// quantization, all in one cooperative launch whose CTAs are co-resident.
// For tensors that fit in L2 the quantize pass re-reads from L2, not HBM.
template <int MODE, bool ROT, bool ROW, bool COL, bool TWO_D>
__global__ void __launch_bounds__(TNT, 2) single_pass_kernel(const QuantArgs a, uint32_t* counter,
                                                              uint64_t timeout_ns) {
  pdl_entry();
  extern __shared__ __align__(16) uint8_t tile_ring[];
  __shared__ __align__(16) TileStaging stg;
  __shared__ uint32_t pass_ok;
  const uint32_t cta = blockIdx.x, ncta = gridDim.x;
  if (!(a.flags & kAlphaProvided)) {
    uint32_t* pr = const_cast<uint32_t*>(a.partials);
    uint32_t* pc = const_cast<uint32_t*>(a.partials_col);
    if constexpr (ROT) {
      amax_tile_body<ROW, COL>(a.x, a.R, a.C, a.ld, a.tiles_c_div, static_cast<uint32_t>(a.tiles_r * a.tiles_c),
                               a.seed, pr, pc, cta, ncta, tile_ring, stg.red);
    } else {
      amax_plain_body<TNT>(a.x, a.R, a.ld, a.chunks_row, pr, cta, ncta, stg.red);
    }
    if (!grid_barrier(counter, ncta, timeout_ns, a.status, &pass_ok)) return;
  }
  if constexpr (TWO_D) {
    quant_tile_2d_body<MODE, ROW, COL>(a, cta, ncta, tile_ring, stg);
  } else if constexpr (ROW && !COL) {
    quant_rows_body<MODE, ROT, TNT, false>(a, cta, ncta, stg.red, stg.tab_r);
  } else {
    quant_tile_1d_body<MODE, ROT, ROW, COL, false>(a, cta, ncta, tile_ring, stg);
  }
}

// ===========================================================================
// Host-side launchers
// ===========================================================================
static int g_sm_count[64] = {0};

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

int amax_partial_count() { return 4 * 148; }

// Workspace: the amax partials of both orientations, then (single pass) the
// grid barrier's counter in its own 16-byte slot.
// NVFP4_VECTOR_SCALES: R maxima (rounded up to 4) then C maxima.
size_t vec_workspace_bytes(int64_t R, int64_t C) {
  return static_cast<size_t>(((R + 3) & ~int64_t(3)) + ((C + 3) & ~int64_t(3))) * sizeof(uint32_t);
}

size_t quant_workspace_bytes(int64_t R, int64_t C, uint32_t flags) {
  if (flags & kVectorScales) return vec_workspace_bytes(R, C);
  if (flags & (kAlphaProvided | kAmaxProvided)) return 0;
  const size_t partials = static_cast<size_t>(2 * amax_partial_count()) * sizeof(uint32_t);
  return (flags & kSinglePass) ? partials + 16 : partials;
}

template <int MODE, bool ROT, bool VEC = false>
static cudaError_t launch_rows(const QuantArgs& a, cudaStream_t st) {
  const uint32_t pairs = (static_cast<uint32_t>(a.R) * a.nb_row.d + 1) / 2;
  const int blocks = static_cast<int>(std::min<int64_t>((pairs + 255) / 256, static_cast<int64_t>(sm_count()) * 8));
  launch_k(quant_rows_kernel<MODE, ROT, 256, VEC>, dim3(std::max(blocks, 1)), dim3(256), 0, st, 1u, a);
  note_launch();
  return cudaGetLastError();
}

template <int MODE, bool ROW, bool COL>
static cudaError_t launch_tile_2d(const QuantArgs& a, cudaStream_t st) {
  constexpr size_t smem = static_cast<size_t>(kTileStages) * kTileBytes;
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    cudaFuncSetAttribute(quant_tile_2d_kernel<MODE, ROW, COL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quant_tile_2d_kernel<MODE, ROW, COL>, TNT, smem) !=
            cudaSuccess || n <= 0)
      n = 1;
    per_sm = n;
  }
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  const int blocks = static_cast<int>(std::min<int64_t>(ntiles, static_cast<int64_t>(sm_count()) * per_sm));
  launch_k(quant_tile_2d_kernel<MODE, ROW, COL>, dim3(std::max(blocks, 1)), dim3(TNT), smem, st, 1u, a);
  note_launch();
  return cudaGetLastError();
}

template <int MODE, bool ROT, bool ROW, bool COL, bool VEC = false>
static cudaError_t launch_tile_1d(const QuantArgs& a, cudaStream_t st) {
  constexpr size_t smem = static_cast<size_t>(kTileStages) * kTileBytes;
  auto fn = quant_tile_1d_kernel<MODE, ROT, ROW, COL, VEC>;
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, tile_1d_threads<MODE>(), smem) != cudaSuccess || n <= 0) n = 1;
    per_sm = n;
  }
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  const int blocks = static_cast<int>(std::min<int64_t>(ntiles, static_cast<int64_t>(sm_count()) * per_sm));
  launch_k(fn, dim3(std::max(blocks, 1)), dim3(tile_1d_threads<MODE>()), smem, st, 1u, a);
  note_launch();
  return cudaGetLastError();
}

template <int MODE, bool ROT, bool VEC = false>
static cudaError_t dispatch_1d(const QuantArgs& a, bool row, bool col, cudaStream_t st) {
  if (row && !col) return launch_rows<MODE, ROT, VEC>(a, st);
  if (row && col) return launch_tile_1d<MODE, ROT, true, true, VEC>(a, st);
  return launch_tile_1d<MODE, ROT, false, true, VEC>(a, st);
}

// NVFP4_VECTOR_SCALES: clear the vector maxima (and amax_out), fold them in,
// then quantize with one tensor scale per row / column.
template <bool ROT>
static cudaError_t launch_amax_vec(const QuantArgs& a, bool row, bool col, cudaStream_t st) {
  const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
  const int blocks = static_cast<int>(std::min<int64_t>(ntiles, static_cast<int64_t>(sm_count()) * 4));
  if (row && col) launch_k(amax_vec_kernel<true, true, ROT>, dim3(std::max(blocks, 1)), dim3(TNT), 0, st, 1u, a);
  else if (row) launch_k(amax_vec_kernel<true, false, ROT>, dim3(std::max(blocks, 1)), dim3(TNT), 0, st, 1u, a);
  else launch_k(amax_vec_kernel<false, true, ROT>, dim3(std::max(blocks, 1)), dim3(TNT), 0, st, 1u, a);
  note_launch();
  return cudaGetLastError();
}

static cudaError_t quantize_vector_scales(QuantArgs a, int mode, bool row, bool col, bool rot, cudaStream_t st) {
  a.vmax_r = const_cast<uint32_t*>(a.partials);
  a.vmax_c = a.vmax_r + ((a.R + 3) & ~int64_t(3));
  cudaError_t e = cudaMemsetAsync(a.vmax_r, 0, vec_workspace_bytes(a.R, a.C), st);
  if (e == cudaSuccess && a.amax_out) e = cudaMemsetAsync(a.amax_out, 0, 2 * sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = rot ? launch_amax_vec<true>(a, row, col, st) : launch_amax_vec<false>(a, row, col, st);
  if (e != cudaSuccess) return e;
  switch (mode) {
    case kModeRTN:
      return rot ? dispatch_1d<kModeRTN, true, true>(a, row, col, st)
                 : dispatch_1d<kModeRTN, false, true>(a, row, col, st);
    case kModeFourSix:
      return rot ? dispatch_1d<kModeFourSix, true, true>(a, row, col, st)
                 : dispatch_1d<kModeFourSix, false, true>(a, row, col, st);
    case kModeRhtSR:
      return dispatch_1d<kModeRhtSR, true, true>(a, row, col, st);
    case kModeRhtSRHw:
      return dispatch_1d<kModeRhtSRHw, true, true>(a, row, col, st);
    default:
      return dispatch_1d<kModeMsEden, true, true>(a, row, col, st);
  }
}

template <int MODE, bool ROT, bool ROW, bool COL, bool TWO_D>
static cudaError_t launch_single_pass(QuantArgs a, cudaStream_t st) {
  auto fn = single_pass_kernel<MODE, ROT, ROW, COL, TWO_D>;
  constexpr size_t smem = static_cast<size_t>(kTileStages) * kTileBytes;   // >= the amax pass's two tiles
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, TNT, smem) != cudaSuccess || n <= 0) n = 1;
    per_sm = n;
  }
  // every CTA must be resident at once (the barrier), and each writes one
  // partial per orientation
  const int grid = std::min(sm_count() * per_sm, amax_partial_count());
  uint32_t* counter = const_cast<uint32_t*>(a.partials) + 2 * amax_partial_count();
  a.npart = grid;
  if (a.partials_col != a.partials) a.partials_col = a.partials + amax_partial_count();
  cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  uint64_t timeout_ns = kBarrierTimeoutNs;
  if (const char* env = std::getenv("NVFP4_BARRIER_TIMEOUT_NS")) {
    char* end = nullptr;
    const unsigned long long v = std::strtoull(env, &end, 10);
    if (end != env && *end == '\0') timeout_ns = v;
  }
  void* args[] = {&a, &counter, &timeout_ns};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fn), dim3(grid), dim3(TNT), args, smem, st);
  note_launch();
  return e;
}

template <int MODE, bool ROT>
static cudaError_t dispatch_single_1d(const QuantArgs& a, bool row, bool col, cudaStream_t st) {
  if (row && !col) return launch_single_pass<MODE, ROT, true, false, false>(a, st);
  if (row && col) return launch_single_pass<MODE, ROT, true, true, false>(a, st);
  return launch_single_pass<MODE, ROT, false, true, false>(a, st);
}

// Launch the amax pass: rows into partials[0, npart), columns (rotated
// only) into partials[npart, 2 npart).  Plain amax is shared by both
// orientations.
static cudaError_t launch_amax(const QuantArgs& a, bool row, bool col, bool rot, cudaStream_t st) {
  const int np = a.npart;
  uint32_t* pr = const_cast<uint32_t*>(a.partials);
  uint32_t* pc = const_cast<uint32_t*>(a.partials_col);
  if (!rot) {
    launch_k(amax_plain_kernel<256>, dim3(np), dim3(256), 0, st, 1u, a.x, a.R, a.ld, a.chunks_row, pr);
  } else {
    const uint32_t ntiles = static_cast<uint32_t>(a.tiles_r * a.tiles_c);
    const FastDiv tcd = a.tiles_c_div;
    if (row && col)
      launch_k(amax_tile_kernel<true, true>, dim3(np), dim3(kAmaxNT), 0, st, 1u, a.x, a.R, a.C, a.ld, tcd, ntiles, a.seed, pr, pc);
    else if (row)
      launch_k(amax_tile_kernel<true, false>, dim3(np), dim3(kAmaxNT), 0, st, 1u, a.x, a.R, a.C, a.ld, tcd, ntiles, a.seed, pr, pc);
    else
      launch_k(amax_tile_kernel<false, true>, dim3(np), dim3(kAmaxNT), 0, st, 1u, a.x, a.R, a.C, a.ld, tcd, ntiles, a.seed, pr, pc);
  }
  note_launch();
  return cudaGetLastError();
}

// nvfp4_amax: out[0..2] (plain, rotated rows, rotated columns) cleared, then
// one pass folds every CTA's maxima into them.
cudaError_t amax_launch(const void* x, int64_t R, int64_t C, int64_t ld, uint32_t flags, uint64_t seed,
                        float* amax_out, int32_t* status, cudaStream_t st) {
  uint32_t* out = reinterpret_cast<uint32_t*>(amax_out);
  cudaError_t e = cudaMemsetAsync(out, 0, 3 * sizeof(uint32_t), st);
  if (e != cudaSuccess || R == 0 || C == 0) return e;
  const bool rot = (flags & kRht) != 0;
  const bool row = rot && (flags & kRowwise), col = rot && (flags & kColwise);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  const int np = amax_partial_count();
  if (!row && !col) {
    launch_k(amax_plain_atomic_kernel<256>, dim3(np), dim3(256), 0, st, 1u, xs, R, ld,
             make_fastdiv(static_cast<uint32_t>(C / 8)), out, status);
  } else {
    const int64_t tiles_r = (R + TR - 1) / TR, tiles_c = (C + TC - 1) / TC;
    const uint32_t ntiles = static_cast<uint32_t>(tiles_r * tiles_c);
    const FastDiv tcd = make_fastdiv(static_cast<uint32_t>(tiles_c));
    if (row && col)
      launch_k(amax_tile_atomic_kernel<true, true>, dim3(np), dim3(kAmaxNT), 0, st, 1u, xs, R, C, ld, tcd, ntiles, seed,
               out, status);
    else if (row)
      launch_k(amax_tile_atomic_kernel<true, false>, dim3(np), dim3(kAmaxNT), 0, st, 1u, xs, R, C, ld, tcd, ntiles, seed,
               out, status);
    else
      launch_k(amax_tile_atomic_kernel<false, true>, dim3(np), dim3(kAmaxNT), 0, st, 1u, xs, R, C, ld, tcd, ntiles, seed,
               out, status);
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t quantize_launch(const void* x, int64_t R, int64_t C, int64_t ld, int mode, uint32_t flags,
                            uint64_t seed, uint32_t stream_id, const float* alpha_in,
                            const QuantOutputs& o, void* workspace, cudaStream_t st) {
  QuantArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.R = R;
  a.C = C;
  a.ld = ld;
  a.seed = seed;
  a.stream_id = stream_id;
  a.flags = flags;
  a.alpha_in = alpha_in;
  a.npart = amax_partial_count();
  a.partials = static_cast<const uint32_t*>(workspace);
  a.partials_col = a.partials;
  a.codes_row = o.codes_row;
  a.scales_row = o.scales_row;
  a.alpha_row = o.alpha_row;
  a.codes_col = o.codes_col;
  a.scales_col = o.scales_col;
  a.alpha_col = o.alpha_col;
  a.amax_out = o.amax_out;
  a.status = o.status;
  a.nb_row = make_fastdiv(static_cast<uint32_t>(C / 16));
  a.tiles_r = (R + TR - 1) / TR;
  a.tiles_c = (C + TC - 1) / TC;
  a.tiles_c_div = make_fastdiv(static_cast<uint32_t>(a.tiles_c > 0 ? a.tiles_c : 1));
  a.chunks_row = make_fastdiv(static_cast<uint32_t>(C / 8 > 0 ? C / 8 : 1));
  const bool row = flags & kRowwise, col = flags & kColwise, two_d = flags & kBlock2D;
  const bool rot = (mode == kModeRhtSR || mode == kModeMsEden || mode == kModeRhtSRHw || (flags & kRht)) && !two_d;
  if (rot) a.partials_col = a.partials + a.npart;
  a.amax_rot = rot ? 1 : 0;
  if (R == 0 || C == 0) return cudaSuccess;
  if (flags & kVectorScales) return quantize_vector_scales(a, mode, row, col, rot, st);

  if ((flags & kSinglePass) && !(flags & kAlphaProvided)) {
    if (two_d) {
      if (mode == kModeRTN) {
        if (row && col) return launch_single_pass<kModeRTN, false, true, true, true>(a, st);
        if (row) return launch_single_pass<kModeRTN, false, true, false, true>(a, st);
        return launch_single_pass<kModeRTN, false, false, true, true>(a, st);
      }
      if (row && col) return launch_single_pass<kModeFourSix, false, true, true, true>(a, st);
      if (row) return launch_single_pass<kModeFourSix, false, true, false, true>(a, st);
      return launch_single_pass<kModeFourSix, false, false, true, true>(a, st);
    }
    switch (mode) {
      case kModeRTN:
        return rot ? dispatch_single_1d<kModeRTN, true>(a, row, col, st)
                   : dispatch_single_1d<kModeRTN, false>(a, row, col, st);
      case kModeFourSix:
        return rot ? dispatch_single_1d<kModeFourSix, true>(a, row, col, st)
                   : dispatch_single_1d<kModeFourSix, false>(a, row, col, st);
      case kModeRhtSR:
        return dispatch_single_1d<kModeRhtSR, true>(a, row, col, st);
      case kModeRhtSRHw:
        return dispatch_single_1d<kModeRhtSRHw, true>(a, row, col, st);
      default:
        return dispatch_single_1d<kModeMsEden, true>(a, row, col, st);
    }
  }

  if (!(flags & (kAlphaProvided | kAmaxProvided))) {
    cudaError_t e = launch_amax(a, row || two_d, col && !two_d, rot, st);
    if (e != cudaSuccess) return e;
  }
  if (two_d) {
    if (mode == kModeRTN) {
      if (row && col) return launch_tile_2d<kModeRTN, true, true>(a, st);
      if (row) return launch_tile_2d<kModeRTN, true, false>(a, st);
      return launch_tile_2d<kModeRTN, false, true>(a, st);
    }
    if (row && col) return launch_tile_2d<kModeFourSix, true, true>(a, st);
    if (row) return launch_tile_2d<kModeFourSix, true, false>(a, st);
    return launch_tile_2d<kModeFourSix, false, true>(a, st);
  }
  switch (mode) {
    case kModeRTN:
      return rot ? dispatch_1d<kModeRTN, true>(a, row, col, st) : dispatch_1d<kModeRTN, false>(a, row, col, st);
    case kModeFourSix:
      return rot ? dispatch_1d<kModeFourSix, true>(a, row, col, st)
                 : dispatch_1d<kModeFourSix, false>(a, row, col, st);
    case kModeRhtSR:
      return dispatch_1d<kModeRhtSR, true>(a, row, col, st);
    case kModeRhtSRHw:
      return dispatch_1d<kModeRhtSRHw, true>(a, row, col, st);
    default:
      return dispatch_1d<kModeMsEden, true>(a, row, col, st);
  }
}

}  // namespace nvfp4
