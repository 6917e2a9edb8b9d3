// nvfp4_device.cuh -- device-side building blocks of the NVFP4 quantizer.
//
// Every floating-point step is one IEEE binary32 operation with round to
// nearest even, written with the explicit __f*_rn intrinsics so the compiler
// cannot contract or reorder it; the whole library is also built with
// -fmad=false.  The encoders follow:
//   * Four Over Six (Chinese translation), §2.1 Eq. 1-3: tensor scale, block
//     scale, element rounding; §1 Table 1: the 4/6 selector.
//   * NVFP4 pretraining write-up, §一 (E2M1 values, E4M3 block scales per 16
//     values, FP32 tensor scale), §二 (random Hadamard transform, 2D blocks,
//     stochastic rounding), §四 (hardware conversions with round-to-nearest-even).
//   * Quartet II / MS-EDEN write-up, §一: rotate, round values to nearest,
//     randomness on the E4M3 scale only.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11).  The ten round keys depend only on the seed, so a thread expands
// them once and each draw costs ten rounds of two wide multiplies and two
// three-input XORs.
// ---------------------------------------------------------------------------
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys K;
  uint32_t a = static_cast<uint32_t>(seed), b = static_cast<uint32_t>(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = a;
    K.k1[r] = b;
    a += 0x9E3779B9u;
    b += 0xBB67AE85u;
  }
  return K;
}

__device__ __forceinline__ uint4 philox(const PhiloxKeys& K, uint32_t c0, uint32_t c1,
                                        uint32_t c2, uint32_t c3) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    c0 = hi1 ^ c1 ^ K.k0[r];
    c1 = lo1;
    c2 = hi0 ^ c3 ^ K.k1[r];
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// Counter words of the quantizer's draws: (unit_lo, unit_hi, c2, tag).
constexpr uint32_t kTagValueSR = 1u;   // 16-bit fields for element rounding
constexpr uint32_t kTagScaleSR = 2u;   // 24-bit field for the E4M3 scale
constexpr uint32_t kTagSigns = 3u;     // the sign diagonal of the rotation
constexpr uint32_t kTagValueSRHw = 4u; // one word per 4 elements for the hardware SR convert

// ---------------------------------------------------------------------------
// bf16 <-> f32
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// The same with the sign flipped where m = 0x80000000 (m is 0 or bit 31).
// Adding bit 31 modulo 2^32 flips it exactly as an exclusive or does, and a
// shift followed by an add is one instruction; the high half masks and
// flips in one three-input logic operation.
__device__ __forceinline__ float bf16lo_flip(uint32_t w, uint32_t m) { return __uint_as_float((w << 16) + m); }
__device__ __forceinline__ float bf16hi_flip(uint32_t w, uint32_t m) { return __uint_as_float((w & 0xFFFF0000u) ^ m); }

// 8 bf16 packed in a uint4 -> 8 floats
__device__ __forceinline__ void unpack8(const uint4 u, float* v) {
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x);
  v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z);
  v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}

// ---------------------------------------------------------------------------
// E4M3 block scales (OCP E4M3FN, non-negative): 127 finite codes, max 448.
// ---------------------------------------------------------------------------
// Normal codes (b >= 8): exponent and mantissa bits move up as one field and
// the exponent is rebiased from 7 to 127 (+120 << 3 before the shift).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  return (b >= 8u) ? __uint_as_float((b + (120u << 3)) << 20)
                   : __fmul_rn(static_cast<float>(b), 0.001953125f);  // b * 2^-9, exact
}

// Round to nearest even, saturating at 448 (hardware conversion; PTX
// cvt.rn.satfinite.e4m3x2.f32).  v >= 0.
__device__ __forceinline__ uint32_t e4m3_rne(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Smallest E4M3 value not below v (saturating at 448).  v >= 0.
__device__ __forceinline__ uint32_t e4m3_ceil(float v) {
  uint32_t b = e4m3_rne(v);
  if (b < 0x7Eu && e4m3_value(b) < v) ++b;
  return b;
}

// Stochastic rounding to E4M3 with a 24-bit uniform: up iff u24 < f * 2^24,
// f the position of v between its lower neighbour lo and the next value.
// v >= 0 (saturating at 448).
//   E4M3 normal range [2^-6, 448): the FP32 value truncated to 3 mantissa
//   bits is lo, so lo's code is the top bits of v, (exponent << 3 | m3)
//   rebiased from 127 to 7, and f * 2^24 is the 20 dropped mantissa bits
//   times 16 (an exact integer).
//   Subnormal range [0, 2^-6): the grid step is 2^-9, so with t = 512 v
//   (exact) lo = floor(t) and f = t - lo, both exact.
__device__ __forceinline__ uint32_t e4m3_sr(float v, uint32_t u24) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t lo_n = (b >> 20) - (120u << 3);
  const uint32_t up_n = (u24 < ((b & 0xFFFFFu) << 4)) ? 1u : 0u;
  const float t = __fmul_rn(v, 512.0f);
  const float fl = floorf(t);
  const uint32_t up_s = (static_cast<float>(u24) < __fmul_rn(__fsub_rn(t, fl), 16777216.0f)) ? 1u : 0u;
  // selects rather than early returns: no divergent branch per block
  const uint32_t r = (v >= 0.015625f) ? lo_n + up_n : static_cast<uint32_t>(fl) + up_s;
  return (v < 448.0f) ? r : 0x7Eu;
}

// ---------------------------------------------------------------------------
// E2M1 values: codes sign | index into {0, .5, 1, 1.5, 2, 3, 4, 6}.
// ---------------------------------------------------------------------------
// Byte of two codes -> their two signed grid values (PTX cvt.rn.f16x2.e2m1x2,
// exact), widened to float.
__device__ __forceinline__ void e2m1x2_values(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2) : "r"(byte));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// Stochastic rounding of y to the grid with a 16-bit uniform u16: with the
// grid step 1/m on |y|'s segment ([0,2): 0.5, [2,4): 1, [4,6]: 2), t = |y| m
// is exact, f = t - floor(t) is the position between the neighbours, and the
// magnitude rounds up iff u16 < f * 65536.  |y| >= 6 -> 6.  Returns the
// signed grid value (exactly representable, so its encoding is exact).
// Branch-free: the segment's m and 1 / m (powers of two) are selected.
__device__ __forceinline__ float e2m1_sr_value_nb(float y, uint32_t u16) {
  const float a = fabsf(y);
  const bool lt2 = a < 2.0f, lt4 = a < 4.0f;
  const float m = lt2 ? 2.0f : (lt4 ? 1.0f : 0.5f);
  const float inv_m = lt2 ? 0.5f : (lt4 ? 1.0f : 2.0f);
  const float t = __fmul_rn(a, m);
  const float fl = floorf(t);
  const float f = __fsub_rn(t, fl);
  // (float) u16 from the exact float 2^23 + u16, keeping the integer
  // conversion unit out of the per-element path
  const float fu = __fsub_rn(__uint_as_float(0x4B000000u | u16), 8388608.0f);
  const float up = (fu < __fmul_rn(f, 65536.0f)) ? 1.0f : 0.0f;
  const float q = (a >= 6.0f) ? 6.0f : __fmul_rn(__fadd_rn(fl, up), inv_m);
  return copysignf(q, y);
}

// Four values stochastically rounded to E2M1 by the sm_100a convert with
// caller random bits: a lands in bits 15:12, d in bits 3:0.  Each input draws
// its own 16-bit field from `rbits`; it rounds up when that field plus its
// fraction between grid points, scaled by 2^16, reaches 2^16.  Magnitudes of
// 6 and above saturate to 6.
__device__ __forceinline__ uint32_t e2m1x4_sr_hw(float a, float b, float c, float d, uint32_t rbits) {
  uint16_t r;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=h"(r) : "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbits));
  return r;
}

// ---------------------------------------------------------------------------
// 16-wide Hadamard butterfly, natural (Sylvester) order, strides 1, 2, 4, 8.
// The forward transform is r = (1/4) H16 D v, D flipping the signs selected
// by `signs` (lane-paired below); the inverse is x = D (1/4) H16 r.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void irht16(float* v, uint32_t signs) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i)
    v[i] = __uint_as_float(__float_as_uint(__fmul_rn(v[i], 0.25f)) ^ (((signs >> i) & 1u) << 31));
}

// ---------------------------------------------------------------------------
// Lane-paired arithmetic: two independent blocks share each float2 (x = the
// first block's element, y = the second's), so one packed sm_100 instruction
// does the work of two.  Each component is rounded exactly as the scalar
// __f*_rn operation.
// sub2 forms a - b as fma(b, -1, a): the product b * -1 is exact, so the one
// rounding gives RN(a - b), signed zeros included.  It is for operands that
// are sums (the butterflies): when b is itself a product, the compiler may
// fold the two into one fma and drop the product's rounding, so a - RN(p)
// uses sub2_exact (two scalar subtractions, which are never merged).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// 1.0f that the code generator cannot treat as a constant: its sign and
// exponent bits are ORed with %nsmid >> 31 (the SM count is a launch-time
// value below 2^31, so the bit is always 0).  Hoisted: one read per kernel.
__device__ __forceinline__ float opaque_one() {
  uint32_t n;
  asm("mov.u32 %0, %%nsmid;" : "=r"(n));
  return __uint_as_float(0x3F800000u | (n >> 31));
}
__device__ __forceinline__ float2 fma2_ptx(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}
// a + p, packed, for a product p that must keep its own rounding:
// fma(p, 1, a) adds exactly (p * 1 is exact) with one rounding, and with the
// factor opaque the code generator can neither drop it nor merge p's
// multiply into the fma (measured on sm_100a: with a literal 1.0 it does
// both, and it also merges into add.rn.f32x2 / sub.rn.f32x2).
__device__ __forceinline__ float2 add2_prod(float2 a, float2 p) {
  const float u = opaque_one();
  return fma2_ptx(p, make_float2(u, u), a);
}
__device__ __forceinline__ float2 sub2_exact(float2 a, float2 b) {
  return make_float2(__fsub_rn(a.x, b.x), __fsub_rn(a.y, b.y));
}

// Sign masks of the rotation's diagonal: bit 31 set where element i flips.
struct SignMasks {
  uint32_t m[16];
};
__device__ __forceinline__ SignMasks sign_masks(uint32_t signs) {
  SignMasks s;
#pragma unroll
  for (int i = 0; i < 16; ++i) s.m[i] = ((signs >> i) & 1u) << 31;
  return s;
}

// Two blocks of 16 bf16 (a0/a1: first block's halves, b0/b1: second's) ->
// lane-paired floats with the diagonal's signs applied.
__device__ __forceinline__ void unpack16x2_signed(const uint4 a0, const uint4 a1, const uint4 b0, const uint4 b1,
                                                  const SignMasks& sm, float2* v) {
  const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = make_float2(bf16lo_flip(wa[j], sm.m[2 * j]), bf16lo_flip(wb[j], sm.m[2 * j]));
    v[2 * j + 1] = make_float2(bf16hi_flip(wa[j], sm.m[2 * j + 1]), bf16hi_flip(wb[j], sm.m[2 * j + 1]));
  }
}

// H16 v for two lane-paired blocks (signs already applied): the butterfly
// without the final 1/4.
__device__ __forceinline__ void hadamard16x2(float2* v) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const float2 a = v[i], b = v[i + h];
        v[i] = add2(a, b);
        v[i + h] = sub2(a, b);
      }
    }
  }
}

// (1/4) H16 v of two lane-paired blocks whose signs are already applied.
__device__ __forceinline__ void rht16x2_presigned(float2* v) {
  hadamard16x2(v);
  const float2 q = make_float2(0.25f, 0.25f);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], q);
}

// ---------------------------------------------------------------------------
// Block encoding (one 16-vector).  Codes come back packed: byte j of `lo`
// (j < 4) holds elements 2j, 2j+1; `hi` holds elements 8..15.
// ---------------------------------------------------------------------------
// Byte offset of the scale of (row m, K-block j (16 elements for NVFP4, 32 for MXFP4)) in the tcgen05 block-scale
// layout: 512-byte atoms of 128 rows x 4 K-blocks, K-atoms fastest; inside an
// atom, row m % 32 selects a 16-byte line and (m / 32) % 4 a 4-byte word.
__device__ __forceinline__ int64_t gemm_scale_offset(int64_t m, int64_t j, int64_t kblocks) {
  return ((m >> 7) * (kblocks >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3);
}
// The same in 32-bit arithmetic, for scale arrays below 4 GB.
__device__ __forceinline__ uint32_t gemm_scale_offset32(uint32_t m, uint32_t j, uint32_t kblocks) {
  return ((m >> 7) * (kblocks >> 2) + (j >> 2)) * 512u + (m & 31u) * 16u + ((m >> 5) & 3u) * 4u + (j & 3u);
}

// The layout split over a 64 x 128 tile (r0 = 64 tr, c0 = 128 tc).  Row
// orientation (kb = C / 16 blocks per row), the block of tile row r < 32 and
// tile block column cb: tile part + thread part, and row r + 32 is 4 bytes
// further on; column orientation (kb = R / 16), tile column c: the four
// scale bytes of row blocks 0..3 are the 4-byte word at tile part + thread
// part.
__device__ __forceinline__ int64_t gemm_scale_tile_row(int64_t tr, int64_t tc, int64_t kb) {
  return ((tr >> 1) * (kb >> 2) + 2 * tc) * 512 + (tr & 1) * 8;
}
__device__ __forceinline__ uint32_t gemm_scale_thread_row(int r, int cb) {
  return static_cast<uint32_t>((cb >> 2) * 512 + (cb & 3) + (r & 31) * 16);
}
__device__ __forceinline__ int64_t gemm_scale_tile_col(int64_t tr, int64_t tc, int64_t kb) {
  return (tc * (kb >> 2) + tr) * 512;
}
__device__ __forceinline__ uint32_t gemm_scale_thread_col(int c) {
  return static_cast<uint32_t>((c & 31) * 16 + ((c >> 5) & 3) * 4);
}

struct Packed16 {
  uint32_t lo, hi;
};

// Eq. 2: Delta_raw = amax_b / (alpha * M); the E4M3 rounding is chosen by the
// caller.  A zero denominator gives 0.
__device__ __forceinline__ float scale_raw(float amax_b, float alpha, float M) {
  const float den = __fmul_rn(alpha, M);
  return (den == 0.0f) ? 0.0f : __fdiv_rn(amax_b, den);
}

// ---------------------------------------------------------------------------
// Eight values <-> one word of eight E2M1 codes (element k in bits 4k..4k+3).
// Encoding rounds to nearest even with saturation at +-6 (PTX
// cvt.rn.satfinite.e2m1x2.f32, two values per byte); decoding is exact.
// ---------------------------------------------------------------------------
// Two values -> one byte of codes, y_lo in the low nibble (PTX
// cvt.rn.satfinite.e2m1x2.f32 takes the high element first), returned
// through a 32-bit register.
__device__ __forceinline__ uint32_t e2m1x2_rne(float y_lo, float y_hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(y_lo), "f"(y_hi));
  return r;
}

// Eight values -> one word: four conversions whose bytes are packed inside
// the asm block (a vector mov that builds the word from four .b8 registers;
// only the opposite direction, splitting a word into .b8 registers, is
// avoided, see e2m1x2_to_f16x2).
__device__ __forceinline__ uint32_t e2m1x8_rne(float y0, float y1, float y2, float y3, float y4, float y5,
                                               float y6, float y7) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
  return r;
}

// Each byte is taken out of the word in C++ and handed to the convert through
// a 32-bit register (cvt.u8.u32 inside the asm): unpacking the word into four
// .b8 registers inside one asm block decoded bytes 2 and 3 as zeros in some
// inlining contexts on sm_100a, so this form is used throughout.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2) : "r"(byte));
  return h2;
}

__device__ __forceinline__ void e2m1x8_values(uint32_t w, float* q) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t h2 = e2m1x2_to_f16x2((w >> (8 * k)) & 0xFFu);
    q[2 * k] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    q[2 * k + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
  }
}

// Sign-only codes (magnitude 0) of one lane of sixteen pairs.
template <bool Y>
__device__ __forceinline__ Packed16 sign_codes16(const float2* v) {
  Packed16 p{0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t sign = (__float_as_uint(Y ? v[i].y : v[i].x) >> 31) << 3;
    if (i < 8) p.lo |= sign << (4 * i);
    else p.hi |= sign << (4 * (i - 8));
  }
  return p;
}

// Eq. 3 with round to nearest for two lane-paired blocks with scale bytes sba
// (x) and sbb (y): codes of v times the correctly rounded 1 / (alpha Delta).
// When alpha Delta is 0, or its reciprocal overflows, the magnitudes are 0
// and the codes keep the signs of v.
__device__ __forceinline__ void encode_rne_x2(const float2* v, float alpha, uint32_t sba, uint32_t sbb,
                                              Packed16& pa, Packed16& pb) {
  const float ra = __frcp_rn(__fmul_rn(alpha, e4m3_value(sba)));
  const float rb = __frcp_rn(__fmul_rn(alpha, e4m3_value(sbb)));
  const float2 r2 = make_float2(ra, rb);
  float2 y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = mul2(v[i], r2);
  pa.lo = e2m1x8_rne(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x);
  pa.hi = e2m1x8_rne(y[8].x, y[9].x, y[10].x, y[11].x, y[12].x, y[13].x, y[14].x, y[15].x);
  pb.lo = e2m1x8_rne(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y);
  pb.hi = e2m1x8_rne(y[8].y, y[9].y, y[10].y, y[11].y, y[12].y, y[13].y, y[14].y, y[15].y);
  if (isinf(ra)) pa = sign_codes16<false>(v);
  if (isinf(rb)) pb = sign_codes16<true>(v);
}

// Eight values -> one word of codes and their grid values: each converted
// byte is decoded from its .b8 register in the same asm block
// (cvt.rn.f16x2.e2m1x2, exact), so the word is never taken apart again.
// h[k] holds the values of elements 2k, 2k + 1 as f16x2.
__device__ __forceinline__ uint32_t e2m1x8_rne_dec(float y0, float y1, float y2, float y3, float y4, float y5,
                                                   float y6, float y7, uint32_t* h) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %8, %7;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %10, %9;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %12, %11;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, t0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, t1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, t2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %4, t3;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
  return r;
}

__device__ __forceinline__ float f16_lo(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// Codes of two lane-paired blocks v * rinv (as encode_x2) and their grid
// values q, lane-paired.
__device__ __forceinline__ void encode_decode_x2(const float2* v, float2 rinv2, Packed16& pa, Packed16& pb,
                                                 float2* q) {
  float2 y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = mul2(v[i], rinv2);
  uint32_t ha[8], hb[8];
  pa.lo = e2m1x8_rne_dec(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x, ha);
  pa.hi = e2m1x8_rne_dec(y[8].x, y[9].x, y[10].x, y[11].x, y[12].x, y[13].x, y[14].x, y[15].x, ha + 4);
  pb.lo = e2m1x8_rne_dec(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y, hb);
  pb.hi = e2m1x8_rne_dec(y[8].y, y[9].y, y[10].y, y[11].y, y[12].y, y[13].y, y[14].y, y[15].y, hb + 4);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    q[2 * k] = make_float2(f16_lo(ha[k]), f16_lo(hb[k]));
    q[2 * k + 1] = make_float2(f16_hi(ha[k]), f16_hi(hb[k]));
  }
}

// Grid values of two blocks' codes, lane-paired.
__device__ __forceinline__ void decode16x2(const Packed16& pa, const Packed16& pb, float2* q) {
  float a[16], b[16];
  e2m1x8_values(pa.lo, a);
  e2m1x8_values(pa.hi, a + 8);
  e2m1x8_values(pb.lo, b);
  e2m1x8_values(pb.hi, b + 8);
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = make_float2(a[i], b[i]);
}

// Pairwise sum of 16 terms with strides 8, 4, 2, 1 (the stated summation
// order), two lane-paired blocks at a time.  The packed multiply that
// made e[] may be contracted with a packed add into one fma (measured: the
// rounding of d * d vanished from 4/6 errors), so the first level, which
// consumes the products, adds with the scalar __fadd_rn, which is never
// merged (or, with PACKED, with add2_prod); the later levels add sums only.
// PACKED measured faster for the MS-EDEN sums (225 vs 229 us for the dY
// rows + columns kernel) and slower for the 4/6 errors (the packed fma
// loads the busier FMA pipe).
template <bool PACKED = false>
__device__ __forceinline__ float2 sum16x2(const float2* e) {
  float2 t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    t[i] = PACKED ? add2_prod(e[i + 8], e[i])
                  : make_float2(__fadd_rn(e[i].x, e[i + 8].x), __fadd_rn(e[i].y, e[i + 8].y));
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = add2(t[i], t[i + 4]);
#pragma unroll
  for (int i = 0; i < 2; ++i) t[i] = add2(t[i], t[i + 2]);
  return add2(t[0], t[1]);
}

// Squared error of two lane-paired encodings in the original domain,
// e_i = (v_i - q_i s)^2 summed with sum16x2.
__device__ __forceinline__ float2 sq_error_x2(const float2* v, float alpha, uint32_t sba, uint32_t sbb,
                                              const Packed16& pa, const Packed16& pb) {
  const float2 s2 = make_float2(__fmul_rn(alpha, e4m3_value(sba)), __fmul_rn(alpha, e4m3_value(sbb)));
  float2 q[16], e[16];
  decode16x2(pa, pb, q);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 d = sub2_exact(v[i], mul2(q[i], s2));
    e[i] = mul2(d, d);
  }
  return sum16x2(e);
}

// max(|a|, |b|, |c|) and max(a, b, c) in one instruction each (the sm_100
// three-input max.f32; the absolute values are operand modifiers).
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float r;
  asm("{\n\t.reg .f32 x, y, z;\n\t"
      "abs.f32 x, %1;\n\tabs.f32 y, %2;\n\tabs.f32 z, %3;\n\t"
      "max.f32 %0, x, y, z;\n\t}"
      : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Block maxima of |v| for two lane-paired blocks: 16 values in three levels
// of three-input maxima (5 + 2 + 1 instructions per block); max is exact, so
// the order does not matter.
__device__ __forceinline__ void max_abs16x2(const float2* v, float& ma, float& mb) {
  float a[6], b[6];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    a[i] = max3_abs(v[3 * i].x, v[3 * i + 1].x, v[3 * i + 2].x);
    b[i] = max3_abs(v[3 * i].y, v[3 * i + 1].y, v[3 * i + 2].y);
  }
  a[5] = max3_abs(a[3], a[4], v[15].x);
  b[5] = max3_abs(b[3], b[4], v[15].y);
  ma = fmaxf(max3(a[0], a[1], a[2]), a[5]);
  mb = fmaxf(max3(b[0], b[1], b[2]), b[5]);
}

// Round-to-nearest block quantization of two lane-paired blocks (Four Over
// Six §2.1 Eq. 2-3): scale for M = 6 (or, with four_six, the better of the
// M = 6 and M = 4 candidates by squared error in the original domain, ties
// to M = 6; §1 Table 1), then the E2M1 codes.
template <bool FOUR_SIX>
__device__ __forceinline__ void quantize_pair_rne(const float2* v, float alpha, Packed16& pa, Packed16& pb,
                                                  uint32_t& sba, uint32_t& sbb) {
  float ma, mb;
  max_abs16x2(v, ma, mb);
  if constexpr (!FOUR_SIX) {
    sba = e4m3_rne(scale_raw(ma, alpha, 6.0f));
    sbb = e4m3_rne(scale_raw(mb, alpha, 6.0f));
    encode_rne_x2(v, alpha, sba, sbb, pa, pb);
  } else {
    const uint32_t a6 = e4m3_rne(scale_raw(ma, alpha, 6.0f)), b6 = e4m3_rne(scale_raw(mb, alpha, 6.0f));
    const uint32_t a4 = e4m3_rne(scale_raw(ma, alpha, 4.0f)), b4 = e4m3_rne(scale_raw(mb, alpha, 4.0f));
    Packed16 pa6, pb6, pa4, pb4;
    encode_rne_x2(v, alpha, a6, b6, pa6, pb6);
    encode_rne_x2(v, alpha, a4, b4, pa4, pb4);
    const float2 e6 = sq_error_x2(v, alpha, a6, b6, pa6, pb6);
    const float2 e4 = sq_error_x2(v, alpha, a4, b4, pa4, pb4);
    const bool ta = e4.x < e6.x, tb = e4.y < e6.y;
    sba = ta ? a4 : a6;
    pa = ta ? pa4 : pa6;
    sbb = tb ? b4 : b6;
    pb = tb ? pb4 : pb6;
  }
}

// ---------------------------------------------------------------------------
// Table-driven block encoding.  For a fixed tensor scale alpha the element
// scale of Eq. 3, s = RN(alpha * Delta), and its reciprocal take one of 128
// values (one per E4M3 byte), so each CTA tabulates them once: entry b holds
// {s, rinv} with rinv = RN(1 / s), or 0 where s = 0 or 1 / s overflows (the
// block then encodes as signed zeros, as Eq. 3's reading requires).  A block
// reads one entry instead of decoding its scale byte and rounding a
// reciprocal; the values are the same IEEE results.
// ---------------------------------------------------------------------------
constexpr int kScaleTab = 128;

__device__ __forceinline__ float2 scale_entry(float alpha, uint32_t b) {
  const float s = __fmul_rn(alpha, e4m3_value(b));
  float r = (s == 0.0f) ? 0.0f : __frcp_rn(s);
  if (isinf(r)) r = 0.0f;
  return make_float2(s, r);
}

// Fill tab[0..127] (shared memory) for tensor scale alpha; the caller
// synchronises the CTA before reading it.
template <int NT>
__device__ __forceinline__ void build_scale_tab(float2* tab, float alpha) {
  for (int b = threadIdx.x; b < kScaleTab; b += NT) tab[b] = scale_entry(alpha, static_cast<uint32_t>(b));
}

// Two values rounded to E4M3 (nearest even, saturating at 448) in one
// conversion: a in the low byte, b in the next.  a, b >= 0.
__device__ __forceinline__ uint32_t e4m3x2_rne(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// Smallest E4M3 value not below each of a, b (saturating at 448).
__device__ __forceinline__ void e4m3x2_ceil(float a, float b, uint32_t& ba, uint32_t& bb) {
  const uint32_t r = e4m3x2_rne(a, b);
  ba = r & 0xFFu;
  bb = r >> 8;
  if (ba < 0x7Eu && e4m3_value(ba) < a) ++ba;
  if (bb < 0x7Eu && e4m3_value(bb) < b) ++bb;
}

// Scale contexts of the block encoders.  A context gives, for the two
// lane-paired blocks (x: block a, y: block b), their tensor scales alpha2,
// the Eq. 2 denominators RN(alpha * 6) and RN(alpha * 4), and the entry
// {s, rinv} of a scale byte.
// TabScales: one tensor scale for both blocks, entries from the CTA's table.
struct TabScales {
  const float2* tab;
  float alpha, den6, den4;
  __device__ __forceinline__ float2 alpha2() const { return make_float2(alpha, alpha); }
  __device__ __forceinline__ float2 d6() const { return make_float2(den6, den6); }
  __device__ __forceinline__ float2 d4() const { return make_float2(den4, den4); }
  __device__ __forceinline__ float2 ent_a(uint32_t b) const { return tab[b]; }
  __device__ __forceinline__ float2 ent_b(uint32_t b) const { return tab[b]; }
};

__device__ __forceinline__ TabScales make_scale_ctx(const float2* tab, float alpha) {
  return TabScales{tab, alpha, __fmul_rn(alpha, 6.0f), __fmul_rn(alpha, 4.0f)};
}

// VecScales: a tensor scale per block (one per row or column of the tensor);
// entries are computed per block.
struct VecScales {
  float2 alpha, den6, den4;
  __device__ __forceinline__ float2 alpha2() const { return alpha; }
  __device__ __forceinline__ float2 d6() const { return den6; }
  __device__ __forceinline__ float2 d4() const { return den4; }
  __device__ __forceinline__ float2 ent_a(uint32_t b) const { return scale_entry(alpha.x, b); }
  __device__ __forceinline__ float2 ent_b(uint32_t b) const { return scale_entry(alpha.y, b); }
};

__device__ __forceinline__ VecScales make_vec_scales(float alpha_a, float alpha_b) {
  return VecScales{make_float2(alpha_a, alpha_b), make_float2(__fmul_rn(alpha_a, 6.0f), __fmul_rn(alpha_b, 6.0f)),
                   make_float2(__fmul_rn(alpha_a, 4.0f), __fmul_rn(alpha_b, 4.0f))};
}

// Eq. 2's quotient amax_b / den (0 when den is 0).
__device__ __forceinline__ float scale_quot(float amax_b, float den) {
  const float q = __fdiv_rn(amax_b, den);   // computed either way: a select, not a branch
  return (den == 0.0f) ? 0.0f : q;
}

// Codes of the two lane-paired blocks v * rinv (Eq. 3 as a reciprocal
// multiply; rinv = 0 gives signed zeros).
__device__ __forceinline__ void encode_x2(const float2* v, float2 rinv2, Packed16& pa, Packed16& pb) {
  float2 y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = mul2(v[i], rinv2);
  pa.lo = e2m1x8_rne(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x);
  pa.hi = e2m1x8_rne(y[8].x, y[9].x, y[10].x, y[11].x, y[12].x, y[13].x, y[14].x, y[15].x);
  pb.lo = e2m1x8_rne(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y);
  pb.hi = e2m1x8_rne(y[8].y, y[9].y, y[10].y, y[11].y, y[12].y, y[13].y, y[14].y, y[15].y);
}

// Squared error of two encodings in the original domain (the Four Over Six
// criterion): sum of RN((v - RN(q s))^2), s2 = (s_a, s_b) from the table.
// Same operations as sq_error_x2: the subtraction of the rounded product and
// the first summation level stay scalar (never merged with the products).
__device__ __forceinline__ float2 sq_error_tab(const float2* v, float2 s2, const Packed16& pa, const Packed16& pb) {
  float2 q[16], e[16];
  decode16x2(pa, pb, q);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 d = sub2_exact(v[i], mul2(q[i], s2));
    e[i] = mul2(d, d);
  }
  return sum16x2(e);
}

// Squared error of one encoding whose grid values q are known (the Four
// Over Six criterion): sum of RN((v - RN(q s))^2), as sq_error_tab.
__device__ __forceinline__ float2 sq_error_q(const float2* v, float2 s2, const float2* q) {
  float2 e[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 d = sub2_exact(v[i], mul2(q[i], s2));
    e[i] = mul2(d, d);
  }
  return sum16x2(e);
}

// Round-to-nearest block quantization of two lane-paired blocks from the
// table (Four Over Six §2.1 Eq. 2-3; with FOUR_SIX the better of the M = 6
// and M = 4 candidates by squared error, ties to M = 6, §1 Table 1).
template <bool FOUR_SIX, class S>
__device__ __forceinline__ void quantize_pair_tab(const float2* v, const S& c, Packed16& pa, Packed16& pb,
                                                  uint32_t& sba, uint32_t& sbb) {
  float ma, mb;
  max_abs16x2(v, ma, mb);
  const float2 d6 = c.d6();
  const uint32_t s6 = e4m3x2_rne(scale_quot(ma, d6.x), scale_quot(mb, d6.y));
  const uint32_t a6 = s6 & 0xFFu, b6 = s6 >> 8;
  const float2 ta6 = c.ent_a(a6), tb6 = c.ent_b(b6);
  sba = a6;
  sbb = b6;
  if constexpr (!FOUR_SIX) {
    encode_x2(v, make_float2(ta6.y, tb6.y), pa, pb);
  } else {
    // each candidate's grid values come out of its encoding and feed its
    // error at once
    float2 q[16];
    encode_decode_x2(v, make_float2(ta6.y, tb6.y), pa, pb, q);
    const float2 e6 = sq_error_q(v, make_float2(ta6.x, tb6.x), q);
    const float2 d4 = c.d4();
    const uint32_t s4 = e4m3x2_rne(scale_quot(ma, d4.x), scale_quot(mb, d4.y));
    const uint32_t a4 = s4 & 0xFFu, b4 = s4 >> 8;
    const float2 ta4 = c.ent_a(a4), tb4 = c.ent_b(b4);
    Packed16 pa4, pb4;
    encode_decode_x2(v, make_float2(ta4.y, tb4.y), pa4, pb4, q);
    const float2 e4 = sq_error_q(v, make_float2(ta4.x, tb4.x), q);
    if (e4.x < e6.x) {
      sba = a4;
      pa = pa4;
    }
    if (e4.y < e6.y) {
      sbb = b4;
      pb = pb4;
    }
  }
}

// Unsigned division by a runtime constant d >= 1 for n < 2^32:
// q = (n * mul) >> (32 + shift), mul = ceil(2^(32+shift) / d) (33 bits),
// shift = ceil(log2 d).  The rounding error of mul is below d <= 2^shift, so
// the quotient is exact for every 32-bit n.
struct FastDiv {
  uint32_t d, shift;
  uint64_t mul;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.shift = s;
  f.mul = ((1ull << (32 + s)) + d - 1) / d;
  return f;
}

__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDiv& f) {
  // n * mul < 2^32 * 2^33 would overflow 64 bits only if mul >= 2^32 and n is
  // large; split mul into its high bit and low word.
  const uint64_t lo = static_cast<uint64_t>(n) * static_cast<uint32_t>(f.mul);
  const uint64_t hi = (f.mul >> 32) ? static_cast<uint64_t>(n) : 0ull;  // n * 2^32 / 2^32
  // (n * mul) >> 32 = hi + (lo >> 32)
  const uint64_t t = hi + (lo >> 32);
  return static_cast<uint32_t>(t >> f.shift);
}

}  // namespace nvfp4
