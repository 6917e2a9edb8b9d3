/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 block quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent restatement of the
 * method that the CUDA library is checked against.  Only the test-suite, the
 * smoke check and the CPU-baseline leg of the benchmark load it.  It shares no
 * source, header, table or constant with the CUDA library, and it never calls
 * the CUDA library.
 *
 * Sources (page title, section / equation):
 *   [46]  "Four Over Six: more accurate NVFP4 quantization with adaptive block
 *         scaling" (Chinese translation), §1 (Fig. 1, Table 1) and §2.1 Eq. 1-3.
 *   [NV]  Write-up of NVIDIA's "Pretraining LLMs with NVFP4" (arXiv 2509.25149),
 *         §一 (format), §二 (four techniques), §四 (Blackwell), §六 (procedure).
 *   [Q2]  News write-up of Quartet II / MS-EDEN, §一 (MS-EDEN), §二 (recipe).
 *   [PX]  Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *         1, 2, 3", SC'11 -- the Philox4x32-10 generator.
 *
 * Arithmetic: IEEE-754 binary32, round-to-nearest-even, one rounding per
 * operation, in the order written (build with -ffp-contract=off, no
 * fast-math, SSE arithmetic).  The pages fix the precision of the tensor scale
 * (FP32, [46] §2.1) and of the stored block scale and values (E4M3, E2M1); the
 * intermediate steps are taken in FP32 as well, so that every integer decision
 * (a code, a scale byte, the 4/6 choice) is taken in one stated precision.
 * The GEMM reference is FP64.
 *
 * Readings where the pages are silent are marked "READING:".
 *
 * Parity unpinned: oracle_sr_hw_field, the assignment of a draw's random bits
 * to the four elements the sm_100a stochastic-rounding convert takes at once.
 * It restates that instruction's observed behaviour; no page or identity
 * fixes it beyond the uniformity its tests check.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>
#include <math.h>

/* Status values returned by the oracle (its own definitions). */
#define OR_OK 0
#define OR_ERR_ARG (-1)
#define OR_ERR_SHAPE (-2)
#define OR_ERR_NONFINITE (-4)

/* Modes and flags, numbered like the library's public header (they are the
 * interface both sides implement; the values are restated here, not shared). */
#define OR_RTN 0
#define OR_FOUR_SIX 1
#define OR_RHT_SR 2
#define OR_MS_EDEN 3
#define OR_RHT_SR_HW 4

#define OR_ROWWISE 0x1u
#define OR_COLWISE 0x2u
#define OR_BLOCK2D 0x4u
#define OR_ALPHA_PROVIDED 0x10u
#define OR_HEADROOM 0x200u
#define OR_VECTOR_SCALES 0x400u
#define OR_RHT 0x40u
#define OR_INVERSE_RHT 0x80u

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 [PX]: two multiply rounds per step, Weyl key schedule.     */
/* ------------------------------------------------------------------------ */
void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                          uint32_t out[4]) {
  /* Round multipliers and key increments as given in [PX]. */
  const uint32_t MUL0 = 0xD2511F53u, MUL1 = 0xCD9E8D57u;
  const uint32_t WEYL0 = 0x9E3779B9u, WEYL1 = 0xBB67AE85u;
  uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
  uint32_t k[2] = {key_in[0], key_in[1]};
  for (int round = 0; round < 10; ++round) {
    uint64_t p0 = (uint64_t)MUL0 * (uint64_t)c[0];
    uint64_t p1 = (uint64_t)MUL1 * (uint64_t)c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    uint32_t n3 = lo0;
    c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    k[0] += WEYL0;
    k[1] += WEYL1;
  }
  out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

/* One Philox draw for the quantizer: key = seed, counter = (unit, c2, tag). */
static void draw(uint64_t seed, uint64_t unit, uint32_t c2, uint32_t tag,
                 uint32_t w[4]) {
  uint32_t ctr[4] = {(uint32_t)unit, (uint32_t)(unit >> 32), c2, tag};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  oracle_philox4x32_10(ctr, key, w);
}

#define TAG_FP4_SR 1u
#define TAG_SCALE_SR 2u
#define TAG_SIGNS 3u
#define TAG_FP4_SR_HW 4u

/* READING: the random sign diagonal d of the Hadamard transform ([NV] §二,
 * [Q2] §一 name a random rotation but not its source) is bit i of the first
 * word of the draw (seed, unit 0, c2 0, tag 3); bit set means d_i = -1.  One d
 * serves the whole tensor and both orientations. */
uint32_t oracle_sign_bits(uint64_t seed) {
  uint32_t w[4];
  draw(seed, 0, 0, TAG_SIGNS, w);
  return w[0] & 0xFFFFu;
}

/* ------------------------------------------------------------------------ */
/* Number formats ([NV] §一; [46] §1, §2.1).                                */
/* ------------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* E4M3 (OCP E4M3FN): 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
 * largest finite 448.  Only non-negative scales are ever stored. */
float oracle_e4m3_value(uint8_t b) {
  int e = (b >> 3) & 0xF, m = b & 7;
  float mag;
  if ((b & 0x7F) == 0x7F) return NAN;
  if (e == 0) mag = ldexpf((float)m, -9);
  else mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return (b & 0x80) ? -mag : mag;
}

/* Byte of the largest E4M3 value <= v (v >= 0, finite, v < 448 handled by
 * caller).  Walks the 127 non-negative finite codes: slow and plain. */
static uint8_t e4m3_floor_code(float v) {
  uint8_t best = 0;
  for (int b = 0; b <= 0x7E; ++b)
    if (oracle_e4m3_value((uint8_t)b) <= v) best = (uint8_t)b;
  return best;
}

/* Round-to-nearest, ties to even mantissa, saturating at 448. */
uint8_t oracle_e4m3_rne(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  uint8_t lo = e4m3_floor_code(v);
  float vlo = oracle_e4m3_value(lo);
  if (vlo == v) return lo;
  uint8_t hi = (uint8_t)(lo + 1);
  float vhi = oracle_e4m3_value(hi); /* lo < 0x7E here, so hi is finite */
  double dlo = (double)v - (double)vlo, dhi = (double)vhi - (double)v;
  if (dlo < dhi) return lo;
  if (dhi < dlo) return hi;
  return (lo & 1) ? hi : lo; /* tie: even mantissa */
}

/* Smallest E4M3 value >= v, saturating at 448. */
uint8_t oracle_e4m3_ceil(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  uint8_t lo = e4m3_floor_code(v);
  if (oracle_e4m3_value(lo) == v) return lo;
  return (uint8_t)(lo + 1);
}

/* Stochastic rounding to E4M3 with a 24-bit uniform u24: round up iff
 * u24 < f * 2^24, where f is the position of v between its two neighbours. */
uint8_t oracle_e4m3_sr(float v, uint32_t u24) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  uint8_t lo = e4m3_floor_code(v);
  float vlo = oracle_e4m3_value(lo);
  if (vlo == v) return lo;
  float vhi = oracle_e4m3_value((uint8_t)(lo + 1));
  float f = (v - vlo) / (vhi - vlo); /* exact: Sterbenz, power-of-two gap */
  return ((float)u24 < f * 16777216.0f) ? (uint8_t)(lo + 1) : lo;
}

/* E2M1: the eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 ([46] §1), code =
 * sign bit (bit 3) + magnitude index (bits 0-2). */
static const float E2M1_GRID[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_value(uint8_t code) {
  float mag = E2M1_GRID[code & 7];
  return (code & 8) ? -mag : mag;
}

/* Round to the nearest grid magnitude, ties to the even code, saturate at 6.
 * Sign bit = sign bit of y (a negative value that rounds to 0 gives 0x8). */
uint8_t oracle_e2m1_rne(float y) {
  uint8_t sign = (f32_bits(y) >> 31) ? 8 : 0;
  float a = fabsf(y);
  if (a >= 6.0f) return (uint8_t)(sign | 7);
  int best = 0;
  for (int i = 1; i < 8; ++i) {
    double dbest = fabs((double)a - (double)E2M1_GRID[best]);
    double di = fabs((double)a - (double)E2M1_GRID[i]);
    if (di < dbest || (di == dbest && (i & 1) == 0 && (best & 1) == 1)) best = i;
  }
  return (uint8_t)(sign | best);
}

/* Stochastic rounding to the grid with a 16-bit uniform u16: round the
 * magnitude up iff u16 < f * 65536, f = (a - lo) / (hi - lo).  |y| >= 6 -> 6. */
uint8_t oracle_e2m1_sr(float y, uint32_t u16) {
  uint8_t sign = (f32_bits(y) >> 31) ? 8 : 0;
  float a = fabsf(y);
  if (a >= 6.0f) return (uint8_t)(sign | 7);
  int lo = 0;
  for (int i = 0; i < 8; ++i)
    if (E2M1_GRID[i] <= a) lo = i;
  if (E2M1_GRID[lo] == a) return (uint8_t)(sign | lo);
  float f = (a - E2M1_GRID[lo]) / (E2M1_GRID[lo + 1] - E2M1_GRID[lo]);
  int up = (float)u16 < f * 65536.0f;
  return (uint8_t)(sign | (lo + up));
}

/* Stochastic rounding as the sm_100a conversion cvt.rs.satfinite.e2m1x4.f32
 * performs it with a 16-bit random field r16.  The pages name hardware
 * stochastic rounding ([NV] §四) but not its bit use; this rule was read off
 * the instruction's outputs on B200 (2.65 M conversions, no exception): the
 * magnitude rounds up iff r16 + f * 2^16 >= 2^16, f the exact position of |y|
 * between its grid neighbours (compared here as (a - lo) 2^16 >= (2^16 - r16)
 * gap, both sides exact); |y| >= 6 gives 6.  The threshold rule is pinned by
 * its exact expectation; the assignment of random bits to elements
 * (oracle_sr_hw_field) is the instruction's own and has no source in the
 * pages or the mathematics beyond uniformity: parity unpinned for it. */
uint8_t oracle_e2m1_sr_hw(float y, uint32_t r16) {
  uint8_t sign = (f32_bits(y) >> 31) ? 8 : 0;
  float a = fabsf(y);
  if (a >= 6.0f) return (uint8_t)(sign | 7);
  int lo = 0;
  for (int i = 0; i < 8; ++i)
    if (E2M1_GRID[i] <= a) lo = i;
  if (E2M1_GRID[lo] == a) return (uint8_t)(sign | lo);
  double gap = (double)E2M1_GRID[lo + 1] - (double)E2M1_GRID[lo];
  int up = ((double)a - (double)E2M1_GRID[lo]) * 65536.0 >= (65536.0 - (double)r16) * gap;
  return (uint8_t)(sign | (lo + up));
}

/* The 16-bit field of a group's 32-bit word w (bytes b0..b3) used for the
 * element in position j of its group of four, the group being handed to the
 * instruction last element first: j = 0 takes b2 b0, j = 1 the same 16 bits
 * reversed, j = 2 takes b3 b1, j = 3 the same 16 bits reversed. */
static uint32_t rev16(uint32_t x) {
  uint32_t r = 0;
  for (int i = 0; i < 16; ++i) r |= ((x >> i) & 1u) << (15 - i);
  return r;
}
uint32_t oracle_sr_hw_field(uint32_t w, int j) {
  uint32_t even = (((w >> 16) & 0xFFu) << 8) | (w & 0xFFu);
  uint32_t odd = (((w >> 24) & 0xFFu) << 8) | ((w >> 8) & 0xFFu);
  switch (j & 3) {
    case 0: return even;
    case 1: return rev16(even);
    case 2: return odd;
    default: return rev16(odd);
  }
}

/* ------------------------------------------------------------------------ */
/* 16-wide random Hadamard transform ([NV] §二, [Q2] §一).                   */
/* READING: r = (1/4) H16 D x with the natural (Sylvester) H16, applied as   */
/* an in-place butterfly with strides 1, 2, 4, 8, then a multiply by 1/4.    */
/* ------------------------------------------------------------------------ */
void oracle_rht16(const float x[16], uint32_t sign_bits, float r[16]) {
  float v[16];
  for (int i = 0; i < 16; ++i) v[i] = ((sign_bits >> i) & 1) ? -x[i] : x[i];
  for (int h = 1; h < 16; h <<= 1)
    for (int i = 0; i < 16; ++i)
      if ((i & h) == 0) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  for (int i = 0; i < 16; ++i) r[i] = v[i] * 0.25f;
}

/* Inverse: x = D (1/4) H16 r (H16 H16 = 16 I). */
void oracle_irht16(const float r[16], uint32_t sign_bits, float x[16]) {
  float v[16];
  for (int i = 0; i < 16; ++i) v[i] = r[i];
  for (int h = 1; h < 16; h <<= 1)
    for (int i = 0; i < 16; ++i)
      if ((i & h) == 0) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  for (int i = 0; i < 16; ++i) {
    float t = v[i] * 0.25f;
    x[i] = ((sign_bits >> i) & 1) ? -t : t;
  }
}

/* Pairwise sum of 16 terms with strides 8, 4, 2, 1 (READING: the pages say
 * "lower error" without an order; this tree is the stated order). */
static float sum16(const float e[16]) {
  float t[16];
  for (int i = 0; i < 16; ++i) t[i] = e[i];
  for (int h = 8; h >= 1; h >>= 1)
    for (int i = 0; i < h; ++i) t[i] = t[i] + t[i + h];
  return t[0];
}

/* ------------------------------------------------------------------------ */
/* Eq. 1: tensor scale alpha = amax / (6 * 448)  ([46] §2.1; [NV] §六).      */
/* ------------------------------------------------------------------------ */
float oracle_alpha_from_amax(float amax) { return amax / 2688.0f; }

/* Headroom variant of Eq. 1: alpha = amax / (4 * 448).  Under Four Over Six
 * the M = 4 candidate's raw scale amax_b / (alpha * 4) then stays within the
 * E4M3 range instead of saturating at 448 (Eq. 2 with M = 4 and the plain
 * Eq. 1 reaches 672). */
float oracle_alpha_headroom(float amax) { return amax / 1792.0f; }

/* Block encoding of 16 values (one 1D block) under candidate max M.         */
typedef struct {
  uint8_t code[16];
  uint8_t scale;   /* E4M3 byte of Delta */
} block16_t;

/* Eq. 2: Delta = amax_b / (alpha * M), cast to E4M3; ceil for the RHT+SR
 * mode (READING: rounding the scale up keeps |y| <= 6, so stochastic rounding
 * is never clipped), round-to-nearest-even otherwise. */
static uint8_t block_scale(float amax_b, float alpha, float M, int use_ceil) {
  float den = alpha * M;
  float draw_ = (den == 0.0f) ? 0.0f : amax_b / den;
  return use_ceil ? oracle_e4m3_ceil(draw_) : oracle_e4m3_rne(draw_);
}

/* Eq. 3 with the stored scale: s = alpha * Delta, y = v * (1/s), then E2M1.
 * READING: a correctly rounded reciprocal then a multiply (differs from the
 * division X/(alpha Delta) only at exact ties).  When s is 0 or 1/s is not
 * finite, the magnitudes are 0 (codes keep the sign of v). */
static void encode_values(const float v[16], float alpha, uint8_t scale,
                          int stochastic, const uint32_t u16[16],
                          uint8_t code[16]) {
  float s = alpha * oracle_e4m3_value(scale);
  float rinv = (s == 0.0f) ? INFINITY : 1.0f / s;
  for (int i = 0; i < 16; ++i) {
    uint8_t sign = (f32_bits(v[i]) >> 31) ? 8 : 0;
    if (isinf(rinv)) { code[i] = sign; continue; }
    float y = v[i] * rinv;
    code[i] = stochastic ? oracle_e2m1_sr(y, u16[i]) : oracle_e2m1_rne(y);
  }
}

/* Squared error of one candidate in the original domain:
 * e_i = (v_i - s*q_i)^2, summed with sum16. */
static float block_sq_error(const float v[16], float alpha, const block16_t* b) {
  float s = alpha * oracle_e4m3_value(b->scale);
  float e[16];
  for (int i = 0; i < 16; ++i) {
    float xhat = oracle_e2m1_value(b->code[i]) * s;
    float d = v[i] - xhat;
    e[i] = d * d;
  }
  return sum16(e);
}

static float max_abs16(const float v[16]) {
  float m = 0.0f;
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

/* The random bits of one block: 16-bit SR fields for the values (two draws,
 * tag 1) and the 24-bit SR field for the scale (tag 2, four blocks per draw). */
static void block_bits(uint64_t seed, uint32_t c2, uint64_t blk, uint32_t u16[16],
                       uint32_t* u24) {
  if (u16) {
    for (int j = 0; j < 2; ++j) {
      uint32_t w[4];
      draw(seed, 2 * blk + (uint64_t)j, c2, TAG_FP4_SR, w);
      for (int i = 8 * j; i < 8 * j + 8; ++i)
        u16[i] = (w[(i >> 1) & 3] >> (16 * (i & 1))) & 0xFFFFu;
    }
  }
  if (u24) {
    uint32_t w[4];
    draw(seed, blk >> 2, c2, TAG_SCALE_SR, w);
    *u24 = w[blk & 3] >> 8;
  }
}

/* Quantize one 1D block v[16] (already rotated in RHT modes).  Mode steps:
 *  RTN      : M = 6, Eq. 2 (RNE scale), Eq. 3 (RNE values)          [46] §2.1
 *  FOUR_SIX : both M = 6 and M = 4; keep M = 4 iff its squared error is
 *             strictly lower (tie keeps 6)                    [46] §1; [Q2] §二
 *  RHT_SR   : M = 6, ceil scale, stochastic values            [NV] §二, §七
 *  MS_EDEN  : M = 6 RNE codes; the scale alone is stochastically rounded
 *             from the unbiasing value ||r||^2 / (alpha <r, q>)        [Q2] §一
 */
static void quantize_block(const float v[16], float alpha, int mode,
                           uint64_t seed, uint32_t c2, uint64_t blk,
                           block16_t* out) {
  float amax_b = max_abs16(v);
  if (mode == OR_RTN || mode == OR_FOUR_SIX) {
    block16_t b6;
    b6.scale = block_scale(amax_b, alpha, 6.0f, 0);
    encode_values(v, alpha, b6.scale, 0, NULL, b6.code);
    if (mode == OR_FOUR_SIX) {
      block16_t b4;
      b4.scale = block_scale(amax_b, alpha, 4.0f, 0);
      encode_values(v, alpha, b4.scale, 0, NULL, b4.code);
      float err6 = block_sq_error(v, alpha, &b6);
      float err4 = block_sq_error(v, alpha, &b4);
      *out = (err4 < err6) ? b4 : b6;
    } else {
      *out = b6;
    }
    return;
  }
  if (mode == OR_RHT_SR) {
    uint32_t u16[16];
    block_bits(seed, c2, blk, u16, NULL);
    out->scale = block_scale(amax_b, alpha, 6.0f, 1);
    encode_values(v, alpha, out->scale, 1, u16, out->code);
    return;
  }
  if (mode == OR_RHT_SR_HW) {
    /* as RHT_SR, with the values rounded by the hardware rule: one draw per
     * block (tag 4, unit blk), word g for elements 4g .. 4g+3 */
    uint32_t w[4];
    draw(seed, blk, c2, TAG_FP4_SR_HW, w);
    out->scale = block_scale(amax_b, alpha, 6.0f, 1);
    float s = alpha * oracle_e4m3_value(out->scale);
    float rinv = (s == 0.0f) ? INFINITY : 1.0f / s;
    for (int i = 0; i < 16; ++i) {
      uint8_t sign = (f32_bits(v[i]) >> 31) ? 8 : 0;
      if (isinf(rinv)) { out->code[i] = sign; continue; }
      out->code[i] = oracle_e2m1_sr_hw(v[i] * rinv, oracle_sr_hw_field(w[i >> 2], i & 3));
    }
    return;
  }
  /* MS_EDEN.  READING (the pages fix only "rotate, round the FP4 values to
   * nearest, randomness only on the E4M3 scale, unbiased"): following the
   * EDEN estimator the name refers to, the unbiasing scale is
   * Delta* = sum(r^2) / (alpha * sum(r * q)), stochastically rounded to E4M3,
   * so that E[<r, alpha Delta q>] = ||r||^2. */
  uint8_t prov = block_scale(amax_b, alpha, 6.0f, 0);
  encode_values(v, alpha, prov, 0, NULL, out->code);
  float rr[16], rq[16];
  for (int i = 0; i < 16; ++i) {
    rr[i] = v[i] * v[i];
    rq[i] = v[i] * oracle_e2m1_value(out->code[i]);
  }
  float num = sum16(rr);
  float den = alpha * sum16(rq);
  if (den == 0.0f) { out->scale = 0; return; }
  float dstar = num / den;
  uint32_t u24;
  block_bits(seed, c2, blk, NULL, &u24);
  out->scale = oracle_e4m3_sr(dstar, u24);
}

/* ------------------------------------------------------------------------ */
/* Tensor-level quantization.                                               */
/* ------------------------------------------------------------------------ */
static int rotated(int mode, uint32_t flags) {
  return mode == OR_RHT_SR || mode == OR_MS_EDEN || mode == OR_RHT_SR_HW || (flags & OR_RHT);
}

/* Gather the 16 values of 1D block (i, b) in an orientation: orient 0 = row i,
 * elements 16b..16b+15; orient 1 = column i, rows 16b..16b+15.  Rotated in
 * RHT modes. */
static void gather_block(const uint16_t* x, int64_t ld, int orient, int64_t i,
                         int64_t b, int rot, uint32_t signs, float v[16]) {
  float raw[16];
  for (int k = 0; k < 16; ++k) {
    int64_t r = orient ? (16 * b + k) : i;
    int64_t c = orient ? i : (16 * b + k);
    raw[k] = bf16_to_f32(x[r * ld + c]);
  }
  if (rot) oracle_rht16(raw, signs, v);
  else memcpy(v, raw, sizeof raw);
}

/* amax of the tensor as seen in one orientation (rotated values when rot is
 * set).  Returns OR_ERR_NONFINITE if any element is not finite. */
int oracle_amax(const uint16_t* x, int64_t R, int64_t C, int64_t ld, int orient,
                int rot, uint64_t seed, float* amax) {
  if (R < 0 || C < 0 || ld < C) return OR_ERR_SHAPE;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c)
      if (!isfinite(bf16_to_f32(x[r * ld + c]))) return OR_ERR_NONFINITE;
  float m = 0.0f;
  if (!rot) {
    for (int64_t r = 0; r < R; ++r)
      for (int64_t c = 0; c < C; ++c) m = fmaxf(m, fabsf(bf16_to_f32(x[r * ld + c])));
  } else {
    if ((orient ? R : C) % 16) return OR_ERR_SHAPE;
    uint32_t signs = oracle_sign_bits(seed);
    int64_t nvec = orient ? C : R, nblk = (orient ? R : C) / 16;
#pragma omp parallel for reduction(max : m) schedule(static)
    for (int64_t i = 0; i < nvec; ++i)
      for (int64_t b = 0; b < nblk; ++b) {
        float v[16];
        gather_block(x, ld, orient, i, b, 1, signs, v);
        m = fmaxf(m, max_abs16(v));
      }
  }
  *amax = m;
  return OR_OK;
}

/* 1D quantization in one orientation, for the vectors v0 <= i < v1 (rows
 * when orient = 0, columns when orient = 1).  Output codes: [v1-v0, len/2]
 * bytes, element 2j in the low nibble of byte j (READING: the pages do not
 * fix the nibble order); scales: [v1-v0, len/16] E4M3 bytes, row-major.  The
 * random streams use the global block index, so a range reproduces exactly
 * the same bytes as the full tensor. */
int oracle_quantize_1d(const uint16_t* x, int64_t R, int64_t C, int64_t ld,
                       int orient, int mode, uint32_t flags, uint64_t seed,
                       uint32_t stream_id, float alpha, int64_t v0, int64_t v1,
                       uint8_t* codes, uint8_t* scales) {
  int64_t nvec = orient ? C : R, len = orient ? R : C, nblk = len / 16;
  if (len % 16 || v0 < 0 || v1 > nvec || v0 > v1 || ld < C) return OR_ERR_SHAPE;
  if (mode < OR_RTN || mode > OR_RHT_SR_HW) return OR_ERR_ARG;
  uint32_t c2 = stream_id * 2u + (uint32_t)orient;
  uint32_t signs = oracle_sign_bits(seed);
  int rot = rotated(mode, flags);
#pragma omp parallel for schedule(static)
  for (int64_t i = v0; i < v1; ++i)
    for (int64_t b = 0; b < nblk; ++b) {
      float v[16];
      block16_t q;
      gather_block(x, ld, orient, i, b, rot, signs, v);
      uint64_t blk = (uint64_t)(i * nblk + b);
      quantize_block(v, alpha, mode, seed, c2, blk, &q);
      int64_t o = i - v0;
      if (codes)
        for (int j = 0; j < 8; ++j)
          codes[o * (len / 2) + 8 * b + j] = (uint8_t)(q.code[2 * j] | (q.code[2 * j + 1] << 4));
      if (scales) scales[o * nblk + b] = q.scale;
    }
  return OR_OK;
}

/* 2D 16x16 block scaling for weights ([NV] §二 third technique, §七): one
 * scale per 16x16 tile, so the tensor and its transpose hold the same
 * quantized values.  Modes RTN and FOUR_SIX.  The 4/6 error of a tile is the
 * sum16 over its 16 rows of each row's sum16 (READING).  Computes the block
 * rows br0 <= br < br1.  Row outputs: codes [16(br1-br0), C/2], scales
 * [br1-br0, C/16].  Column outputs: codes [C, 8(br1-br0)] (column c holds
 * rows 16 br0 .. 16 br1 - 1), scales [C/16, br1-br0]. */
int oracle_quantize_2d(const uint16_t* x, int64_t R, int64_t C, int64_t ld,
                       int mode, float alpha, int64_t br0, int64_t br1,
                       uint8_t* codes_row, uint8_t* scales_row,
                       uint8_t* codes_col, uint8_t* scales_col) {
  if (R % 16 || C % 16 || ld < C || br0 < 0 || br1 > R / 16 || br0 > br1) return OR_ERR_SHAPE;
  if (mode != OR_RTN && mode != OR_FOUR_SIX) return OR_ERR_ARG;
  int64_t CB = C / 16, NB = br1 - br0;
#pragma omp parallel for schedule(static)
  for (int64_t br = br0; br < br1; ++br)
    for (int64_t bc = 0; bc < CB; ++bc) {
      float v[16][16];
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i)
        for (int j = 0; j < 16; ++j) {
          v[i][j] = bf16_to_f32(x[(16 * br + i) * ld + 16 * bc + j]);
          amax_b = fmaxf(amax_b, fabsf(v[i][j]));
        }
      int nc = (mode == OR_FOUR_SIX) ? 2 : 1;
      const float Ms[2] = {6.0f, 4.0f};
      uint8_t cand_scale[2];
      uint8_t cand_code[2][16][16];
      float cand_err[2];
      for (int c = 0; c < nc; ++c) {
        cand_scale[c] = block_scale(amax_b, alpha, Ms[c], 0);
        float rowerr[16];
        for (int i = 0; i < 16; ++i) {
          block16_t b;
          b.scale = cand_scale[c];
          encode_values(v[i], alpha, b.scale, 0, NULL, b.code);
          memcpy(cand_code[c][i], b.code, 16);
          rowerr[i] = block_sq_error(v[i], alpha, &b);
        }
        cand_err[c] = sum16(rowerr);
      }
      int pick = (nc == 2 && cand_err[1] < cand_err[0]) ? 1 : 0;
      int64_t lb = br - br0;
      if (scales_row) scales_row[lb * CB + bc] = cand_scale[pick];
      if (scales_col) scales_col[bc * NB + lb] = cand_scale[pick];
      for (int i = 0; i < 16; i += 1)
        for (int j = 0; j < 16; j += 2) {
          /* row-packed: elements (i, j), (i, j+1) share a byte */
          if (codes_row)
            codes_row[(16 * lb + i) * (C / 2) + (16 * bc + j) / 2] =
                (uint8_t)(cand_code[pick][i][j] | (cand_code[pick][i][j + 1] << 4));
        }
      for (int j = 0; j < 16; j += 1)
        for (int i = 0; i < 16; i += 2) {
          /* column-packed: elements (i, j), (i+1, j) share a byte */
          if (codes_col)
            codes_col[(16 * bc + j) * (8 * NB) + (16 * lb + i) / 2] =
                (uint8_t)(cand_code[pick][i][j] | (cand_code[pick][i + 1][j] << 4));
        }
    }
  return OR_OK;
}

/* Full quantization of a bf16 tensor [R, C] (row stride ld elements).
 * Row outputs: codes [R, C/2], scales [R, C/16] (2D: [R/16, C/16]).
 * Column outputs (the transpose, blocks along R): codes [C, R/2],
 * scales [C, R/16] (2D: [C/16, R/16]).  alpha_in != NULL supplies alpha,
 * which must then be finite and >= 0. */
int oracle_quantize(const uint16_t* x, int64_t R, int64_t C, int64_t ld,
                    int mode, uint32_t flags, uint64_t seed, uint32_t stream_id,
                    const float* alpha_in, uint8_t* codes_row, uint8_t* scales_row,
                    float* alpha_row, uint8_t* codes_col, uint8_t* scales_col,
                    float* alpha_col, float* amax_row, float* amax_col) {
  int want_row = (flags & OR_ROWWISE) != 0, want_col = (flags & OR_COLWISE) != 0;
  int two_d = (flags & OR_BLOCK2D) != 0;
  if (mode < OR_RTN || mode > OR_RHT_SR_HW) return OR_ERR_ARG;
  if (!want_row && !want_col) return OR_ERR_ARG;
  if (two_d && rotated(mode, flags)) return OR_ERR_ARG;
  if (alpha_in && !(isfinite(*alpha_in) && *alpha_in >= 0.0f)) return OR_ERR_ARG;
  if (R < 0 || C < 0 || ld < C) return OR_ERR_SHAPE;
  if ((want_row || two_d) && C % 16) return OR_ERR_SHAPE;
  if ((want_col || two_d) && R % 16) return OR_ERR_SHAPE;
  int rot = rotated(mode, flags) && !two_d;
  for (int o = 0; o < 2; ++o) {
    int want = o ? want_col : want_row;
    if (!want) continue;
    float amax = 0.0f;
    int st = oracle_amax(x, R, C, ld, o, rot, seed, &amax);
    if (st) return st;
    float alpha = alpha_in ? *alpha_in
                           : ((flags & OR_HEADROOM) ? oracle_alpha_headroom(amax) : oracle_alpha_from_amax(amax));
    if (o == 0) {
      if (amax_row) *amax_row = amax;
      if (alpha_row) *alpha_row = alpha;
    } else {
      if (amax_col) *amax_col = amax;
      if (alpha_col) *alpha_col = alpha;
    }
    if (!two_d)
      oracle_quantize_1d(x, R, C, ld, o, mode, flags, seed, stream_id, alpha, 0,
                         o ? C : R, o ? codes_col : codes_row, o ? scales_col : scales_row);
  }
  if (two_d) {
    /* 2D blocks: one tensor scale for both orientations (the same quantized
     * values), from the plain amax. */
    float amax = 0.0f;
    int st = oracle_amax(x, R, C, ld, 0, 0, seed, &amax);
    if (st) return st;
    float alpha = alpha_in ? *alpha_in
                           : ((flags & OR_HEADROOM) ? oracle_alpha_headroom(amax) : oracle_alpha_from_amax(amax));
    oracle_quantize_2d(x, R, C, ld, mode, alpha, 0, R / 16,
                       want_row ? codes_row : NULL, want_row ? scales_row : NULL,
                       want_col ? codes_col : NULL, want_col ? scales_col : NULL);
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Finer tensor scales ([NV] §九: the single global amax is named as a       */
/* limitation, with per-row or per-block global scales as the remedy).       */
/* ------------------------------------------------------------------------ */
/* READING: the pages name the remedy without defining it.  The oracle takes
 * the plainest form: Eq. 1 applied to each vector of the quantized operand on
 * its own -- a row of x for the row orientation, a column of x for the column
 * orientation (the rows of the GEMM operand, one per output row or column of
 * the product) -- alpha_i = amax_i / (6 * 448), amax_i over that vector's
 * (rotated) values; everything else is unchanged.  A "per-block" global scale
 * with the 16-element block as its unit would coincide with the E4M3 block
 * scale itself, so that variant is not a separate mode. */
int oracle_amax_vectors(const uint16_t* x, int64_t R, int64_t C, int64_t ld, int orient,
                        int rot, uint64_t seed, float* amax) {
  if (R < 0 || C < 0 || ld < C) return OR_ERR_SHAPE;
  int64_t nvec = orient ? C : R, len = orient ? R : C;
  if (rot && len % 16) return OR_ERR_SHAPE;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c)
      if (!isfinite(bf16_to_f32(x[r * ld + c]))) return OR_ERR_NONFINITE;
  uint32_t signs = oracle_sign_bits(seed);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nvec; ++i) {
    float m = 0.0f;
    if (!rot) {
      for (int64_t k = 0; k < len; ++k) {
        int64_t r = orient ? k : i, c = orient ? i : k;
        m = fmaxf(m, fabsf(bf16_to_f32(x[r * ld + c])));
      }
    } else {
      for (int64_t b = 0; b < len / 16; ++b) {
        float v[16];
        gather_block(x, ld, orient, i, b, 1, signs, v);
        m = fmaxf(m, max_abs16(v));
      }
    }
    amax[i] = m;
  }
  return OR_OK;
}

/* 1D quantization with one tensor scale per vector (flag OR_VECTOR_SCALES):
 * alpha[i] = Eq. 1 of vector i's amax (or the headroom form), then the
 * vector is quantized exactly as oracle_quantize_1d would with that alpha.
 * Outputs as oracle_quantize; alpha_row [R] and alpha_col [C] are vectors;
 * amax_row / amax_col receive the largest vector amax of the orientation. */
int oracle_quantize_vector_scales(const uint16_t* x, int64_t R, int64_t C, int64_t ld,
                                  int mode, uint32_t flags, uint64_t seed, uint32_t stream_id,
                                  uint8_t* codes_row, uint8_t* scales_row, float* alpha_row,
                                  uint8_t* codes_col, uint8_t* scales_col, float* alpha_col,
                                  float* amax_row, float* amax_col) {
  int want_row = (flags & OR_ROWWISE) != 0, want_col = (flags & OR_COLWISE) != 0;
  if (mode < OR_RTN || mode > OR_RHT_SR_HW) return OR_ERR_ARG;
  if (!want_row && !want_col) return OR_ERR_ARG;
  if (flags & (OR_BLOCK2D | OR_ALPHA_PROVIDED)) return OR_ERR_ARG;
  if (R < 0 || C < 0 || ld < C) return OR_ERR_SHAPE;
  if (want_row && C % 16) return OR_ERR_SHAPE;
  if (want_col && R % 16) return OR_ERR_SHAPE;
  int rot = rotated(mode, flags);
  for (int o = 0; o < 2; ++o) {
    if (!(o ? want_col : want_row)) continue;
    int64_t nvec = o ? C : R, len = o ? R : C;
    float* av = (float*)malloc(sizeof(float) * (size_t)(nvec > 0 ? nvec : 1));
    int st = oracle_amax_vectors(x, R, C, ld, o, rot, seed, av);
    if (st) { free(av); return st; }
    float tmax = 0.0f;
    uint8_t* codes = o ? codes_col : codes_row;
    uint8_t* scales = o ? scales_col : scales_row;
    float* alpha = o ? alpha_col : alpha_row;
    for (int64_t i = 0; i < nvec; ++i) {
      tmax = fmaxf(tmax, av[i]);
      float a = (flags & OR_HEADROOM) ? oracle_alpha_headroom(av[i]) : oracle_alpha_from_amax(av[i]);
      if (alpha) alpha[i] = a;
      oracle_quantize_1d(x, R, C, ld, o, mode, flags, seed, stream_id, a, i, i + 1,
                         codes ? codes + i * (len / 2) : NULL, scales ? scales + i * (len / 16) : NULL);
    }
    if (o == 0 && amax_row) *amax_row = tmax;
    if (o == 1 && amax_col) *amax_col = tmax;
    free(av);
  }
  return OR_OK;
}

/* Dequantization: xhat = q * (alpha * Delta), optionally rotated back
 * (inverse transform along each 16-block).  codes [R, C/2]; scales [R, C/16]
 * or, with BLOCK2D, [R/16, C/16].  Output fp32 [R, C]. */
int oracle_dequantize(const uint8_t* codes, const uint8_t* scales, float alpha,
                      int64_t R, int64_t C, uint32_t flags, uint64_t seed,
                      float* y) {
  if (R < 0 || C < 0 || C % 16) return OR_ERR_SHAPE;
  int two_d = (flags & OR_BLOCK2D) != 0;
  if (two_d && R % 16) return OR_ERR_SHAPE;
  if (two_d && (flags & OR_INVERSE_RHT)) return OR_ERR_ARG;
  uint32_t signs = oracle_sign_bits(seed);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t b = 0; b < C / 16; ++b) {
      uint8_t sb = two_d ? scales[(r / 16) * (C / 16) + b] : scales[r * (C / 16) + b];
      float s = alpha * oracle_e4m3_value(sb);
      float v[16];
      for (int k = 0; k < 16; ++k) {
        int64_t c = 16 * b + k;
        uint8_t byte = codes[r * (C / 2) + c / 2];
        uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        v[k] = oracle_e2m1_value(q) * s;
      }
      if (flags & OR_INVERSE_RHT) {
        float t[16];
        oracle_irht16(v, signs, t);
        memcpy(v, t, sizeof t);
      }
      for (int k = 0; k < 16; ++k) y[r * C + 16 * b + k] = v[k];
    }
  return OR_OK;
}

/* GEMM reference in FP64: D[m, n] = alphaA alphaB sum_k (qA DeltaA)(qB DeltaB)
 * for TN operands A [M, K] and B [N, K] (codes [rows, K/2], scales
 * [rows, K/16] row-major).  Only the listed rows and columns are computed
 * (rows == NULL: all rows; cols == NULL: all columns); D is [nrows, ncols]. */
void oracle_gemm_f64(const uint8_t* A, const uint8_t* sA, float alphaA,
                     const uint8_t* B, const uint8_t* sB, float alphaB,
                     int64_t M, int64_t N, int64_t K, const int64_t* rows,
                     int64_t nrows, const int64_t* cols, int64_t ncols,
                     double* D) {
  if (!rows) nrows = M;
  if (!cols) ncols = N;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows ? rows[i] : i;
    double* arow = (double*)malloc(sizeof(double) * (size_t)K);
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = A[m * (K / 2) + k / 2];
      uint8_t q = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
      arow[k] = (double)oracle_e2m1_value(q) * (double)oracle_e4m3_value(sA[m * (K / 16) + k / 16]);
    }
    for (int64_t j = 0; j < ncols; ++j) {
      int64_t n = cols ? cols[j] : j;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = B[n * (K / 2) + k / 2];
        uint8_t q = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        double b = (double)oracle_e2m1_value(q) * (double)oracle_e4m3_value(sB[n * (K / 16) + k / 16]);
        acc += arow[k] * b;
      }
      D[i * ncols + j] = acc * (double)alphaA * (double)alphaB;
    }
    free(arow);
  }
}

/* GEMM reference in FP64 with one tensor scale per operand row:
 * D[m, n] = alphaA[m] alphaB[n] sum_k (qA DeltaA)(qB DeltaB); operands as in
 * oracle_gemm_f64, alphaA [M], alphaB [N]. */
void oracle_gemm_f64_vector_scales(const uint8_t* A, const uint8_t* sA, const float* alphaA,
                                   const uint8_t* B, const uint8_t* sB, const float* alphaB,
                                   int64_t M, int64_t N, int64_t K, const int64_t* rows,
                                   int64_t nrows, const int64_t* cols, int64_t ncols,
                                   double* D) {
  if (!rows) nrows = M;
  if (!cols) ncols = N;
  oracle_gemm_f64(A, sA, 1.0f, B, sB, 1.0f, M, N, K, rows, nrows, cols, ncols, D);
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows ? rows[i] : i;
    for (int64_t j = 0; j < ncols; ++j) {
      int64_t n = cols ? cols[j] : j;
      D[i * ncols + j] *= (double)alphaA[m] * (double)alphaB[n];
    }
  }
}

/* Expose the block quantizer alone (one 16-vector, one candidate policy) for
 * the worked-example pin: alpha supplied, no rotation. */
int oracle_quantize_block16(const float v[16], float alpha, int mode, uint64_t seed,
                            uint32_t c2, uint64_t blk, uint8_t codes_out[16],
                            uint8_t* scale_out) {
  block16_t q;
  quantize_block(v, alpha, mode, seed, c2, blk, &q);
  memcpy(codes_out, q.code, 16);
  *scale_out = q.scale;
  return OR_OK;
}

/* Squared block error of given codes/scale (diagnostic for the 4/6 pins). */
float oracle_block_sq_error(const float v[16], float alpha, const uint8_t codes[16],
                            uint8_t scale) {
  block16_t b;
  memcpy(b.code, codes, 16);
  b.scale = scale;
  return block_sq_error(v, alpha, &b);
}

/* ------------------------------------------------------------------------ */
/* MXFP4: 32-element blocks, one power-of-two (UE8M0) scale per block, E2M1  */
/* values, no tensor scale ([NV] §一 and §五; the AMD MI355X write-up, 01-02, */
/* with a fixed rotation).                                                   */
/* ------------------------------------------------------------------------ */
/* READING: the pages give the block size (32), the scale format (UE8M0,
 * power-of-two) and nothing of how the scale is chosen.  The oracle takes the
 * OCP microscaling rule: shared exponent e = floor(log2(amax_b)) - 2 (2 being
 * the largest E2M1 exponent), clamped to the UE8M0 range [-127, 127]; an
 * all-zero block takes -127.  Stored byte = e + 127.  Values are
 * q_i = E2M1-RNE(v_i / 2^e), saturating at 6 (so block maxima in [6, 8) * 2^e
 * clip to 6). */
int oracle_mx_exponent(float amax) {
  if (!(amax > 0.0f)) return -127;
  int k;
  frexpf(amax, &k);          /* amax = m 2^k, m in [0.5, 1): floor(log2) = k - 1 */
  int e = (k - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

float oracle_e8m0_value(uint8_t b) {
  if (b == 0xFF) return NAN;
  return ldexpf(1.0f, (int)b - 127);
}

/* One 32-vector: scale byte and codes. */
static void mx_block(const float v[32], uint8_t code[32], uint8_t* scale) {
  float m = 0.0f;
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  int e = oracle_mx_exponent(m);
  *scale = (uint8_t)(e + 127);
  for (int i = 0; i < 32; ++i) code[i] = oracle_e2m1_rne(ldexpf(v[i], -e));
}

/* Quantize bf16 x [R, C] to MXFP4 in the requested orientations: rows (32
 * consecutive elements of a row; codes [R, C/2], scales [R, C/32]) and / or
 * columns (32 consecutive rows of a column, stored transposed: codes
 * [C, R/2], scales [C, R/32]).  With OR_RHT each 16-element half of a block
 * is first rotated by (1/4) H16 D, D drawn from seed as for NVFP4 (a fixed
 * seed gives the deterministic rotation).  Non-finite input returns
 * OR_ERR_NONFINITE. */
int oracle_mx_quantize(const uint16_t* x, int64_t R, int64_t C, int64_t ld,
                       uint32_t flags, uint64_t seed, uint8_t* codes_row,
                       uint8_t* scales_row, uint8_t* codes_col,
                       uint8_t* scales_col) {
  int want_row = (flags & OR_ROWWISE) != 0, want_col = (flags & OR_COLWISE) != 0;
  if (!want_row && !want_col) return OR_ERR_ARG;
  if (R < 0 || C < 0 || ld < C) return OR_ERR_SHAPE;
  if ((want_row && C % 32) || (want_col && R % 32)) return OR_ERR_SHAPE;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c)
      if (!isfinite(bf16_to_f32(x[r * ld + c]))) return OR_ERR_NONFINITE;
  int rot = (flags & OR_RHT) != 0;
  uint32_t signs = oracle_sign_bits(seed);
  for (int orient = 0; orient < 2; ++orient) {
    if (orient == 0 && !want_row) continue;
    if (orient == 1 && !want_col) continue;
    int64_t nvec = orient ? C : R, len = orient ? R : C;
    uint8_t* codes = orient ? codes_col : codes_row;
    uint8_t* scales = orient ? scales_col : scales_row;
    for (int64_t i = 0; i < nvec; ++i)
      for (int64_t b = 0; b < len / 32; ++b) {
        float v[32];
        gather_block(x, ld, orient, i, 2 * b, rot, signs, v);
        gather_block(x, ld, orient, i, 2 * b + 1, rot, signs, v + 16);
        uint8_t q[32];
        mx_block(v, q, &scales[i * (len / 32) + b]);
        for (int k = 0; k < 16; ++k)
          codes[i * (len / 2) + 16 * b + k] = (uint8_t)(q[2 * k] | (q[2 * k + 1] << 4));
      }
  }
  return OR_OK;
}

/* Decode MXFP4 codes [R, C/2] and scales [R, C/32] to fp32: y = q 2^e, then
 * with OR_INVERSE_RHT each 16-element half goes through D (1/4) H16. */
int oracle_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t R,
                         int64_t C, uint32_t flags, uint64_t seed, float* y) {
  if (R < 0 || C < 0 || C % 32) return OR_ERR_SHAPE;
  uint32_t signs = oracle_sign_bits(seed);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t b = 0; b < C / 16; ++b) {
      float s = oracle_e8m0_value(scales[r * (C / 32) + b / 2]);
      float v[16];
      for (int k = 0; k < 16; ++k) {
        int64_t c = 16 * b + k;
        uint8_t byte = codes[r * (C / 2) + c / 2];
        uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        v[k] = oracle_e2m1_value(q) * s;
      }
      if (flags & OR_INVERSE_RHT) {
        float t[16];
        oracle_irht16(v, signs, t);
        memcpy(v, t, sizeof t);
      }
      for (int k = 0; k < 16; ++k) y[r * C + 16 * b + k] = v[k];
    }
  return OR_OK;
}

/* MXFP4 GEMM reference in FP64: D[m, n] = sum_k (qA 2^eA)(qB 2^eB) for TN
 * operands A [M, K] and B [N, K] (codes [rows, K/2], UE8M0 scales
 * [rows, K/32] row-major); no tensor scales.  Rows / columns as for
 * oracle_gemm_f64. */
void oracle_mx_gemm_f64(const uint8_t* A, const uint8_t* sA, const uint8_t* B,
                        const uint8_t* sB, int64_t M, int64_t N, int64_t K,
                        const int64_t* rows, int64_t nrows, const int64_t* cols,
                        int64_t ncols, double* D) {
  if (!rows) nrows = M;
  if (!cols) ncols = N;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows ? rows[i] : i;
    double* arow = (double*)malloc(sizeof(double) * (size_t)K);
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = A[m * (K / 2) + k / 2];
      uint8_t q = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
      arow[k] = (double)oracle_e2m1_value(q) * (double)oracle_e8m0_value(sA[m * (K / 32) + k / 32]);
    }
    for (int64_t j = 0; j < ncols; ++j) {
      int64_t n = cols ? cols[j] : j;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = B[n * (K / 2) + k / 2];
        uint8_t q = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        acc += arow[k] * (double)oracle_e2m1_value(q) * (double)oracle_e8m0_value(sB[n * (K / 32) + k / 32]);
      }
      D[i * ncols + j] = acc;
    }
    free(arow);
  }
}
