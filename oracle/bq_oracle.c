/*
 * bq_oracle.c -- plain CPU oracle for block-scaled (MX) activation quantization
 * and the block-scaled GEMM that consumes it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, calls or
 * includes this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant generator with the CUDA path.
 *
 * Written to be read against the pages, not to be fast:
 *   - every operand is decoded exactly and products are summed in fp64;
 *   - the activation quantizer follows the step order of the
 *     "formats.py" page (dsv41-sampled-drafting, code/offload/dspark/native):
 *     module docstring's description of act_qdq (the kernel quantizer it
 *     mirrors) and the functions act_scale / act_quant / act_qdq /
 *     _log2_ceil_pow2;
 *   - the number formats follow the same page's module docstring
 *     ("Formats" paragraph) and its constants FP4_TABLE, FP8_MAX, BLOCK,
 *     E8M0_NAN, E4M3_NAN;
 *   - the MXFP4 activation quantizer (for FP4 x FP4 products, the A4W4 GEMMs
 *     of the "fp4-gemm" page, README "Available Functions") is not spelled
 *     out on the pages: it is the same per-32 rule with the E2M1 format's
 *     largest value 6 in place of 448, and E2M1 codes packed two per byte with
 *     the even element in the low nibble (the pages' MXFP4 weight layout);
 *   - NVFP4 (the A4W4 kernels of the "fp4-gemm" page name it: E2M1 codes
 *     with one E4M3 scale per 16 values and a per-tensor fp32 scale) is not
 *     spelled out either: the tensor is first multiplied by the caller's
 *     per-tensor scale, each block of 16 takes the smallest E4M3 scale that
 *     holds its largest value (the round-up counterpart of the MX rule, so no
 *     value clips below the top of the E4M3 range), codes are E2M1 of
 *     x / scale; the GEMM undoes the per-tensor scales through alpha;
 *   - the gradient quantizer of the backward pass (E5M2 codes, the pages'
 *     "hip_quant" README, "Stochastic E5M2 Backward Gradients" and "Block-wise
 *     FP8 Scaling") takes the same per-32 rule with E5M2's largest finite
 *     value 57344, rounding to nearest even or stochastically between the two
 *     neighbouring E5M2 values; the page draws each element's random number
 *     from its seed and its index with no state, which here is a
 *     counter-based generator (Philox4x64-10) keyed by the seed and counted by
 *     the element's index.
 *
 * Floating point: compile with -ffp-contract=off and without fast-math so that
 * every float expression below is one IEEE binary32 operation, as the page's
 * fp32 tensor arithmetic is.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_NAN_SCALE (-1) /* E8M0 byte 255 */
#define ORACLE_ERR_NAN_CODE (-2)  /* E4M3 byte 0x7F or 0xFF */
#define ORACLE_ERR_SHAPE (-3)     /* K not a multiple of 32, bad kind */
#define ORACLE_ERR_NONFINITE (-4) /* NaN/Inf activation (outside the contract) */

#define BLOCK 32 /* one scale per 32 consecutive elements ("BLOCK = 32") */

/* ------------------------------------------------------------------ */
/* Number formats ("Formats" paragraph of the formats.py page).        */
/* ------------------------------------------------------------------ */

/* E8M0: one byte b means 2^(b-127); b = 255 is NaN and is refused. */
int oracle_decode_e8m0(uint8_t b, double *out) {
  if (b == 255) return ORACLE_ERR_NAN_SCALE;
  *out = ldexp(1.0, (int)b - 127);
  return ORACLE_OK;
}

/* E2M1 (FP4) code -> value, from the format's fields: bit 3 sign, bits 2..1
 * exponent (bias 1), bit 0 mantissa; exponent field 0 is the subnormal
 * 0.m x 2^0.  Code 8 is -0.0.  (The page lists the result as FP4_TABLE; the
 * tests compare this against that printed table.) */
double oracle_decode_fp4(uint8_t code) {
  int sign = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

/* E4M3 (e4m3fn): bias 7, no infinities, 0x7F/0xFF are NaN (refused).
 * Normal: (-1)^s 2^(E-7) (1 + m/8); subnormal (E = 0): (-1)^s 2^-6 (m/8). */
int oracle_decode_e4m3(uint8_t b, double *out) {
  if ((b & 0x7F) == 0x7F) return ORACLE_ERR_NAN_CODE;
  int s = b >> 7;
  int E = (b >> 3) & 0xF;
  int m = b & 7;
  double mag = (E == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, E - 7);
  *out = s ? -mag : mag;
  return ORACLE_OK;
}

/* The 127 non-negative finite E4M3 magnitudes, indexed by code 0x00..0x7E;
 * they increase strictly with the code. */
static double e4m3_mag[127];
static int e4m3_mag_ready = 0;
static void e4m3_table_init(void) {
  if (e4m3_mag_ready) return;
  for (int c = 0; c < 127; ++c) oracle_decode_e4m3((uint8_t)c, &e4m3_mag[c]);
  e4m3_mag_ready = 1;
}

/* Round a binary32 value to E4M3 with round-to-nearest, ties to even,
 * saturating at +-448 (the page clamps to [-448, 448] before converting, so
 * saturation is never what decides a result there).  The sign is kept:
 * negative values that round to zero give 0x80 (-0).
 * Method: find the two neighbouring representable magnitudes in the sorted
 * table and pick the nearer; on a tie pick the even code (the code's low bit
 * is the mantissa's low bit). */
uint8_t oracle_encode_e4m3(float v) {
  e4m3_table_init();
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  uint8_t code;
  if (a >= e4m3_mag[126]) {
    code = 126; /* 448 */
  } else {
    int lo = 0, hi = 126; /* invariant: mag[lo] <= a < mag[hi] */
    while (hi - lo > 1) {
      int mid = (lo + hi) / 2;
      if (e4m3_mag[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - e4m3_mag[lo], dhi = e4m3_mag[hi] - a;
    if (dlo < dhi) code = (uint8_t)lo;
    else if (dhi < dlo) code = (uint8_t)hi;
    else code = (uint8_t)((lo % 2 == 0) ? lo : hi);
  }
  return (uint8_t)(sign | code);
}

/* Element-wise oracle_encode_e4m3 over n values. */
void oracle_encode_e4m3_n(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_encode_e4m3(v[i]);
}

/* Round a binary32 value to E2M1 (FP4) with round-to-nearest, ties to even,
 * saturating at +-6, the sign kept (negative values that round to zero give
 * code 8, -0).  The same method as the E4M3 encoder: the 8 non-negative
 * magnitudes of codes 0..7 increase with the code (decoded by
 * oracle_decode_fp4); take the nearer neighbour, on a tie the even code. */
uint8_t oracle_encode_fp4(float v) {
  double mag[8];
  for (int c = 0; c < 8; ++c) mag[c] = oracle_decode_fp4((uint8_t)c);
  uint8_t sign = signbit(v) ? 0x8 : 0x0;
  double a = fabs((double)v);
  uint8_t code;
  if (a >= mag[7]) {
    code = 7; /* 6 */
  } else {
    int lo = 0;
    while (mag[lo + 1] <= a) ++lo; /* mag[lo] <= a < mag[lo + 1] */
    int hi = lo + 1;
    double dlo = a - mag[lo], dhi = mag[hi] - a;
    if (dlo < dhi) code = (uint8_t)lo;
    else if (dhi < dlo) code = (uint8_t)hi;
    else code = (uint8_t)((lo % 2 == 0) ? lo : hi);
  }
  return (uint8_t)(sign | code);
}

void oracle_encode_fp4_n(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_encode_fp4(v[i]);
}

/* E5M2: bias 15, two mantissa bits, exponent field 31 is Inf / NaN (refused
 * here: the quantizer never produces them).  Normal: (-1)^s 2^(E-15) (1 + m/4);
 * subnormal (E = 0): (-1)^s 2^-14 (m/4).  Largest finite 0x7B = 57344. */
int oracle_decode_e5m2(uint8_t b, double *out) {
  int s = b >> 7;
  int E = (b >> 2) & 0x1F;
  int m = b & 3;
  if (E == 31) return ORACLE_ERR_NAN_CODE;
  double mag = (E == 0) ? ldexp(m / 4.0, -14) : ldexp(1.0 + m / 4.0, E - 15);
  *out = s ? -mag : mag;
  return ORACLE_OK;
}

/* The 124 non-negative finite E5M2 magnitudes, codes 0x00..0x7B, increasing. */
static double e5m2_mag[124];
static int e5m2_mag_ready = 0;
static void e5m2_table_init(void) {
  if (e5m2_mag_ready) return;
  for (int c = 0; c < 124; ++c) oracle_decode_e5m2((uint8_t)c, &e5m2_mag[c]);
  e5m2_mag_ready = 1;
}

/* Index of the largest finite E5M2 magnitude <= a (a >= 0, below the top). */
static int e5m2_floor_code(double a) {
  int lo = 0, hi = 123; /* mag[lo] <= a < mag[hi] */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (e5m2_mag[mid] <= a) lo = mid; else hi = mid;
  }
  return lo;
}

/* binary32 -> E5M2, round to nearest even, saturating at +-57344, sign kept. */
uint8_t oracle_encode_e5m2(float v) {
  e5m2_table_init();
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  uint8_t code;
  if (a >= e5m2_mag[123]) {
    code = 123;
  } else {
    int lo = e5m2_floor_code(a), hi = lo + 1;
    double dlo = a - e5m2_mag[lo], dhi = e5m2_mag[hi] - a;
    if (dlo < dhi) code = (uint8_t)lo;
    else if (dhi < dlo) code = (uint8_t)hi;
    else code = (uint8_t)((lo % 2 == 0) ? lo : hi);
  }
  return (uint8_t)(sign | code);
}

void oracle_encode_e5m2_n(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_encode_e5m2(v[i]);
}

/* Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC 2011): ten rounds of two 64 x 64 -> 128-bit
 * multiplications on a 4-word counter, the 2-word key bumped by the Weyl
 * constants between rounds. */
static void mulhilo64(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo) {
  unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
  *hi = (uint64_t)(p >> 64);
  *lo = (uint64_t)p;
}

void oracle_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(M0, x0, &hi0, &lo0);
    mulhilo64(M1, x2, &hi1, &lo1);
    uint64_t y0 = hi1 ^ x1 ^ k0, y1 = lo1, y2 = hi0 ^ x3 ^ k1, y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The uniform draw of element `index` under `seed`: one Philox4x64-10 block
 * (counter (index / 8, 0, 0, 0), key (seed, 0)) serves 8 elements, element
 * index takes the 32-bit half (index % 2, low half first) of word
 * (index / 2) % 4, as a double in [0, 1) with 2^-32 resolution. */
double oracle_uniform(uint64_t seed, uint64_t index) {
  uint64_t ctr[4] = {index >> 3, 0, 0, 0}, key[2] = {seed, 0}, out[4];
  oracle_philox4x64_10(ctr, key, out);
  uint64_t word = out[(index >> 1) & 3];
  uint32_t half = (uint32_t)((index & 1) ? (word >> 32) : (word & 0xFFFFFFFFu));
  return ldexp((double)half, -32);
}

/* Stochastic E5M2 rounding of binary32 v (|v| <= 57344 after the clamp):
 * lo and hi are the neighbouring E5M2 magnitudes around |v|; the result is hi
 * when u < (|v| - lo) / (hi - lo) (exact in double), else lo; sign kept. */
uint8_t oracle_encode_e5m2_sr(float v, double u) {
  e5m2_table_init();
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a >= e5m2_mag[123]) return (uint8_t)(sign | 123);
  int lo = e5m2_floor_code(a);
  double d = (a - e5m2_mag[lo]) / (e5m2_mag[lo + 1] - e5m2_mag[lo]);
  return (uint8_t)(sign | (u < d ? lo + 1 : lo));
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary32 -> bfloat16, round to nearest even (finite inputs; an overflow
 * gives +-Inf as IEEE rounding does). */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1;
  u += 0x7FFF + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* Activation quantization (formats.py page: act_scale, act_quant,      */
/* act_qdq, _log2_ceil_pow2; the module docstring on act_qdq).          */
/* ------------------------------------------------------------------ */

/* The per-group steps, for one group of 32 binary32 values:
 *   amax = max(max_i |x_i|, 1e-4)                       (fp32)
 *   t    = fp32(amax * fp32(1/448))
 *   e    = ceil(log2 t), read from t's exponent bits: the unbiased exponent,
 *          plus one when any mantissa bit is set (t is a positive normal)
 *   s    = 2^e;   scale byte = e + 127
 *   q_i  = E4M3_RNE(clamp(x_i / s, -448, 448))
 * Returns the scale byte, or -1 if the group holds a NaN or Inf. */
static int act_quant_group(const float *x, uint8_t *q) {
  float amax = 0.0f;
  for (int i = 0; i < BLOCK; ++i) {
    if (!isfinite(x[i])) return -1;
    float ax = fabsf(x[i]);
    if (ax > amax) amax = ax;
  }
  const float floor_ = 1e-4f;
  if (amax < floor_) amax = floor_;
  const float inv448 = (float)(1.0 / 448.0);
  float t = amax * inv448;
  uint32_t bits;
  memcpy(&bits, &t, 4);
  int e = (int)((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
  float s = ldexpf(1.0f, e);
  for (int i = 0; i < BLOCK; ++i) {
    float y = x[i] / s;
    if (y > 448.0f) y = 448.0f;
    if (y < -448.0f) y = -448.0f;
    q[i] = oracle_encode_e4m3(y);
  }
  return e + 127;
}

/* x: bf16 bit patterns, M rows of K elements, row stride ldx elements.
 * q: [M, K] E4M3 codes (row stride K).  sf: [M, K/32] E8M0 bytes, row-major.
 * Returns ORACLE_OK, ORACLE_ERR_SHAPE (K % 32 != 0) or ORACLE_ERR_NONFINITE. */
int oracle_act_quant(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                     uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  float buf[BLOCK];
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t g = 0; g < G; ++g) {
      for (int i = 0; i < BLOCK; ++i) buf[i] = bf16_to_f32(x[m * ldx + g * BLOCK + i]);
      int b = act_quant_group(buf, q + m * K + g * BLOCK);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      sf[m * G + g] = (uint8_t)b;
    }
  }
  return ORACLE_OK;
}

/* Same steps on binary32 input (used to pin the encoder and the scale rule on
 * values that are not bf16). */
int oracle_act_quant_f32(const float *x, int64_t M, int64_t K, uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t g = 0; g < G; ++g) {
      int b = act_quant_group(x + m * K + g * BLOCK, q + m * K + g * BLOCK);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      sf[m * G + g] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* The dequantized activation: value = fp32(q) * s in binary32, then stored
 * as bf16 (round to nearest even).  y: [M, K] bf16 bit patterns. */
int oracle_act_qdq(const uint8_t *q, const uint8_t *sf, int64_t M, int64_t K, uint16_t *y) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double qv, sv;
      if (oracle_decode_e4m3(q[m * K + k], &qv)) return ORACLE_ERR_NAN_CODE;
      if (oracle_decode_e8m0(sf[m * G + k / BLOCK], &sv)) return ORACLE_ERR_NAN_SCALE;
      float v = (float)qv * (float)sv;
      y[m * K + k] = oracle_f32_to_bf16(v);
    }
  return ORACLE_OK;
}

/* MXFP4 activation quantization: the steps of act_quant_group with the
 * E2M1 maximum 6 in place of 448:
 *   amax = max(max_i |x_i|, 1e-4)                       (fp32)
 *   t    = fp32(amax * fp32(1/6))
 *   e    = ceil(log2 t) from t's exponent bits;  scale byte = e + 127
 *   q_i  = E2M1_RNE(clamp(x_i / 2^e, -6, 6))
 * codes[i] gets one code per byte.  Returns the scale byte, or -1 for a NaN
 * or Inf in the group. */
static int act_quant_fp4_group(const float *x, uint8_t *codes) {
  float amax = 0.0f;
  for (int i = 0; i < BLOCK; ++i) {
    if (!isfinite(x[i])) return -1;
    float ax = fabsf(x[i]);
    if (ax > amax) amax = ax;
  }
  const float floor_ = 1e-4f;
  if (amax < floor_) amax = floor_;
  const float inv6 = (float)(1.0 / 6.0);
  float t = amax * inv6;
  uint32_t bits;
  memcpy(&bits, &t, 4);
  int e = (int)((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
  float s = ldexpf(1.0f, e);
  for (int i = 0; i < BLOCK; ++i) {
    float y = x[i] / s;
    if (y > 6.0f) y = 6.0f;
    if (y < -6.0f) y = -6.0f;
    codes[i] = oracle_encode_fp4(y);
  }
  return e + 127;
}

/* Packs 32 one-per-byte codes into 16 bytes, element 2j in the low nibble of
 * byte j. */
static void pack_fp4(const uint8_t *codes, uint8_t *out) {
  for (int j = 0; j < BLOCK / 2; ++j) out[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
}

/* x: bf16 bit patterns [M, ldx]; q: [M, K/2] packed E2M1 codes; sf: [M, K/32]
 * E8M0 bytes.  Returns ORACLE_OK, ORACLE_ERR_SHAPE or ORACLE_ERR_NONFINITE. */
int oracle_act_quant_fp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                         uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  float buf[BLOCK];
  uint8_t codes[BLOCK];
  for (int64_t m = 0; m < M; ++m)
    for (int64_t g = 0; g < G; ++g) {
      for (int i = 0; i < BLOCK; ++i) buf[i] = bf16_to_f32(x[m * ldx + g * BLOCK + i]);
      int b = act_quant_fp4_group(buf, codes);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      pack_fp4(codes, q + m * (K / 2) + g * (BLOCK / 2));
      sf[m * G + g] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* The same steps on binary32 input [M, K]. */
int oracle_act_quant_fp4_f32(const float *x, int64_t M, int64_t K, uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  uint8_t codes[BLOCK];
  for (int64_t m = 0; m < M; ++m)
    for (int64_t g = 0; g < G; ++g) {
      int b = act_quant_fp4_group(x + m * K + g * BLOCK, codes);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      pack_fp4(codes, q + m * (K / 2) + g * (BLOCK / 2));
      sf[m * G + g] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* NVFP4 block scale: the smallest positive E4M3 value >= t (t >= 0 finite):
 * 2^-9 (the smallest subnormal) for t <= 2^-9, 448 for t > 448. */
uint8_t oracle_e4m3_ceil(float t) {
  e4m3_table_init();
  double a = (double)t;
  if (a <= e4m3_mag[1]) return 1;
  if (a >= e4m3_mag[126]) return 126;
  int c = 1;
  while (e4m3_mag[c] < a) ++c; /* mag[c - 1] < a <= mag[c] */
  return (uint8_t)c;
}

/* NVFP4 quantization of one group of 16 values already multiplied by the
 * per-tensor scale (binary32): amax = max |x|, t = fp32(amax * fp32(1/6)),
 * s = oracle_e4m3_ceil(t), q = E2M1_RNE(clamp(fp32(x / s), -6, 6)) with the
 * sign kept.  Returns the scale byte, -1 for a NaN / Inf. */
static int nvfp4_group(const float *x, uint8_t *codes) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) {
    if (!isfinite(x[i])) return -1;
    float ax = fabsf(x[i]);
    if (ax > amax) amax = ax;
  }
  const float inv6 = (float)(1.0 / 6.0);
  float t = amax * inv6;
  uint8_t sb = oracle_e4m3_ceil(t);
  double sd;
  oracle_decode_e4m3(sb, &sd);
  float s = (float)sd;
  for (int i = 0; i < 16; ++i) {
    float y = x[i] / s;
    if (y > 6.0f) y = 6.0f;
    if (y < -6.0f) y = -6.0f;
    codes[i] = oracle_encode_fp4(y);
  }
  return sb;
}

/* x bf16 [M, ldx]; g the per-tensor scale; q [M, K/2] packed E2M1 codes,
 * sf [M, K/16] E4M3 scale bytes.  Each value is first fp32(x * g).
 * K % 16 == 0. */
int oracle_act_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, float g,
                           uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % 16) return ORACLE_ERR_SHAPE;
  const int64_t G = K / 16;
  float buf[16];
  uint8_t codes[16];
  for (int64_t m = 0; m < M; ++m)
    for (int64_t gi = 0; gi < G; ++gi) {
      for (int i = 0; i < 16; ++i) buf[i] = bf16_to_f32(x[m * ldx + gi * 16 + i]) * g;
      int b = nvfp4_group(buf, codes);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      for (int j = 0; j < 8; ++j)
        q[m * (K / 2) + gi * 8 + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
      sf[m * G + gi] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* Gradient quantization, E5M2 codes: the per-32 rule with E5M2's largest
 * finite value 57344 in place of 448,
 *   t = fp32(max(amax, 1e-4) * fp32(1/57344)),  e = ceil(log2 t),
 *   q = E5M2(clamp(x / 2^e, -57344, 57344)), round to nearest even, or
 *       stochastic with the uniform draw of the element's index (sr != 0),
 * for the 32 values x[i * stride] whose source indices are idx0 + i * istride.
 * Writes one code per element to q[i * qstride]; returns the scale byte or -1
 * for a NaN / Inf. */
static int grad_quant_group(const float *x, int64_t stride, uint8_t *q, int64_t qstride,
                            int sr, uint64_t seed, uint64_t idx0, uint64_t istride) {
  float amax = 0.0f;
  for (int i = 0; i < BLOCK; ++i) {
    float v = x[i * stride];
    if (!isfinite(v)) return -1;
    float av = fabsf(v);
    if (av > amax) amax = av;
  }
  const float floor_ = 1e-4f;
  if (amax < floor_) amax = floor_;
  const float inv = (float)(1.0 / 57344.0);
  float t = amax * inv;
  uint32_t bits;
  memcpy(&bits, &t, 4);
  int e = (int)((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
  float s = ldexpf(1.0f, e);
  for (int i = 0; i < BLOCK; ++i) {
    float y = x[i * stride] / s;
    if (y > 57344.0f) y = 57344.0f;
    if (y < -57344.0f) y = -57344.0f;
    q[i * qstride] = sr ? oracle_encode_e5m2_sr(y, oracle_uniform(seed, idx0 + i * istride))
                        : oracle_encode_e5m2(y);
  }
  return e + 127;
}

/* The E4M3 rule of act_quant_group on a strided group (for the transposed
 * activation operand of the weight gradient). */
static int e4m3_quant_group_strided(const float *x, int64_t stride, uint8_t *q, int64_t qstride) {
  float buf[BLOCK];
  uint8_t codes[BLOCK];
  for (int i = 0; i < BLOCK; ++i) buf[i] = x[i * stride];
  int b = act_quant_group(buf, codes);
  if (b < 0) return -1;
  for (int i = 0; i < BLOCK; ++i) q[i * qstride] = codes[i];
  return b;
}

/* Row-wise gradient quantization: x bf16 [M, ldx] -> q [M, K] E5M2, sf
 * [M, K/32].  Element (m, k) has index m * K + k. */
int oracle_grad_quant(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int sr,
                      uint64_t seed, uint8_t *q, uint8_t *sf) {
  if (K <= 0 || K % BLOCK) return ORACLE_ERR_SHAPE;
  const int64_t G = K / BLOCK;
  float buf[BLOCK];
  for (int64_t m = 0; m < M; ++m)
    for (int64_t g = 0; g < G; ++g) {
      for (int i = 0; i < BLOCK; ++i) buf[i] = bf16_to_f32(x[m * ldx + g * BLOCK + i]);
      int b = grad_quant_group(buf, 1, q + m * K + g * BLOCK, 1, sr, seed,
                               (uint64_t)(m * K + g * BLOCK), 1);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      sf[m * G + g] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* Transposed quantization: x bf16 [R, ldx] (C columns used) quantized along
 * R, per 32 consecutive rows of one column, written transposed: q [C, R],
 * sf [C, R/32].  fmt 0: E4M3 (the act_quant rule), 1: E5M2 (the gradient
 * rule; element (r, c) has index r * C + c).  This is the quantization of the
 * transposed matrix by the row-wise rule. */
int oracle_quant_transposed(const uint16_t *x, int64_t R, int64_t C, int64_t ldx, int fmt,
                            int sr, uint64_t seed, uint8_t *q, uint8_t *sf) {
  if (R <= 0 || R % BLOCK || C < 0 || fmt < 0 || fmt > 1 || (sr && fmt != 1))
    return ORACLE_ERR_SHAPE;
  const int64_t G = R / BLOCK;
  float col[BLOCK];
  for (int64_t c = 0; c < C; ++c)
    for (int64_t g = 0; g < G; ++g) {
      for (int i = 0; i < BLOCK; ++i) col[i] = bf16_to_f32(x[(g * BLOCK + i) * ldx + c]);
      int b = fmt == 1 ? grad_quant_group(col, 1, q + c * R + g * BLOCK, 1, sr, seed,
                                          (uint64_t)(g * BLOCK * C + c), (uint64_t)C)
                       : e4m3_quant_group_strided(col, 1, q + c * R + g * BLOCK, 1);
      if (b < 0) return ORACLE_ERR_NONFINITE;
      sf[c * G + g] = (uint8_t)b;
    }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Exact operand decode + fp64 GEMM with the fused epilogue.            */
/* ------------------------------------------------------------------ */

/* Weight kinds. */
#define ORACLE_B_FP4 0     /* E2M1 packed [N, K/2], low nibble = even k; scales [N, K/32] */
#define ORACLE_B_FP8BLK 1  /* E4M3 [N, K]; scales [ceil(N/32), ceil(K/32)], one per 32x32 block */
#define ORACLE_B_FP8ROW 2  /* E4M3 [N, K]; scales [N, K/32] (MXFP8 along K) */
#define ORACLE_B_NVFP4 3   /* E2M1 packed [N, K/2]; E4M3 scales [N, K/16] */

/* Activation kinds. */
#define ORACLE_A_E4M3 0 /* E4M3 [M, K]; scales [M, K/32] */
#define ORACLE_A_FP4 1  /* E2M1 packed [M, K/2], low nibble = even k; scales [M, K/32] */
#define ORACLE_A_E5M2 2 /* E5M2 [M, K] (gradients); scales [M, K/32] */
#define ORACLE_A_NVFP4 3 /* E2M1 packed [M, K/2]; E4M3 scales [M, K/16] */

#define ORACLE_ACT_NONE 0
#define ORACLE_ACT_GELU 1

typedef struct {
  const uint8_t *aq, *asf;
  const uint8_t *b, *bsf;
  int akind;
  int bkind;
  int64_t M, N, K;
  const uint16_t *bias, *residual;
  int64_t ld_res;
  double alpha;
  int act;
  /* full output */
  double *ref, *sumabs;
  /* sampled output (when ms != NULL) */
  const int64_t *ms, *ns;
  int64_t count;
  int64_t begin, end;
  int status;
} gemm_job;

/* Decoded A value a[m][k] = code * 2^(b - 127) (exact in double), the code
 * E4M3 or packed E2M1. */
static int dec_a(const gemm_job *J, int64_t m, int64_t k, double *v) {
  double c, s;
  if (J->akind == ORACLE_A_NVFP4) {
    uint8_t byte = J->aq[m * (J->K / 2) + k / 2];
    c = oracle_decode_fp4((k % 2 == 0) ? (byte & 0x0F) : (byte >> 4));
    if (oracle_decode_e4m3(J->asf[m * (J->K / 16) + k / 16], &s)) return ORACLE_ERR_NAN_SCALE;
    *v = c * s;
    return ORACLE_OK;
  }
  if (J->akind == ORACLE_A_FP4) {
    uint8_t byte = J->aq[m * (J->K / 2) + k / 2];
    c = oracle_decode_fp4((k % 2 == 0) ? (byte & 0x0F) : (byte >> 4));
  } else if (J->akind == ORACLE_A_E5M2) {
    if (oracle_decode_e5m2(J->aq[m * J->K + k], &c)) return ORACLE_ERR_NAN_CODE;
  } else if (oracle_decode_e4m3(J->aq[m * J->K + k], &c)) {
    return ORACLE_ERR_NAN_CODE;
  }
  if (oracle_decode_e8m0(J->asf[m * (J->K / BLOCK) + k / BLOCK], &s)) return ORACLE_ERR_NAN_SCALE;
  *v = c * s;
  return ORACLE_OK;
}

/* Decoded B value b[n][k] for the three weight formats (formats.py page:
 * decode_fp4, decode_fp8_block, fp4_codes). */
static int dec_b(const gemm_job *J, int64_t n, int64_t k, double *v) {
  const int64_t K = J->K;
  double c, s;
  uint8_t sb;
  if (J->bkind == ORACLE_B_NVFP4) {
    uint8_t byte = J->b[n * (K / 2) + k / 2];
    c = oracle_decode_fp4((k % 2 == 0) ? (byte & 0x0F) : (byte >> 4));
    if (oracle_decode_e4m3(J->bsf[n * (K / 16) + k / 16], &s)) return ORACLE_ERR_NAN_SCALE;
    *v = c * s;
    return ORACLE_OK;
  }
  if (J->bkind == ORACLE_B_FP4) {
    uint8_t byte = J->b[n * (K / 2) + k / 2];
    uint8_t code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    c = oracle_decode_fp4(code);
    sb = J->bsf[n * (K / BLOCK) + k / BLOCK];
  } else {
    if (oracle_decode_e4m3(J->b[n * K + k], &c)) return ORACLE_ERR_NAN_CODE;
    if (J->bkind == ORACLE_B_FP8BLK) {
      int64_t kb = (K + BLOCK - 1) / BLOCK;
      sb = J->bsf[(n / BLOCK) * kb + k / BLOCK];
    } else {
      sb = J->bsf[n * (K / BLOCK) + k / BLOCK];
    }
  }
  if (oracle_decode_e8m0(sb, &s)) return ORACLE_ERR_NAN_SCALE;
  *v = c * s;
  return ORACLE_OK;
}

static double bf16d(const uint16_t *p, int64_t i) { return (double)bf16_to_f32(p[i]); }

/* One output element: acc = sum_k a[m][k] b[n][k] in fp64, sumabs =
 * sum_k |a b|; then ref = act(alpha * acc + bias[n]) + residual[m][n] with
 * act = erf-GELU 0.5 t (1 + erf(t / sqrt 2)) or identity. */
static int one_element(const gemm_job *J, const double *arow, int64_t m, int64_t n,
                       double *ref, double *sabs) {
  double acc = 0.0, sa = 0.0;
  for (int64_t k = 0; k < J->K; ++k) {
    double bv;
    int st = dec_b(J, n, k, &bv);
    if (st) return st;
    double p = arow[k] * bv;
    acc += p;
    sa += fabs(p);
  }
  double t = J->alpha * acc;
  if (J->bias) t += bf16d(J->bias, n);
  if (J->act == ORACLE_ACT_GELU) t = 0.5 * t * (1.0 + erf(t / sqrt(2.0)));
  if (J->residual) t += bf16d(J->residual, m * J->ld_res + n);
  *ref = t;
  *sabs = sa;
  return ORACLE_OK;
}

static void *gemm_worker(void *arg) {
  gemm_job *J = (gemm_job *)arg;
  double *arow = (double *)malloc(sizeof(double) * (size_t)J->K);
  if (!arow) { J->status = ORACLE_ERR_SHAPE; return NULL; }
  J->status = ORACLE_OK;
  if (J->ms == NULL) {
    for (int64_t m = J->begin; m < J->end && !J->status; ++m) {
      for (int64_t k = 0; k < J->K && !J->status; ++k) J->status = dec_a(J, m, k, &arow[k]);
      for (int64_t n = 0; n < J->N && !J->status; ++n)
        J->status = one_element(J, arow, m, n, &J->ref[m * J->N + n], &J->sumabs[m * J->N + n]);
    }
  } else {
    for (int64_t i = J->begin; i < J->end && !J->status; ++i) {
      int64_t m = J->ms[i], n = J->ns[i];
      for (int64_t k = 0; k < J->K && !J->status; ++k) J->status = dec_a(J, m, k, &arow[k]);
      if (!J->status) J->status = one_element(J, arow, m, n, &J->ref[i], &J->sumabs[i]);
    }
  }
  free(arow);
  return NULL;
}

static int run_jobs(gemm_job *proto, int64_t total, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > total) nthreads = (int)(total > 0 ? total : 1);
  gemm_job jobs[256];
  pthread_t th[256];
  int64_t per = (total + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = *proto;
    jobs[t].begin = t * per < total ? t * per : total;
    jobs[t].end = (t + 1) * per < total ? (t + 1) * per : total;
    pthread_create(&th[t], NULL, gemm_worker, &jobs[t]);
  }
  int status = ORACLE_OK;
  for (int t = 0; t < nthreads; ++t) {
    pthread_join(th[t], NULL);
    if (jobs[t].status && !status) status = jobs[t].status;
  }
  return status;
}

/* Full GEMM: ref[m][n], sumabs[m][n] for all M x N outputs.
 * A: aq [M, K] E4M3 codes, asf [M, K/32] E8M0 (row-major).
 * B: see ORACLE_B_*.  bias: [N] bf16 or NULL.  residual: [M, ld_res] bf16 or
 * NULL.  Rows are spread over nthreads POSIX threads. */
int oracle_gemm_ex(const uint8_t *aq, const uint8_t *asf, int akind, const uint8_t *b,
                   const uint8_t *bsf, int bkind, int64_t M, int64_t N, int64_t K,
                   const uint16_t *bias, const uint16_t *residual, int64_t ld_res, double alpha,
                   int act, double *ref, double *sumabs, int nthreads) {
  if (K <= 0 || K % BLOCK || bkind < 0 || bkind > 3 || akind < 0 || akind > 3)
    return ORACLE_ERR_SHAPE;
  gemm_job J = {aq, asf, b, bsf, akind, bkind, M, N, K, bias, residual, ld_res, alpha, act,
                ref, sumabs, NULL, NULL, 0, 0, 0, 0};
  return run_jobs(&J, M, nthreads);
}

int oracle_gemm(const uint8_t *aq, const uint8_t *asf, const uint8_t *b, const uint8_t *bsf,
                int bkind, int64_t M, int64_t N, int64_t K, const uint16_t *bias,
                const uint16_t *residual, int64_t ld_res, double alpha, int act,
                double *ref, double *sumabs, int nthreads) {
  return oracle_gemm_ex(aq, asf, ORACLE_A_E4M3, b, bsf, bkind, M, N, K, bias, residual, ld_res,
                        alpha, act, ref, sumabs, nthreads);
}

/* Sampled GEMM: the same per-element definition at count (m, n) pairs. */
int oracle_gemm_sampled_ex(const uint8_t *aq, const uint8_t *asf, int akind, const uint8_t *b,
                           const uint8_t *bsf, int bkind, int64_t M, int64_t N, int64_t K,
                           const uint16_t *bias, const uint16_t *residual, int64_t ld_res,
                           double alpha, int act, const int64_t *ms, const int64_t *ns,
                           int64_t count, double *ref, double *sumabs, int nthreads) {
  if (K <= 0 || K % BLOCK || bkind < 0 || bkind > 3 || akind < 0 || akind > 3)
    return ORACLE_ERR_SHAPE;
  gemm_job J = {aq, asf, b, bsf, akind, bkind, M, N, K, bias, residual, ld_res, alpha, act,
                ref, sumabs, ms, ns, count, 0, 0, 0};
  return run_jobs(&J, count, nthreads);
}

int oracle_gemm_sampled(const uint8_t *aq, const uint8_t *asf, const uint8_t *b,
                        const uint8_t *bsf, int bkind, int64_t M, int64_t N, int64_t K,
                        const uint16_t *bias, const uint16_t *residual, int64_t ld_res,
                        double alpha, int act, const int64_t *ms, const int64_t *ns,
                        int64_t count, double *ref, double *sumabs, int nthreads) {
  return oracle_gemm_sampled_ex(aq, asf, ORACLE_A_E4M3, b, bsf, bkind, M, N, K, bias, residual,
                                ld_res, alpha, act, ms, ns, count, ref, sumabs, nthreads);
}
