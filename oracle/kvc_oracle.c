/*
 * kvc_oracle.c — plain, slow CPU oracle of the FastKVComp-style KV-cache codec.
 *
 * TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use this file. It shares no code with the CUDA library.
 *
 * Each function states the passage or reading it follows. The pages used:
 *   [P2] "Beyond Compression Ratio: High-Throughput KV Compression for
 *        Disaggregated LLM Serving" (arxivlens), Abstract and Methodology:
 *        distribution transformation and low-bit quantization fused, no
 *        intermediate tensor; LC-style lossless backend built from composable
 *        primitives.
 *   [P3] "FastKVComp: checking whether high-throughput KV compression pays
 *        off" (podcast), episode notes: the pipeline is a randomized Hadamard
 *        transform, low-bit quantization and a lossless codec; only the
 *        quantization loses information; the cache crosses a link to a decode
 *        GPU, so a decoder inverts the pipeline.
 * The stage list comes from the pages; the exact rules are readings R1..R12
 * (named at each function) chosen as the plainest definitions the pages admit.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math (no FMA fusion, no
 * excess precision: x86-64 SSE evaluates float in float).
 */
#include "kvc_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ========================================================================== */
/* Sign generator. Reading R3: one +-1 diagonal over head_dim for the whole   */
/* tensor ("randomized" Hadamard, [P3]). Its bits are the outputs of          */
/* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number       */
/* generators", OOPSLA 2014) started from state = sign_seed; channel c is     */
/* negated iff bit (c mod 64) of output number floor(c/64) is 1.              */
/* ========================================================================== */
uint64_t orc_splitmix64_next(uint64_t *state) {
  uint64_t z;
  *state += 0x9E3779B97F4A7C15ull; /* golden-ratio increment */
  z = *state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void orc_sign_words(uint64_t seed, int d, uint64_t *words) {
  uint64_t state = seed;
  int i;
  for (i = 0; i < (d + 63) / 64; i++) words[i] = orc_splitmix64_next(&state);
}

/* Reading R20 (per-(layer, kv, head) sign diagonals, the FP4Quant abstract's
 * variant of the randomized transform): vector index i (= its position in
 * the order [layer][kv][head]) takes the SplitMix64 outputs number
 * i*W .. i*W + W - 1 (W = ceil(d / 64)) of the same generator from state =
 * sign_seed. Output n comes from state seed + (n + 1) * gamma, so the
 * generator is advanced by i*W increments first; index 0 is reading R3. */
void orc_sign_words_at(uint64_t seed, int d, uint64_t index, uint64_t *words) {
  const uint64_t W = (uint64_t)((d + 63) / 64);
  uint64_t state = seed + index * W * 0x9E3779B97F4A7C15ull;
  uint64_t i;
  for (i = 0; i < W; i++) words[i] = orc_splitmix64_next(&state);
}

static int sign_bit(const uint64_t *words, int c) {
  return (int)((words[c / 64] >> (c % 64)) & 1u);
}

/* ========================================================================== */
/* Walsh-Hadamard transform ([P3] "randomized Hadamard transform").           */
/* Reading R1: unnormalized, y = H_d x with the Sylvester matrix H_d.         */
/* Reading R2: the butterfly order is normative because fp32 sums round:      */
/* strides h = 1, 2, 4, ..., d/2 in ascending order; within a stride every    */
/* pair (i, i+h) with (i & h) == 0 becomes (a+b, a-b), one rounding each.     */
/* ========================================================================== */
void orc_fwht(float *y, int d) {
  int h, i;
  for (h = 1; h < d; h *= 2) {
    for (i = 0; i < d; i++) {
      if ((i & h) == 0) {
        float a = y[i];
        float b = y[i + h];
        y[i] = a + b;
        y[i + h] = a - b;
      }
    }
  }
}

/* Reading R4: the meta is stored divided by 2^k, k = floor(log2(d)/2), so that
 * it sits in the range of the orthonormal transform (|H x| ~ sqrt(d)|x|). */
int orc_meta_shift(int d) {
  int l = 0;
  while ((1 << l) < d) l++;
  return l / 2;
}

/* ========================================================================== */
/* Number formats.                                                            */
/* ========================================================================== */
float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of an fp32 */
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (decoded output, reading R9). */
uint16_t orc_f32_to_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* fp16 (IEEE binary16) -> fp32, exact. */
float orc_f16_to_f32(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) {
    if (m) return NAN;
    return s ? -INFINITY : INFINITY;
  }
  if (e == 0)
    v = ldexp((double)m, -24);
  else
    v = ldexp((double)(1024 + m), e - 25);
  return (float)(s ? -v : v);
}

/* Encodes a non-negative value that already lies on the binary16 grid. */
static uint16_t f16_bits_of_grid_value(double r) {
  int e2;
  if (r < ldexp(1.0, -14)) return (uint16_t)ldexp(r, 24); /* subnormal */
  frexp(r, &e2);                                           /* r in [2^(e2-1), 2^e2) */
  return (uint16_t)(((e2 - 1 + 15) << 10) |
                    (int)ldexp(ldexp(r, -(e2 - 1)) - 1.0, 10));
}

/* fp32 -> fp16 with a directed rounding. The exact value of x is taken in
 * double, scaled by the quantum of its binary16 binade (exact), rounded to an
 * integer toward or away from zero, and scaled back. toward_neg = 1 rounds
 * toward -inf (RD), 0 toward +inf (RU). */
static uint16_t f32_to_f16_directed(float x, int toward_neg) {
  int neg, away, e, E, qexp;
  double a, q, n, r;
  uint16_t sgn;
  if (isnan(x)) return 0x7E00;
  neg = signbit(x) ? 1 : 0;
  sgn = (uint16_t)(neg << 15);
  if (isinf(x)) return (uint16_t)(sgn | 0x7C00);
  a = fabs((double)x);
  if (a == 0.0) return sgn;
  away = toward_neg ? neg : !neg; /* magnitude grows for RD<0 and RU>0 */
  frexp(a, &e);
  E = e - 1;                              /* a in [2^E, 2^(E+1)) */
  qexp = (E < -14) ? -24 : E - 10;        /* spacing of the binade */
  q = ldexp(a, -qexp);
  n = away ? ceil(q) : floor(q);
  r = ldexp(n, qexp);
  if (r > 65504.0) return (uint16_t)(sgn | (away ? 0x7C00 : 0x7BFF));
  if (r == 0.0) return sgn;
  return (uint16_t)(sgn | f16_bits_of_grid_value(r));
}

uint16_t orc_f32_to_f16_rd(float x) { return f32_to_f16_directed(x, 1); }
uint16_t orc_f32_to_f16_ru(float x) { return f32_to_f16_directed(x, 0); }

static int f16_is_inf(uint16_t h) { return (h & 0x7FFFu) == 0x7C00u; }

/* ========================================================================== */
/* Code packing. Reading R6: codes of one vector in channel order, LSB first: */
/* 4-bit: byte j = q[2j] | q[2j+1] << 4;                                      */
/* 2-bit: byte j = q[4j] | q[4j+1] << 2 | q[4j+2] << 4 | q[4j+3] << 6;        */
/* 8-bit (reading R21): byte j = q[j].                                        */
/* ========================================================================== */
void orc_pack_codes(const uint8_t *q, int d, int bits, uint8_t *packed) {
  int per = 8 / bits, j, i;
  for (j = 0; j < d / per; j++) {
    uint8_t b = 0;
    for (i = 0; i < per; i++) b = (uint8_t)(b | (q[j * per + i] << (i * bits)));
    packed[j] = b;
  }
}

void orc_unpack_codes(const uint8_t *packed, int d, int bits, uint8_t *q) {
  int per = 8 / bits, c;
  uint8_t mask = (uint8_t)((1 << bits) - 1);
  for (c = 0; c < d; c++)
    q[c] = (uint8_t)((packed[c / per] >> ((c % per) * bits)) & mask);
}

/* One code of reading R5: t = fl(y - zf), p = fl(t * r) (two separate fp32
 * operations, each rounded to nearest even; the file is built without FMA
 * contraction), then p rounded to the nearest integer, ties to even, and
 * clamped to [0, qmax]. nearbyint() in the default rounding mode is
 * round-half-even, and p is an fp32 value, exact in double. */
int orc_quantize_scalar(float y, float zf, float r, int qmax) {
  float t = y - zf;
  float p = t * r;
  double n = nearbyint((double)p);
  if (n < 0.0) n = 0.0;
  if (n > (double)qmax) n = (double)qmax;
  return (int)n;
}

/* ---- FP4 (reading R22) ---------------------------------------------------- */
/* e2m1 (1 sign, 2 exponent, 1 mantissa bit, no inf/NaN): magnitude index   */
/* i = 0..7 has the values 0, 0.5, 1, 1.5, 2, 3, 4, 6; code = i | 8 for a    */
/* negative value (never for magnitude 0).                                    */
float orc_e2m1_to_f32(int code) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  return (code & 8) ? -mag[code & 7] : mag[code & 7];
}

/* The e2m1 code nearest to p, ties to the even magnitude index (even
 * mantissa bit); magnitudes above 6 give 6; zero is always code 0. The
 * nearest value is found by scanning the eight magnitudes in double. */
int orc_f32_to_e2m1_rne(float p) {
  double a = fabs((double)p), best = 1e300;
  int i, bi = 0;
  if (a >= 6.0) /* the largest magnitude (the scan's differences lose 4 vs 6 far above it) */
    return p < 0.0f ? (7 | 8) : 7;
  for (i = 0; i < 8; i++) {
    double e = fabs(a - (double)orc_e2m1_to_f32(i));
    if (e < best || (e == best && (i & 1) == 0)) {
      best = e;
      bi = i;
    }
  }
  return (bi != 0 && p < 0.0f) ? (bi | 8) : bi;
}

/* e4m3 (the fn variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no inf, 0x7F/0xFF NaN; largest finite 448; subnormals m * 2^-9). */
float orc_e4m3_to_f32(int b) {
  int e = (b >> 3) & 15, m = b & 7;
  float v;
  if ((b & 0x7F) == 0x7F) return NAN;
  v = e ? ldexpf(1.0f + (float)m / 8.0f, e - 7) : ldexpf((float)m, -9);
  return (b & 0x80) ? -v : v;
}

/* The smallest non-negative finite e4m3 value >= x (x >= 0, finite), 448
 * (0x7E) if x exceeds it: a scan over the 127 non-negative finite codes,
 * which are increasing in their bit patterns. */
int orc_f32_to_e4m3_ru(float x) {
  int b;
  for (b = 0; b < 0x7F; b++)
    if ((double)orc_e4m3_to_f32(b) >= (double)x) return b;
  return 0x7E;
}

/* One code of reading R19 (symmetric absmax): p = fl(y * r) (one fp32
 * rounding), then the nearest integer to p, ties to even, clamped to
 * [-qh, qh], qh = 2^(b-1) - 1. The stored code is that integer + 2^(b-1). */
int orc_quantize_scalar_sym(float y, float r, int bits) {
  const int qh = (1 << (bits - 1)) - 1;
  float p = y * r;
  double n = nearbyint((double)p);
  if (n < (double)-qh) n = (double)-qh;
  if (n > (double)qh) n = (double)qh;
  return (int)n + (1 << (bits - 1));
}

/* ========================================================================== */
/* Quantization of one vector ([P2] Methodology: distribution transformation  */
/* then low-bit quantization; [P3]: only this step loses information).        */
/* Reading R5 (asymmetric min/max group quantization with fp16 meta):         */
/*   groups are g consecutive channels of the transformed vector y;           */
/*   mn, mx = group min and max, then mn+0, mx+0 (so -0 becomes +0);          */
/*   z_h = RD16(mn * 2^-k),  zf = f32(z_h) * 2^k;                             */
/*   s32 = (mx - zf) / (2^b - 1),  s_h = RU16(s32 * 2^-k), sf = f32(s_h)*2^k; */
/*   r = 0 if s_h == 0 else 1/sf;  t = y - zf, p = t * r (each one fp32   */
/*   rounding, no fused multiply-add);                                       */
/*   q = clamp(nearest integer to p, ties to even, 0, 2^b - 1).              */
/* Directed rounding makes the grid zf + q*sf cover [mn, mx]. A non-finite y  */
/* gives NONFINITE; an infinite z_h or s_h gives RANGE (reading R8). The meta */
/* of group j is 4 bytes: s_h then z_h, little-endian.                        */
/* ========================================================================== */
int orc_quantize_vector(const uint16_t *x, int d, int bits, int g,
                        const uint64_t *sign_words, uint8_t *codes,
                        uint8_t *meta) {
  return orc_quantize_vector_q(x, d, bits, g, ORC_QUANT_ASYM, sign_words, codes, meta);
}

/* Reading R19 (symmetric absmax, one of the quantizer variants of the
 * FP4Quant abstract), in the meta format of reading R5 so that the decoder
 * of reading R9 is unchanged:
 *   a = max |y| over the group (+0);  s32 = a / (2^(b-1) - 1);
 *   s_h = RU16(s32 * 2^-k), sf = f32(s_h) * 2^k;  r = 0 if s_h == 0 else 1/sf;
 *   code = clamp(nearest integer to fl(y * r), ties to even, -qh, qh) + 2^(b-1);
 *   z_h = fp16 of -2^(b-1) * f32(s_h) (exact: a power-of-two multiple; +0
 *   when s_h is 0), so zf + code * sf = (code - 2^(b-1)) * sf exactly.
 * A non-finite y gives NONFINITE, an infinite s_h or z_h RANGE (R8). */
/* Reading R22 (the FP4Quant abstract: micro-grouped dual-scale FP4), bits
 * 4, in the 4-byte-per-group meta of reading R6:
 *   a = max |y| over the group (+0);
 *   s2_h = RU16(fl(a / 2688) * 2^-k), s2 = f32(s2_h) * 2^k   (2688 = 6 * 448);
 *   per half-group j (g/2 channels): a_j = max |y| over it,
 *     s1_j = e4m3 RU(fl(a_j / (6 * s2))), at most 448 (0 when s2 is 0);
 *     S_j = s1_j * s2 (exact in fp32), r_j = 0 if S_j == 0 else fl(1 / S_j);
 *   code = e2m1 nearest to fl(y * r_j), ties to even, |.| <= 6;
 *   meta bytes: s2_h (little-endian), s1_0, s1_1.
 * The decoded value e2m1(code) * S_j is exact in fp32. A non-finite y gives
 * NONFINITE, an infinite s2_h RANGE. */
static int quantize_group_fp4(const float *yg, int g, int k, uint8_t *q, uint8_t *m) {
  float a = 0.0f, up = ldexpf(1.0f, k), down = ldexpf(1.0f, -k), s2;
  uint16_t s2h;
  int c, j;
  for (c = 0; c < g; c++)
    if (fabsf(yg[c]) > a) a = fabsf(yg[c]);
  a = a + 0.0f;
  s2h = orc_f32_to_f16_ru((a / 2688.0f) * down);
  s2 = orc_f16_to_f32(s2h) * up;
  m[0] = (uint8_t)(s2h & 0xFF);
  m[1] = (uint8_t)(s2h >> 8);
  if (f16_is_inf(s2h)) {
    for (c = 0; c < g; c++) q[c] = 0;
    m[2] = m[3] = 0;
    return ORC_ERR_RANGE;
  }
  for (j = 0; j < 2; j++) {
    const float *yh = yg + j * (g / 2);
    float aj = 0.0f, S, r;
    int s1;
    for (c = 0; c < g / 2; c++)
      if (fabsf(yh[c]) > aj) aj = fabsf(yh[c]);
    s1 = s2 == 0.0f ? 0 : orc_f32_to_e4m3_ru(aj / (6.0f * s2));
    S = orc_e4m3_to_f32(s1) * s2;
    r = S == 0.0f ? 0.0f : 1.0f / S;
    for (c = 0; c < g / 2; c++) q[j * (g / 2) + c] = (uint8_t)orc_f32_to_e2m1_rne(yh[c] * r);
    m[2 + j] = (uint8_t)s1;
  }
  return ORC_OK;
}

int orc_quantize_vector_q(const uint16_t *x, int d, int bits, int g, int quant,
                          const uint64_t *sign_words, uint8_t *codes,
                          uint8_t *meta) {
  float y[ORC_MAX_D];
  uint8_t q[ORC_MAX_D];
  int k = orc_meta_shift(d);
  float up = ldexpf(1.0f, k), down = ldexpf(1.0f, -k);
  int qmax = (1 << bits) - 1;
  int status = ORC_OK;
  int c, j;

  for (c = 0; c < d; c++) {
    y[c] = orc_bf16_to_f32(x[c]);
    if (sign_bit(sign_words, c)) y[c] = -y[c];
  }
  orc_fwht(y, d);

  for (j = 0; j < d / g; j++) {
    const float *yg = y + j * g;
    float mn = yg[0], mx = yg[0], zf, s32, sf, r;
    uint16_t zh, sh;
    int finite = 1;
    for (c = 0; c < g; c++) {
      if (!isfinite(yg[c])) finite = 0;
      if (yg[c] < mn) mn = yg[c];
      if (yg[c] > mx) mx = yg[c];
    }
    if (!finite) {
      status = ORC_ERR_NONFINITE;
      for (c = 0; c < g; c++) q[j * g + c] = 0;
      memset(meta + 4 * j, 0, 4);
      continue;
    }
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    if (quant == ORC_QUANT_FP4) {
      const int st = quantize_group_fp4(yg, g, k, q + j * g, meta + 4 * j);
      if (st != ORC_OK && status == ORC_OK) status = st;
      continue;
    }
    if (quant == ORC_QUANT_SYM) {
      const float a = fabsf(mn) > fabsf(mx) ? fabsf(mn) : fabsf(mx);
      const int qh = (1 << (bits - 1)) - 1;
      s32 = a / (float)qh;
      sh = orc_f32_to_f16_ru(s32 * down);
      zh = (sh & 0x7FFFu) == 0 ? 0
                               : f32_to_f16_directed(-ldexpf(orc_f16_to_f32(sh), bits - 1), 1);
    } else {
      zh = orc_f32_to_f16_rd(mn * down);
      zf = orc_f16_to_f32(zh) * up;
      s32 = (mx - zf) / (float)qmax;
      sh = orc_f32_to_f16_ru(s32 * down);
    }
    sf = orc_f16_to_f32(sh) * up;
    zf = orc_f16_to_f32(zh) * up;
    if (f16_is_inf(zh) || f16_is_inf(sh)) {
      if (status == ORC_OK) status = ORC_ERR_RANGE;
      for (c = 0; c < g; c++) q[j * g + c] = 0;
    } else {
      r = ((sh & 0x7FFFu) == 0) ? 0.0f : 1.0f / sf;
      for (c = 0; c < g; c++)
        q[j * g + c] = (uint8_t)(quant == ORC_QUANT_SYM
                                     ? orc_quantize_scalar_sym(yg[c], r, bits)
                                     : orc_quantize_scalar(yg[c], zf, r, qmax));
    }
    meta[4 * j + 0] = (uint8_t)(sh & 0xFF);
    meta[4 * j + 1] = (uint8_t)(sh >> 8);
    meta[4 * j + 2] = (uint8_t)(zh & 0xFF);
    meta[4 * j + 3] = (uint8_t)(zh >> 8);
  }
  orc_pack_codes(q, d, bits, codes);
  return status;
}

/* The decoder's transformed values y^ of one vector (fp32):
 *   readings R5 / R19 (reading R9): y^ = zf + q*sf, the product rounded,
 *   then the sum rounded;
 *   reading R22 (FP4): y^ = e2m1(q) * (s1_j * s2), exact. */
static void grid_values(const uint8_t *codes, const uint8_t *meta, int d, int bits, int g,
                        int quant, float *y) {
  uint8_t q[ORC_MAX_D];
  int k = orc_meta_shift(d), c, j;
  float up = ldexpf(1.0f, k);
  orc_unpack_codes(codes, d, bits, q);
  for (j = 0; j < d / g; j++) {
    uint16_t sh = (uint16_t)(meta[4 * j] | (meta[4 * j + 1] << 8));
    uint16_t zh = (uint16_t)(meta[4 * j + 2] | (meta[4 * j + 3] << 8));
    float sf = orc_f16_to_f32(sh) * up;
    float zf = orc_f16_to_f32(zh) * up;
    for (c = j * g; c < (j + 1) * g; c++) {
      if (quant == ORC_QUANT_FP4) {
        const float S = orc_e4m3_to_f32(meta[4 * j + 2 + (c - j * g) / (g / 2)]) * sf;
        y[c] = orc_e2m1_to_f32(q[c]) * S;
      } else {
        float p = (float)q[c] * sf;
        y[c] = zf + p;
      }
    }
  }
}

/* Decode of one vector, the inverse path of [P3]. Reading R9:
 *   y^ as grid_values;
 *   the same butterfly as the encoder (H_d H_d = d I);
 *   x^ = bf16_RNE(sign_c * (u * 2^-log2(d))). */
void orc_dequantize_vector(const uint8_t *codes, const uint8_t *meta, int d,
                           int bits, int g, const uint64_t *sign_words,
                           uint16_t *xhat) {
  orc_dequantize_vector_q(codes, meta, d, bits, g, ORC_QUANT_ASYM, sign_words, xhat);
}

void orc_dequantize_vector_q(const uint8_t *codes, const uint8_t *meta, int d, int bits, int g,
                             int quant, const uint64_t *sign_words, uint16_t *xhat) {
  float y[ORC_MAX_D];
  int l2d = 0, c;
  float inv_d;
  while ((1 << l2d) < d) l2d++;
  inv_d = ldexpf(1.0f, -l2d);
  grid_values(codes, meta, d, bits, g, quant, y);
  orc_fwht(y, d);
  for (c = 0; c < d; c++) {
    float u = y[c] * inv_d;
    if (sign_bit(sign_words, c)) u = -u;
    xhat[c] = orc_f32_to_bf16_rne(u);
  }
}

/* The same decode without the final bf16 rounding, in double: y^ as above
 * (fp32, the decoder's value), then x^_c = sign_c * (H_d y^)_c / d evaluated in
 * double (every fp32 input and product is exact there; the butterfly's sums
 * round at 2^-53). Reading R18: these are the key and value vectors an
 * attention step that consumes the compressed cache works with; the bf16
 * rounding of the decoder moves each of them by at most half a bf16 ulp. */
void orc_dequantize_vector_f64(const uint8_t *codes, const uint8_t *meta, int d,
                               int bits, int g, const uint64_t *sign_words,
                               double *xhat) {
  orc_dequantize_vector_f64_q(codes, meta, d, bits, g, ORC_QUANT_ASYM, sign_words, xhat);
}

void orc_dequantize_vector_f64_q(const uint8_t *codes, const uint8_t *meta, int d, int bits,
                                 int g, int quant, const uint64_t *sign_words, double *xhat) {
  float yf[ORC_MAX_D];
  double y[ORC_MAX_D];
  int c, h, i;
  grid_values(codes, meta, d, bits, g, quant, yf);
  for (c = 0; c < d; c++) y[c] = (double)yf[c];
  for (h = 1; h < d; h *= 2)
    for (i = 0; i < d; i++)
      if ((i & h) == 0) {
        double a = y[i], b = y[i + h];
        y[i] = a + b;
        y[i + h] = a - b;
      }
  for (c = 0; c < d; c++) xhat[c] = (sign_bit(sign_words, c) ? -y[c] : y[c]) / (double)d;
}

/* ========================================================================== */
/* Lossless stage on one 16 KB chunk ([P2]: LC-style backend composed of      */
/* primitives). The components are a bit-plane shuffle, zero-byte            */
/* elimination with a bitmap, and a prefix sum over chunk sizes.              */
/* Reading R10: the chunk is 4096 little-endian u32 words w[j]; plane p       */
/* (p = 0..31, LSB first) is 512 bytes; bit (j mod 8) of byte p*512 + j/8 of  */
/* the output is bit p of w[j]. Only full 16 KB chunks are shuffled.          */
/* ========================================================================== */
static uint32_t word_at(const uint8_t *b, int j) {
  return (uint32_t)b[4 * j] | ((uint32_t)b[4 * j + 1] << 8) |
         ((uint32_t)b[4 * j + 2] << 16) | ((uint32_t)b[4 * j + 3] << 24);
}

void orc_bitplane_shuffle(const uint8_t *in, uint8_t *out) {
  int p, j;
  memset(out, 0, ORC_CHUNK);
  for (j = 0; j < ORC_CHUNK / 4; j++) {
    uint32_t w = word_at(in, j);
    for (p = 0; p < 32; p++)
      if ((w >> p) & 1u) out[p * 512 + j / 8] |= (uint8_t)(1u << (j % 8));
  }
}

void orc_bitplane_unshuffle(const uint8_t *in, uint8_t *out) {
  int p, j;
  for (j = 0; j < ORC_CHUNK / 4; j++) {
    uint32_t w = 0;
    for (p = 0; p < 32; p++)
      if ((in[p * 512 + j / 8] >> (j % 8)) & 1u) w |= 1u << p;
    out[4 * j] = (uint8_t)w;
    out[4 * j + 1] = (uint8_t)(w >> 8);
    out[4 * j + 2] = (uint8_t)(w >> 16);
    out[4 * j + 3] = (uint8_t)(w >> 24);
  }
}

/* Reading R11: zero-byte elimination writes a 2048-byte bitmap (bit i, LSB
 * first, says shuffled byte i is nonzero) followed by the nonzero bytes in
 * order. It is used only if strictly shorter than the chunk; otherwise the
 * chunk is stored raw, as the original unshuffled bytes. A short chunk (the
 * tail of a region) is always raw. The decoder tells the two apart by size:
 * size == chunk length means raw. Returns the encoded size. */
uint32_t orc_lossless_encode_chunk(const uint8_t *in, uint32_t len,
                                   uint8_t *out) {
  uint8_t s[ORC_CHUNK];
  uint32_t nnz = 0, i;
  if (len < ORC_CHUNK) {
    memcpy(out, in, len);
    return len;
  }
  orc_bitplane_shuffle(in, s);
  for (i = 0; i < ORC_CHUNK; i++)
    if (s[i]) nnz++;
  if (ORC_BITMAP + nnz >= ORC_CHUNK) {
    memcpy(out, in, ORC_CHUNK);
    return ORC_CHUNK;
  }
  memset(out, 0, ORC_BITMAP);
  nnz = 0;
  for (i = 0; i < ORC_CHUNK; i++) {
    if (s[i]) {
      out[i / 8] |= (uint8_t)(1u << (i % 8));
      out[ORC_BITMAP + nnz] = s[i];
      nnz++;
    }
  }
  return ORC_BITMAP + nnz;
}

int orc_lossless_decode_chunk(const uint8_t *in, uint32_t size, uint32_t len,
                              uint8_t *out) {
  uint8_t s[ORC_CHUNK];
  uint32_t i, pos = 0;
  if (size == len) {
    memcpy(out, in, len);
    return ORC_OK;
  }
  if (len != ORC_CHUNK || size < ORC_BITMAP || size >= ORC_CHUNK)
    return ORC_ERR_CORRUPT;
  for (i = 0; i < ORC_CHUNK; i++) {
    if ((in[i / 8] >> (i % 8)) & 1u) {
      if (ORC_BITMAP + pos >= size) return ORC_ERR_CORRUPT;
      s[i] = in[ORC_BITMAP + pos];
      pos++;
    } else {
      s[i] = 0;
    }
  }
  if (ORC_BITMAP + pos != size) return ORC_ERR_CORRUPT;
  orc_bitplane_unshuffle(s, out);
  return ORC_OK;
}

/* ========================================================================== */
/* Composable lossless pipelines ([P2]: the backend is "searchable", built   */
/* from primitives composed into pipelines). Reading R17 adds two primitives */
/* to the bit-plane shuffle and zero-byte elimination above, each pinned on  */
/* its own: an XOR of each 32-bit word with the previous word, restarting at */
/* every run of 32 vectors (the fp16 scale/zero pairs of neighbouring groups */
/* and tokens share their sign and exponent bits, so the XOR clears most of  */
/* those bit planes), and a second level of zero-byte elimination applied to */
/* the 2048-byte bitmap. A chunk's pipeline id (0..3, see kvc_oracle.h) says */
/* which were applied.                                                        */
/* ========================================================================== */
static void put_word(uint8_t *b, int j, uint32_t w) {
  b[4 * j] = (uint8_t)w;
  b[4 * j + 1] = (uint8_t)(w >> 8);
  b[4 * j + 2] = (uint8_t)(w >> 16);
  b[4 * j + 3] = (uint8_t)(w >> 24);
}

/* w'[j] = w[j] XOR w[j-1] unless j starts a run (j mod run_words == 0), with
 * w the original words; in place, so from the last word down. run_words is
 * 32 vectors' worth of words. */
void orc_xor_words(uint8_t *chunk, uint32_t n_words, int run_words) {
  int64_t j;
  for (j = (int64_t)n_words - 1; j >= 1; j--)
    if (j % run_words != 0)
      put_word(chunk, (int)j, word_at(chunk, (int)j) ^ word_at(chunk, (int)j - 1));
}

/* The inverse: from the first word up, each word XOR the restored previous
 * one, except at the start of a run. */
void orc_unxor_words(uint8_t *chunk, uint32_t n_words, int run_words) {
  uint32_t j;
  for (j = 1; j < n_words; j++)
    if (j % run_words != 0)
      put_word(chunk, (int)j, word_at(chunk, (int)j) ^ word_at(chunk, (int)j - 1));
}

/* Two-level zero-byte elimination of a shuffled chunk: the 2048-byte bitmap B
 * of the one-level form (bit i = shuffled byte i is nonzero) is itself
 * reduced to a 256-byte bitmap B2 (bit i = byte i of B is nonzero) and its
 * nonzero bytes. Output: B2, then the nonzero bytes of B in order, then the
 * nonzero shuffled bytes in order. Returns the size. */
uint32_t orc_ze2_encode(const uint8_t *sh, uint8_t *out) {
  uint8_t b[ORC_BITMAP];
  uint32_t i, pos;
  memset(b, 0, sizeof b);
  for (i = 0; i < ORC_CHUNK; i++)
    if (sh[i]) b[i / 8] |= (uint8_t)(1u << (i % 8));
  memset(out, 0, ORC_BITMAP2);
  pos = ORC_BITMAP2;
  for (i = 0; i < ORC_BITMAP; i++)
    if (b[i]) {
      out[i / 8] |= (uint8_t)(1u << (i % 8));
      out[pos++] = b[i];
    }
  for (i = 0; i < ORC_CHUNK; i++)
    if (sh[i]) out[pos++] = sh[i];
  return pos;
}

int orc_ze2_decode(const uint8_t *in, uint32_t size, uint8_t *sh) {
  uint8_t b[ORC_BITMAP];
  uint32_t i, pos = ORC_BITMAP2;
  if (size < ORC_BITMAP2) return ORC_ERR_CORRUPT;
  for (i = 0; i < ORC_BITMAP; i++) {
    if ((in[i / 8] >> (i % 8)) & 1u) {
      if (pos >= size) return ORC_ERR_CORRUPT;
      b[i] = in[pos++];
    } else {
      b[i] = 0;
    }
  }
  for (i = 0; i < ORC_CHUNK; i++) {
    if ((b[i / 8] >> (i % 8)) & 1u) {
      if (pos >= size) return ORC_ERR_CORRUPT;
      sh[i] = in[pos++];
    } else {
      sh[i] = 0;
    }
  }
  return pos == size ? ORC_OK : ORC_ERR_CORRUPT;
}

/* A full chunk through pipeline `pipe` (no raw fallback, so `out` needs room
 * for ORC_BITMAP2 + ORC_BITMAP + ORC_CHUNK bytes). s: words per vector (the
 * XOR of pipelines 1 and 3 restarts every 32 vectors, 32 * s words). Returns
 * the size. */
uint32_t orc_chunk_encode_pipe(const uint8_t *in, int pipe, int s, uint8_t *out) {
  uint8_t w[ORC_CHUNK], sh[ORC_CHUNK];
  uint32_t i, nnz = 0;
  memcpy(w, in, ORC_CHUNK);
  if (pipe == ORC_PIPE_XOR_ZE || pipe == ORC_PIPE_XOR_ZE2) orc_xor_words(w, ORC_CHUNK / 4, 32 * s);
  orc_bitplane_shuffle(w, sh);
  if (pipe == ORC_PIPE_ZE2 || pipe == ORC_PIPE_XOR_ZE2) return orc_ze2_encode(sh, out);
  memset(out, 0, ORC_BITMAP);
  for (i = 0; i < ORC_CHUNK; i++) {
    if (sh[i]) {
      out[i / 8] |= (uint8_t)(1u << (i % 8));
      out[ORC_BITMAP + nnz++] = sh[i];
    }
  }
  return ORC_BITMAP + nnz;
}

/* Inverse of any pipeline, or a raw chunk (size == len, pipe 0). */
int orc_chunk_decode_pipe(const uint8_t *in, uint32_t size, uint32_t len, int pipe, int s,
                          uint8_t *out) {
  uint8_t sh[ORC_CHUNK];
  int st;
  if (pipe < 0 || pipe > 3) return ORC_ERR_CORRUPT;
  if (size == len) {
    if (pipe != 0) return ORC_ERR_CORRUPT;
    memcpy(out, in, len);
    return ORC_OK;
  }
  if (len != ORC_CHUNK || size >= ORC_CHUNK) return ORC_ERR_CORRUPT;
  if (pipe == ORC_PIPE_ZE || pipe == ORC_PIPE_XOR_ZE) {
    st = orc_lossless_decode_chunk(in, size, len, out);
    if (st != ORC_OK) return st;
  } else {
    st = orc_ze2_decode(in, size, sh);
    if (st != ORC_OK) return st;
    orc_bitplane_unshuffle(sh, out);
  }
  if (pipe == ORC_PIPE_XOR_ZE || pipe == ORC_PIPE_XOR_ZE2)
    orc_unxor_words(out, ORC_CHUNK / 4, 32 * s);
  return ORC_OK;
}

/* Reading R17, the encoder's choice for one chunk: FIXED tries pipeline 0,
 * SEARCH every candidate of the region (code chunks 0 and 2; meta chunks 0..3
 * when a vector holds at least two meta words, else 0 and 1), NONE none. The
 * shortest candidate wins, ties to the lower id; it is used only if strictly
 * shorter than the chunk, which is otherwise stored raw (pipeline 0). Short
 * chunks are always raw. */
uint32_t orc_chunk_encode_select(const uint8_t *in, uint32_t len, int is_meta, int s, int mode,
                                 uint8_t *out, int *pipe) {
  uint8_t tmp[ORC_BITMAP2 + ORC_BITMAP + ORC_CHUNK]; /* a candidate may exceed the chunk */
  int cand[4], n = 0, k, best = -1;
  uint32_t best_size = len, sz;
  *pipe = 0;
  if (len < ORC_CHUNK || mode == ORC_LOSSLESS_NONE) {
    memcpy(out, in, len);
    return len;
  }
  cand[n++] = ORC_PIPE_ZE;
  if (mode == ORC_LOSSLESS_SEARCH) {
    if (is_meta) cand[n++] = ORC_PIPE_XOR_ZE;
    if (!is_meta || s >= 2) cand[n++] = ORC_PIPE_ZE2;
    if (is_meta && s >= 2) cand[n++] = ORC_PIPE_XOR_ZE2;
  }
  for (k = 0; k < n; k++) {
    sz = orc_chunk_encode_pipe(in, cand[k], s, tmp);
    if (sz < best_size) {
      best_size = sz;
      best = cand[k];
    }
  }
  if (best < 0) {
    memcpy(out, in, len);
    return len;
  }
  orc_chunk_encode_pipe(in, best, s, out);
  *pipe = best;
  return best_size;
}

/* ========================================================================== */
/* Stream layout. Reading R12 (self-describing stream, little-endian):        */
/*   [0,64)    header: u32 magic "KVC1", u16 version 1, u16 header bytes 64,  */
/*             u8 bits, u8 k, u8 origin (0 dense, 1 paged), u8 flags (bit 0: */
/*             some code chunk uses zero-byte elimination), u32 group,        */
/*             u32 layers, u32 kv (=2), u32 kv_heads, u32 head_dim,           */
/*             u64 tokens (sum over requests), u64 sign_seed,                 */
/*             u32 n_requests, u32 n_chunks, u64 stream_bytes;                */
/*   then      u64 chunk table [n_chunks]: bits 0..15 = unpadded size,        */
/*             bits 16..59 = offset from the data base in 16-byte units,      */
/*             bits 60..63 = the chunk's lossless pipeline id (R17; 0 raw);   */
/*   then      u32 token lengths [n_requests];                                */
/*   then      zeros up to a 16-byte boundary = data base;                    */
/*   then      the chunks, each zero-padded to 16 bytes, at their offsets.    */
/* The codes region (packed codes of all vectors in logical order) and the    */
/* meta region (4 bytes per group) are cut into 16 KB chunks separately (a    */
/* meta chunk covers R = g*b/32 code chunks: a "segment"). Stream order is    */
/* every code chunk, then every meta chunk. Chunk offsets are the exclusive   */
/* prefix sum of the padded chunk sizes in that order.                        */
/* ========================================================================== */
static uint64_t round16(uint64_t x) { return (x + 15u) & ~(uint64_t)15u; }

/* Byte offset (from the data base) held in bits 16..59 of a table entry. */
#define ENTRY_OFFSET(e) ((((e) >> 16) & 0xFFFFFFFFFFFull) * 16)

int orc_check_desc(const orc_desc *d) {
  int r;
  if (!d) return ORC_ERR_INVALID_ARG;
  if (d->bits != 2 && d->bits != 4 && d->bits != 8) return ORC_ERR_UNSUPPORTED;
  if (d->quant != ORC_QUANT_ASYM && d->quant != ORC_QUANT_SYM && d->quant != ORC_QUANT_FP4)
    return ORC_ERR_UNSUPPORTED;
  if (d->quant == ORC_QUANT_FP4 && d->bits != 4) return ORC_ERR_UNSUPPORTED;
  if (d->signs != ORC_SIGNS_GLOBAL && d->signs != ORC_SIGNS_PER_VECTOR)
    return ORC_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256)
    return ORC_ERR_UNSUPPORTED;
  if (d->group != 32 && d->group != 64 && d->group != 128)
    return ORC_ERR_UNSUPPORTED;
  if (d->group > d->head_dim) return ORC_ERR_UNSUPPORTED;
  if (d->layers < 0 || d->kv_heads < 0 || d->n_requests < 0)
    return ORC_ERR_INVALID_ARG;
  if (d->n_requests > 0 && !d->token_lens) return ORC_ERR_INVALID_ARG;
  for (r = 0; r < d->n_requests; r++)
    if (d->token_lens[r] > 0x7FFFFFFFu) return ORC_ERR_INVALID_ARG;
  return ORC_OK;
}

int orc_layout_of(const orc_desc *d, orc_layout *lay) {
  uint64_t T = 0, i;
  int st = orc_check_desc(d), r;
  if (st != ORC_OK) return st;
  for (r = 0; r < d->n_requests; r++) T += d->token_lens[r];
  lay->V = (uint64_t)d->layers * 2u * (uint64_t)d->kv_heads * T;
  lay->code_bytes = (uint32_t)(d->head_dim * d->bits / 8);
  lay->meta_bytes = (uint32_t)((d->head_dim / d->group) * 4);
  lay->vec_per_code = ORC_CHUNK / lay->code_bytes;
  lay->code_per_seg = (uint32_t)(d->group * d->bits / 32);
  lay->n_code = (lay->V + lay->vec_per_code - 1) / lay->vec_per_code;
  lay->n_seg = (lay->n_code + lay->code_per_seg - 1) / lay->code_per_seg;
  lay->n_meta = lay->n_seg;
  lay->n_chunks = lay->n_code + lay->n_meta;
  lay->data_base =
      round16(ORC_HEADER + 8u * lay->n_chunks + 4u * (uint64_t)d->n_requests);
  lay->max_bytes = lay->data_base;
  /* every chunk at its raw length, padded */
  for (i = 0; i < lay->n_code; i++) {
    uint64_t v0 = i * lay->vec_per_code;
    uint64_t nv = lay->V - v0 < lay->vec_per_code ? lay->V - v0 : lay->vec_per_code;
    lay->max_bytes += round16(nv * lay->code_bytes);
  }
  for (i = 0; i < lay->n_meta; i++) {
    uint64_t vm = (uint64_t)lay->vec_per_code * lay->code_per_seg;
    uint64_t v0 = i * vm;
    uint64_t nv = lay->V - v0 < vm ? lay->V - v0 : vm;
    lay->max_bytes += round16(nv * lay->meta_bytes);
  }
  return ORC_OK;
}

uint64_t orc_max_compressed_bytes(const orc_desc *d) {
  orc_layout lay;
  if (orc_layout_of(d, &lay) != ORC_OK) return 0;
  return lay.max_bytes;
}

uint64_t orc_code_chunk_index(const orc_layout *lay, uint64_t c) {
  (void)lay;
  return c;
}

uint64_t orc_meta_chunk_index(const orc_layout *lay, uint64_t s) {
  return lay->n_code + s;
}

static void put16(uint8_t *p, uint16_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
}
static void put32(uint8_t *p, uint32_t v) {
  int i;
  for (i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put64(uint8_t *p, uint64_t v) {
  int i;
  for (i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint16_t get16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get32(const uint8_t *p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) |
         ((uint32_t)p[3] << 24);
}
static uint64_t get64(const uint8_t *p) {
  return (uint64_t)get32(p) | ((uint64_t)get32(p + 4) << 32);
}

/* The (layer, kv, head) index of stream vector v (order [layer][kv][head]
 * [request][token], requests concatenated): v / T, T the total tokens. */
static uint64_t vector_index(const orc_desc *d, const orc_layout *lay, uint64_t v) {
  uint64_t T = lay->V / (2u * (uint64_t)d->layers * (uint64_t)d->kv_heads);
  return v / T;
}

/* Segment s's chunks from its vectors, for a layout computed once by the
 * caller (orc_encode_segment and the compressor below). */
static int encode_segment_in(const orc_desc *d, const orc_layout *lay, uint64_t s,
                             const uint16_t *vectors, uint8_t *chunks,
                             uint32_t *sizes, uint8_t *pipes, uint32_t *n_out) {
  int pipe;
  uint64_t vm, v0, nv, v, c0, c1, c;
  uint8_t *codes, *meta;
  uint64_t sw[4];
  uint32_t pos = 0;
  int st = ORC_OK, vst;
  vm = (uint64_t)lay->vec_per_code * lay->code_per_seg;
  v0 = s * vm;
  nv = lay->V - v0 < vm ? lay->V - v0 : vm;
  orc_sign_words(d->sign_seed, d->head_dim, sw);
  codes = (uint8_t *)malloc((size_t)(nv * lay->code_bytes));
  meta = (uint8_t *)malloc((size_t)(nv * lay->meta_bytes));
  for (v = 0; v < nv; v++) {
    if (d->signs == ORC_SIGNS_PER_VECTOR)
      orc_sign_words_at(d->sign_seed, d->head_dim, vector_index(d, lay, v0 + v), sw);
    vst = orc_quantize_vector_q(vectors + v * d->head_dim, d->head_dim, d->bits,
                                d->group, d->quant, sw, codes + v * lay->code_bytes,
                                meta + v * lay->meta_bytes);
    if (vst != ORC_OK && st == ORC_OK) st = vst;
  }
  c0 = s * lay->code_per_seg;
  c1 = c0 + lay->code_per_seg < lay->n_code ? c0 + lay->code_per_seg : lay->n_code;
  *n_out = 0;
  for (c = c0; c < c1; c++) {
    uint64_t a = (c - c0) * lay->vec_per_code;
    uint64_t b = a + lay->vec_per_code < nv ? a + lay->vec_per_code : nv;
    uint32_t sz = orc_chunk_encode_select(
        codes + a * lay->code_bytes, (uint32_t)((b - a) * lay->code_bytes), 0,
        (int)(lay->code_bytes / 4), d->lossless, chunks + pos, &pipe);
    pipes[*n_out] = (uint8_t)pipe;
    sizes[(*n_out)++] = sz;
    pos += sz;
  }
  sizes[*n_out] = orc_chunk_encode_select(meta, (uint32_t)(nv * lay->meta_bytes), 1,
                                          (int)(lay->meta_bytes / 4), d->lossless,
                                          chunks + pos, &pipe);
  pipes[(*n_out)++] = (uint8_t)pipe;
  free(codes);
  free(meta);
  return st;
}

int orc_encode_segment(const orc_desc *d, uint64_t s, const uint16_t *vectors,
                       uint8_t *chunks, uint32_t *sizes, uint8_t *pipes, uint32_t *n_out) {
  orc_layout lay;
  int st = orc_layout_of(d, &lay);
  if (st != ORC_OK) return st;
  if (s >= lay.n_seg) return ORC_ERR_INVALID_ARG;
  return encode_segment_in(d, &lay, s, vectors, chunks, sizes, pipes, n_out);
}

static int decode_segment_in(const orc_desc *d, const orc_layout *lay, uint64_t s,
                             const uint8_t *chunks, const uint32_t *sizes,
                             const uint8_t *pipes, uint16_t *vectors, double *vals) {
  uint64_t vm, v0, nv, v, c0, c1, c, i = 0;
  uint8_t *codes, *meta;
  uint64_t sw[4];
  uint32_t pos = 0;
  int st = ORC_OK;
  vm = (uint64_t)lay->vec_per_code * lay->code_per_seg;
  v0 = s * vm;
  nv = lay->V - v0 < vm ? lay->V - v0 : vm;
  orc_sign_words(d->sign_seed, d->head_dim, sw);
  codes = (uint8_t *)malloc((size_t)(nv * lay->code_bytes));
  meta = (uint8_t *)malloc((size_t)(nv * lay->meta_bytes));
  c0 = s * lay->code_per_seg;
  c1 = c0 + lay->code_per_seg < lay->n_code ? c0 + lay->code_per_seg : lay->n_code;
  for (c = c0; c < c1 && st == ORC_OK; c++, i++) {
    uint64_t a = (c - c0) * lay->vec_per_code;
    uint64_t b = a + lay->vec_per_code < nv ? a + lay->vec_per_code : nv;
    /* code chunks: pipelines 0 and 2 only */
    if (pipes[i] != ORC_PIPE_ZE && pipes[i] != ORC_PIPE_ZE2) st = ORC_ERR_CORRUPT;
    else
      st = orc_chunk_decode_pipe(chunks + pos, sizes[i], (uint32_t)((b - a) * lay->code_bytes),
                                 pipes[i], (int)(lay->code_bytes / 4),
                                 codes + a * lay->code_bytes);
    pos += sizes[i];
  }
  if (st == ORC_OK)
    st = orc_chunk_decode_pipe(chunks + pos, sizes[i], (uint32_t)(nv * lay->meta_bytes),
                               pipes[i], (int)(lay->meta_bytes / 4), meta);
  if (st == ORC_OK)
    for (v = 0; v < nv; v++) {
      if (d->signs == ORC_SIGNS_PER_VECTOR)
        orc_sign_words_at(d->sign_seed, d->head_dim, vector_index(d, lay, v0 + v), sw);
      if (vals)
        orc_dequantize_vector_f64_q(codes + v * lay->code_bytes, meta + v * lay->meta_bytes,
                                    d->head_dim, d->bits, d->group, d->quant, sw,
                                    vals + v * d->head_dim);
      else
        orc_dequantize_vector_q(codes + v * lay->code_bytes, meta + v * lay->meta_bytes,
                                d->head_dim, d->bits, d->group, d->quant, sw,
                                vectors + v * d->head_dim);
    }
  free(codes);
  free(meta);
  return st;
}

int orc_decode_segment(const orc_desc *d, uint64_t s, const uint8_t *chunks,
                       const uint32_t *sizes, const uint8_t *pipes, uint16_t *vectors) {
  orc_layout lay;
  int st = orc_layout_of(d, &lay);
  if (st != ORC_OK) return st;
  if (s >= lay.n_seg) return ORC_ERR_INVALID_ARG;
  return decode_segment_in(d, &lay, s, chunks, sizes, pipes, vectors, NULL);
}

/* Runs fn(job, s) for every segment s in [0, n_seg) on n_threads threads
 * (segment s on thread s mod n_threads; 1 thread: the caller, in order).
 * Segments are independent, so the order does not change any result. */
typedef struct {
  void *job;
  void (*fn)(void *job, uint64_t s);
  uint64_t first, n_seg, step;
} seg_pool_part;

static void *seg_pool_run(void *arg) {
  seg_pool_part *p = (seg_pool_part *)arg;
  uint64_t s;
  for (s = p->first; s < p->n_seg; s += p->step) p->fn(p->job, s);
  return NULL;
}

static void for_each_segment(uint64_t n_seg, int n_threads, void *job,
                             void (*fn)(void *job, uint64_t s)) {
  pthread_t th[ORC_MAX_THREADS];
  seg_pool_part part[ORC_MAX_THREADS];
  int t, started = 0;
  if (n_threads < 1) n_threads = 1;
  if (n_threads > ORC_MAX_THREADS) n_threads = ORC_MAX_THREADS;
  if ((uint64_t)n_threads > n_seg) n_threads = n_seg ? (int)n_seg : 1;
  for (t = 0; t < n_threads; t++) {
    part[t].job = job;
    part[t].fn = fn;
    part[t].first = (uint64_t)t;
    part[t].n_seg = n_seg;
    part[t].step = (uint64_t)n_threads;
  }
  for (t = 1; t < n_threads; t++)
    if (pthread_create(&th[t], NULL, seg_pool_run, &part[t]) == 0) started = t;
    else break;
  /* threads that could not start leave their segments to this thread */
  if (started + 1 < n_threads) {
    for (t = started + 1; t < n_threads; t++) seg_pool_run(&part[t]);
  }
  seg_pool_run(&part[0]);
  for (t = 1; t <= started; t++) pthread_join(th[t], NULL);
}

/* Reading R16 (the encoder's choice for the code region; a decoder accepts
 * either outcome). Storing a code chunk eliminated shifts every later code
 * chunk, so elimination in the code region is kept only if it pays for that
 * shift: with S = the padded bytes it saves over all code chunks and T = the
 * padded bytes of the code chunks from the first shrinking one to the end of
 * the region, it is kept iff 64 * S >= T; otherwise every code chunk is
 * stored raw. 1/64 is where the time to move T bytes through HBM twice (read
 * and write, about 6.4 TB/s) equals the time to send S bytes over a
 * 400 Gbit/s link. sizes[c] and lens[c] are the eliminated-or-raw size and
 * the raw length of code chunk c, in code-chunk order. Returns 1 if some
 * chunk shrinks and elimination pays, 0 otherwise. */
int orc_code_elim_pays(const uint32_t *sizes, const uint32_t *lens, uint64_t n_code) {
  uint64_t c, S = 0, T = 0;
  int seen = 0;
  for (c = 0; c < n_code; c++) {
    if (sizes[c] != lens[c]) seen = 1;
    if (seen) {
      T += round16(lens[c]);
      S += round16(lens[c]) - round16(sizes[c]);
    }
  }
  return seen && 64 * S >= T;
}

/* One segment of the compressor: its chunks go to the store slots of their
 * stream chunk indices. */
typedef struct {
  const orc_desc *d;
  const orc_layout *lay;
  const uint16_t *vectors;
  uint8_t *store;
  uint32_t *all_sizes;
  uint8_t *all_pipes;
  uint64_t *where;
  int *seg_status;
} enc_job;

static void enc_one_segment(void *arg, uint64_t s) {
  enc_job *j = (enc_job *)arg;
  const orc_layout *lay = j->lay;
  uint64_t vm = (uint64_t)lay->vec_per_code * lay->code_per_seg;
  uint8_t *seg = (uint8_t *)malloc((size_t)(lay->code_per_seg + 1) * ORC_CHUNK);
  uint32_t sizes[ORC_MAX_SEG + 1], n, k, pos = 0;
  uint8_t pipes[ORC_MAX_SEG + 1];
  j->seg_status[s] = encode_segment_in(j->d, lay, s, j->vectors + s * vm * j->d->head_dim,
                                       seg, sizes, pipes, &n);
  for (k = 0; k < n; k++) {
    uint64_t idx = (k + 1 < n) ? orc_code_chunk_index(lay, s * lay->code_per_seg + k)
                               : orc_meta_chunk_index(lay, s);
    memcpy(j->store + idx * ORC_CHUNK, seg + pos, sizes[k]);
    j->all_sizes[idx] = sizes[k];
    j->all_pipes[idx] = pipes[k];
    j->where[idx] = idx * ORC_CHUNK;
    pos += sizes[k];
  }
  free(seg);
}

int orc_compress(const orc_desc *d, const uint16_t *vectors, uint8_t *out,
                 uint64_t capacity, uint64_t *out_bytes) {
  return orc_compress_mt(d, vectors, out, capacity, out_bytes, 1);
}

int orc_compress_mt(const orc_desc *d, const uint16_t *vectors, uint8_t *out,
                    uint64_t capacity, uint64_t *out_bytes, int n_threads) {
  orc_layout lay;
  uint64_t s, off = 0, T = 0, i;
  uint8_t *store;
  uint32_t *all_sizes;
  uint8_t *all_pipes;
  uint64_t *where; /* chunk index -> position in store */
  int *seg_status;
  enc_job job;
  int st = orc_layout_of(d, &lay), r;
  if (st != ORC_OK) return st;
  if (capacity < lay.max_bytes) return ORC_ERR_CAPACITY;
  for (r = 0; r < d->n_requests; r++) T += d->token_lens[r];
  memset(out, 0, (size_t)lay.data_base);
  put32(out + 0, ORC_MAGIC);
  put16(out + 4, 1);
  put16(out + 6, ORC_HEADER);
  out[8] = (uint8_t)d->bits;
  out[9] = (uint8_t)orc_meta_shift(d->head_dim);
  out[10] = (uint8_t)d->origin;
  /* header flags: bit 0 set below; bits 1..2 the quantizer (R19), bit 3
     the sign diagonals (R20) */
  out[11] = (uint8_t)((d->quant << 1) | (d->signs << 3));
  put32(out + 12, (uint32_t)d->group);
  put32(out + 16, (uint32_t)d->layers);
  put32(out + 20, 2);
  put32(out + 24, (uint32_t)d->kv_heads);
  put32(out + 28, (uint32_t)d->head_dim);
  put64(out + 32, T);
  put64(out + 40, d->sign_seed);
  put32(out + 48, (uint32_t)d->n_requests);
  put32(out + 52, (uint32_t)lay.n_chunks);
  for (r = 0; r < d->n_requests; r++)
    put32(out + ORC_HEADER + 8 * lay.n_chunks + 4 * r, d->token_lens[r]);
  /* encode every segment, remembering where each chunk's bytes are */
  store = (uint8_t *)malloc((size_t)(lay.n_chunks ? lay.n_chunks : 1) * ORC_CHUNK);
  all_sizes = (uint32_t *)malloc((size_t)(lay.n_chunks ? lay.n_chunks : 1) * 4);
  all_pipes = (uint8_t *)malloc((size_t)(lay.n_chunks ? lay.n_chunks : 1));
  where = (uint64_t *)malloc((size_t)(lay.n_chunks ? lay.n_chunks : 1) * 8);
  seg_status = (int *)malloc((size_t)(lay.n_seg ? lay.n_seg : 1) * sizeof(int));
  job.d = d;
  job.lay = &lay;
  job.vectors = vectors;
  job.store = store;
  job.all_sizes = all_sizes;
  job.all_pipes = all_pipes;
  job.where = where;
  job.seg_status = seg_status;
  for_each_segment(lay.n_seg, n_threads, &job, enc_one_segment);
  /* the first error in segment order wins */
  for (s = 0; s < lay.n_seg; s++)
    if (seg_status[s] != ORC_OK && st == ORC_OK) st = seg_status[s];
  free(seg_status);
  /* reading R16: keep elimination in the code region only if it pays for
     the shift of the code chunks after the first shrinking one */
  if (lay.n_code) {
    uint32_t *csz = (uint32_t *)malloc((size_t)lay.n_code * 4);
    uint32_t *clen = (uint32_t *)malloc((size_t)lay.n_code * 4);
    for (i = 0; i < lay.n_code; i++) {
      uint64_t nv = lay.V - i * lay.vec_per_code;
      if (nv > lay.vec_per_code) nv = lay.vec_per_code;
      csz[i] = all_sizes[orc_code_chunk_index(&lay, i)];
      clen[i] = (uint32_t)(nv * lay.code_bytes);
    }
    if (!orc_code_elim_pays(csz, clen, lay.n_code)) {
      uint8_t raw[ORC_CHUNK];
      for (i = 0; i < lay.n_code; i++) {
        uint64_t idx = orc_code_chunk_index(&lay, i);
        if (csz[i] == clen[i]) continue;
        if (orc_chunk_decode_pipe(store + where[idx], csz[i], clen[i], all_pipes[idx],
                                  (int)(lay.code_bytes / 4), raw) != ORC_OK &&
            st == ORC_OK)
          st = ORC_ERR_CORRUPT; /* cannot happen: the chunk was just encoded */
        memcpy(store + where[idx], raw, clen[i]);
        all_sizes[idx] = clen[i];
        all_pipes[idx] = 0;
      }
    }
    free(csz);
    free(clen);
  }
  /* lay the chunks out in index order */
  for (i = 0; i < lay.n_chunks; i++) {
    uint64_t padded = round16(all_sizes[i]);
    /* entry: bits 0..15 size, 16..59 offset / 16, 60..63 pipeline id */
    put64(out + ORC_HEADER + 8 * i,
          ((uint64_t)all_pipes[i] << 60) | ((off / 16) << 16) | all_sizes[i]);
    memset(out + lay.data_base + off, 0, (size_t)padded);
    memcpy(out + lay.data_base + off, store + where[i], all_sizes[i]);
    off += padded;
  }
  /* header flags, bit 0: some code chunk uses zero-byte elimination (a
     decoder may use it to skip looking for such chunks) */
  for (i = 0; i < lay.n_code; i++) {
    uint64_t nv = lay.V - i * lay.vec_per_code;
    if (nv > lay.vec_per_code) nv = lay.vec_per_code;
    if (all_sizes[orc_code_chunk_index(&lay, i)] != nv * lay.code_bytes) {
      out[11] |= 1;
      break;
    }
  }
  free(store);
  free(all_sizes);
  free(all_pipes);
  free(where);
  put64(out + 56, lay.data_base + off);
  *out_bytes = lay.data_base + off;
  return st;
}

/* One segment of the decompressor: its chunks are gathered from the stream
 * by the (already validated) chunk table and decoded. */
typedef struct {
  const orc_desc *d;
  const orc_layout *lay;
  const uint8_t *stream;
  uint16_t *vectors;
  double *vals; /* non-null: unrounded values instead of bf16 */
  int *seg_status;
} dec_job;

static void dec_one_segment(void *arg, uint64_t s) {
  dec_job *j = (dec_job *)arg;
  const orc_layout *lay = j->lay;
  uint64_t vm = (uint64_t)lay->vec_per_code * lay->code_per_seg;
  uint64_t c0 = s * lay->code_per_seg;
  uint64_t c1 = c0 + lay->code_per_seg < lay->n_code ? c0 + lay->code_per_seg : lay->n_code;
  uint64_t i, k = 0;
  uint32_t pos = 0, sizes[ORC_MAX_SEG + 1];
  uint8_t pipes[ORC_MAX_SEG + 1];
  uint8_t *seg = (uint8_t *)malloc((size_t)(lay->code_per_seg + 1) * ORC_CHUNK);
  for (i = c0; i <= c1; i++, k++) { /* code chunks c0..c1-1, then the meta chunk */
    uint64_t idx = i < c1 ? orc_code_chunk_index(lay, i) : orc_meta_chunk_index(lay, s);
    uint64_t e = get64(j->stream + ORC_HEADER + 8 * idx);
    uint32_t sz = (uint32_t)(e & 0xFFFFu);
    memcpy(seg + pos, j->stream + lay->data_base + ENTRY_OFFSET(e), sz);
    sizes[k] = sz;
    pipes[k] = (uint8_t)(e >> 60);
    pos += sz;
  }
  j->seg_status[s] = decode_segment_in(
      j->d, lay, s, seg, sizes, pipes, j->vectors ? j->vectors + s * vm * j->d->head_dim : NULL,
      j->vals ? j->vals + s * vm * j->d->head_dim : NULL);
  free(seg);
}

int orc_decompress(const uint8_t *stream, uint64_t stream_bytes,
                   const orc_desc *expect, uint16_t *vectors) {
  return orc_decompress_mt(stream, stream_bytes, expect, vectors, 1);
}

static int decompress_impl(const uint8_t *stream, uint64_t stream_bytes,
                           const orc_desc *expect, uint16_t *vectors, double *vals,
                           int n_threads);

int orc_decompress_mt(const uint8_t *stream, uint64_t stream_bytes,
                      const orc_desc *expect, uint16_t *vectors, int n_threads) {
  return decompress_impl(stream, stream_bytes, expect, vectors, NULL, n_threads);
}

int orc_decode_values_mt(const uint8_t *stream, uint64_t stream_bytes,
                         const orc_desc *expect, double *vals, int n_threads) {
  return decompress_impl(stream, stream_bytes, expect, NULL, vals, n_threads);
}

static int decompress_impl(const uint8_t *stream, uint64_t stream_bytes,
                           const orc_desc *expect, uint16_t *vectors, double *vals,
                           int n_threads) {
  orc_layout lay;
  uint64_t s, T = 0, expect_off = 0, total;
  int *seg_status;
  dec_job job;
  int st = orc_layout_of(expect, &lay), r;
  if (st != ORC_OK) return st;
  if (stream_bytes < ORC_HEADER) return ORC_ERR_CORRUPT;
  for (r = 0; r < expect->n_requests; r++) T += expect->token_lens[r];
  if (get32(stream) != ORC_MAGIC || get16(stream + 4) != 1 ||
      get16(stream + 6) != ORC_HEADER || stream[8] != expect->bits ||
      stream[9] != orc_meta_shift(expect->head_dim) ||
      get32(stream + 12) != (uint32_t)expect->group ||
      get32(stream + 16) != (uint32_t)expect->layers || get32(stream + 20) != 2 ||
      get32(stream + 24) != (uint32_t)expect->kv_heads ||
      get32(stream + 28) != (uint32_t)expect->head_dim || get64(stream + 32) != T ||
      get64(stream + 40) != expect->sign_seed ||
      get32(stream + 48) != (uint32_t)expect->n_requests ||
      get32(stream + 52) != lay.n_chunks)
    return ORC_ERR_CORRUPT;
  total = get64(stream + 56);
  if (total > stream_bytes || total < lay.data_base) return ORC_ERR_CORRUPT;
  for (r = 0; r < expect->n_requests; r++)
    if (get32(stream + ORC_HEADER + 8 * lay.n_chunks + 4 * r) !=
        expect->token_lens[r])
      return ORC_ERR_CORRUPT;
  /* the table: offsets are the prefix sum of padded sizes, in index order */
  for (s = 0; s < lay.n_chunks; s++) {
    uint64_t e = get64(stream + ORC_HEADER + 8 * s);
    uint32_t sz = (uint32_t)(e & 0xFFFFu);
    uint64_t off = ENTRY_OFFSET(e);
    if (off != expect_off || sz > ORC_CHUNK || lay.data_base + off + round16(sz) > total)
      return ORC_ERR_CORRUPT;
    expect_off = off + round16(sz);
  }
  /* header flags: bit 0 must be set if a code chunk uses zero-byte
     elimination; bits 1..3 name the quantizer and the sign diagonals, which
     must be the expected ones; the other bits are zero */
  if ((stream[11] & 0xF0u) || ((stream[11] >> 1) & 3u) != (unsigned)expect->quant ||
      ((stream[11] >> 3) & 1u) != (unsigned)expect->signs)
    return ORC_ERR_CORRUPT;
  for (s = 0; s < lay.n_code && !(stream[11] & 1u); s++) {
    uint64_t nv = lay.V - s * lay.vec_per_code;
    if (nv > lay.vec_per_code) nv = lay.vec_per_code;
    if ((get64(stream + ORC_HEADER + 8 * orc_code_chunk_index(&lay, s)) & 0xFFFFu) !=
        nv * lay.code_bytes)
      return ORC_ERR_CORRUPT;
  }
  seg_status = (int *)malloc((size_t)(lay.n_seg ? lay.n_seg : 1) * sizeof(int));
  job.d = expect;
  job.lay = &lay;
  job.stream = stream;
  job.vectors = vectors;
  job.vals = vals;
  job.seg_status = seg_status;
  for_each_segment(lay.n_seg, n_threads, &job, dec_one_segment);
  /* the first error in segment order wins */
  for (s = 0; s < lay.n_seg; s++)
    if (seg_status[s] != ORC_OK && st == ORC_OK) st = seg_status[s];
  free(seg_status);
  if (st == ORC_OK && lay.data_base + expect_off != total) st = ORC_ERR_CORRUPT;
  return st;
}

/* ========================================================================== */
/* Attention over a compressed cache (reading R18; the ZipFusion abstract on  */
/* the first page: decode attention that consumes the compressed KV cache).   */
/* One decode step of grouped-query attention for every layer and request:   */
/* query head j of layer l and request r reads kv head h = j / q_per_kv;     */
/*   s_t = scale * (q . k^_t),  p = softmax_t(s),  o = sum_t p_t v^_t,       */
/* t over the request's tokens, k^ and v^ the stream's decoded key and value */
/* vectors without the bf16 rounding (orc_dequantize_vector_f64), all in     */
/* double. q: bf16 [layers][n_requests][kv_heads * q_per_kv][d]; out: double  */
/* of the same shape (zeros for a request without tokens).                   */
/* ========================================================================== */
int orc_attend(const uint8_t *stream, uint64_t stream_bytes, const orc_desc *expect,
               const uint16_t *q, int q_per_kv, double scale, double *out, int n_threads) {
  orc_layout lay;
  double *vals, *s = NULL;
  uint64_t T = 0, cum = 0, t;
  int st = orc_layout_of(expect, &lay), l, r, j, c, H, d, Hq;
  if (st != ORC_OK) return st;
  if (q_per_kv < 1) return ORC_ERR_INVALID_ARG;
  d = expect->head_dim;
  H = expect->kv_heads;
  Hq = H * q_per_kv;
  for (r = 0; r < expect->n_requests; r++) T += expect->token_lens[r];
  vals = (double *)malloc((size_t)(lay.V ? lay.V : 1) * (size_t)d * sizeof(double));
  st = orc_decode_values_mt(stream, stream_bytes, expect, vals, n_threads);
  if (st == ORC_OK) s = (double *)malloc((size_t)(T ? T : 1) * sizeof(double));
  for (r = 0, cum = 0; st == ORC_OK && r < expect->n_requests; cum += expect->token_lens[r], r++) {
    const uint64_t n = expect->token_lens[r];
    for (l = 0; l < expect->layers; l++) {
      for (j = 0; j < Hq; j++) {
        const uint64_t qi = (((uint64_t)l * expect->n_requests + r) * Hq + j) * d;
        const int h = j / q_per_kv;
        const double *K = vals + ((((uint64_t)l * 2 + 0) * H + h) * T + cum) * d;
        const double *Vv = vals + ((((uint64_t)l * 2 + 1) * H + h) * T + cum) * d;
        double m = -INFINITY, den = 0.0;
        for (c = 0; c < d; c++) out[qi + c] = 0.0;
        if (n == 0) continue;
        for (t = 0; t < n; t++) {
          double acc = 0.0;
          for (c = 0; c < d; c++) acc += (double)orc_bf16_to_f32(q[qi + c]) * K[t * d + c];
          s[t] = scale * acc;
          if (s[t] > m) m = s[t];
        }
        for (t = 0; t < n; t++) {
          const double p = exp(s[t] - m);
          den += p;
          for (c = 0; c < d; c++) out[qi + c] += p * Vv[t * d + c];
        }
        for (c = 0; c < d; c++) out[qi + c] /= den;
      }
    }
  }
  free(s);
  free(vals);
  return st;
}

/* ========================================================================== */
/* Logical vector order [layer][kv][head][request][token]; requests are       */
/* concatenated along tokens. Dense input: one request of `tokens` tokens.   */
/* Strides are in elements; head_dim is contiguous.                           */
/* ========================================================================== */
void orc_gather_dense(const uint16_t *base, int layers, int kv_heads,
                      int64_t tokens, int d, int64_t s_layer, int64_t s_kv,
                      int64_t s_head, int64_t s_token, uint64_t v_begin,
                      uint64_t v_end, uint16_t *out) {
  uint64_t v;
  (void)layers;
  for (v = v_begin; v < v_end; v++) {
    int64_t t = (int64_t)(v % (uint64_t)tokens);
    uint64_t lkh = v / (uint64_t)tokens;
    int64_t h = (int64_t)(lkh % (uint64_t)kv_heads);
    int64_t kv = (int64_t)((lkh / (uint64_t)kv_heads) % 2u);
    int64_t l = (int64_t)(lkh / (uint64_t)kv_heads / 2u);
    const uint16_t *src = base + l * s_layer + kv * s_kv + h * s_head + t * s_token;
    memcpy(out + (v - v_begin) * (uint64_t)d, src, (size_t)d * 2u);
  }
}

void orc_gather_paged(const uint16_t *pool, int layers, int kv_heads, int d,
                      int64_t s_layer, int64_t s_page, int64_t s_kv,
                      int64_t s_head, int64_t s_slot, int page_tokens,
                      int n_requests, const uint32_t *seq_lens,
                      const int32_t *page_table, int64_t pt_stride,
                      uint64_t v_begin, uint64_t v_end, uint16_t *out) {
  uint64_t v, T = 0;
  int r;
  (void)layers;
  for (r = 0; r < n_requests; r++) T += seq_lens[r];
  for (v = v_begin; v < v_end; v++) {
    uint64_t u = v % T, lkh = v / T;
    int64_t h = (int64_t)(lkh % (uint64_t)kv_heads);
    int64_t kv = (int64_t)((lkh / (uint64_t)kv_heads) % 2u);
    int64_t l = (int64_t)(lkh / (uint64_t)kv_heads / 2u);
    int64_t t, page;
    const uint16_t *src;
    r = 0;
    while (u >= seq_lens[r]) {
      u -= seq_lens[r];
      r++;
    }
    t = (int64_t)u;
    page = page_table[(int64_t)r * pt_stride + t / page_tokens];
    src = pool + l * s_layer + page * s_page + kv * s_kv + h * s_head +
          (t % page_tokens) * s_slot;
    memcpy(out + (v - v_begin) * (uint64_t)d, src, (size_t)d * 2u);
  }
}
