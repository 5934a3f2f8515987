/*
 * Exhaustive pins of the oracle's scalar conversions against independent
 * implementations: x86 F16C hardware conversion (VCVTPS2PH with an explicit
 * rounding mode) for fp32 -> fp16 round-down / round-up.
 * Test code only; linked with the oracle by tests/test_oracle_scalar.py.
 */
#include <immintrin.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#include "../../oracle/kvc_oracle.h"

static uint16_t f16c(float x, int toward_neg) {
  __m128 v = _mm_set_ss(x);
  __m128i h = toward_neg ? _mm_cvtps_ph(v, _MM_FROUND_TO_NEG_INF | _MM_FROUND_NO_EXC)
                         : _mm_cvtps_ph(v, _MM_FROUND_TO_POS_INF | _MM_FROUND_NO_EXC);
  return (uint16_t)_mm_extract_epi16(h, 0);
}

/* Returns the number of non-NaN fp32 bit patterns in [lo, hi] where the
 * oracle and F16C disagree; the first mismatch goes to *first. */
uint64_t pin_f16_directed(uint32_t lo, uint32_t hi, int toward_neg, uint32_t *first) {
  uint64_t bad = 0;
  uint64_t u;
  *first = 0;
  for (u = lo; u <= hi; u++) {
    uint32_t b = (uint32_t)u;
    float x;
    uint16_t a, r;
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) continue; /* NaN payloads differ by design */
    memcpy(&x, &b, 4);
    a = toward_neg ? orc_f32_to_f16_rd(x) : orc_f32_to_f16_ru(x);
    r = f16c(x, toward_neg);
    if (a != r) {
      if (!bad) *first = b;
      bad++;
    }
  }
  return bad;
}

typedef struct {
  uint32_t lo, hi;
  int toward_neg, stride;
  uint64_t bad;
  uint32_t first;
} pin_job;

static void *pin_worker(void *arg) {
  pin_job *j = (pin_job *)arg;
  uint64_t u;
  for (u = j->lo; u <= j->hi; u += (uint64_t)j->stride) {
    uint32_t b = (uint32_t)u, f;
    uint64_t n = pin_f16_directed(b, b, j->toward_neg, &f);
    if (n && !j->bad) j->first = f;
    j->bad += n;
  }
  return 0;
}

/* Same as pin_f16_directed, split over `threads` threads; patterns are taken
 * every `stride` steps (stride 1 = every pattern). */
uint64_t pin_f16_directed_mt(uint32_t lo, uint32_t hi, int toward_neg, int threads,
                             int stride, uint32_t *first) {
  pthread_t tid[64];
  pin_job job[64];
  uint64_t span = ((uint64_t)hi - lo + 1), per, bad = 0;
  int t;
  if (threads > 64) threads = 64;
  per = (span + (uint64_t)threads - 1) / (uint64_t)threads;
  per = (per + (uint64_t)stride - 1) / (uint64_t)stride * (uint64_t)stride;
  *first = 0;
  for (t = 0; t < threads; t++) {
    uint64_t a = lo + (uint64_t)t * per, b = a + per - 1;
    if (a > hi) { threads = t; break; }
    if (b > hi) b = hi;
    job[t].lo = (uint32_t)a; job[t].hi = (uint32_t)b; job[t].toward_neg = toward_neg;
    job[t].stride = stride; job[t].bad = 0; job[t].first = 0;
    pthread_create(&tid[t], 0, pin_worker, &job[t]);
  }
  for (t = 0; t < threads; t++) {
    pthread_join(tid[t], 0);
    if (job[t].bad && !bad) *first = job[t].first;
    bad += job[t].bad;
  }
  return bad;
}

/* Array maps used by the Python pins. */
void map_f32_to_bf16(const float *x, uint64_t n, uint16_t *out) {
  uint64_t i;
  for (i = 0; i < n; i++) out[i] = orc_f32_to_bf16_rne(x[i]);
}
void map_f16_to_f32(const uint16_t *h, uint64_t n, float *out) {
  uint64_t i;
  for (i = 0; i < n; i++) out[i] = orc_f16_to_f32(h[i]);
}
