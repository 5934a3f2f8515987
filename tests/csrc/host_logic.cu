// Host-side exports of the library's host/device helpers (compiled host-only
// by the tests): fast division, the 32x32 bit transpose, sign masks.
#include <cstring>

#include "../../kv_cache_compression_04_b200/csrc/kvc_device.cuh"

extern "C" {
uint32_t hl_fdiv(uint32_t d, uint32_t n) { return kvc::fdiv(kvc::make_fastdiv(d), n); }
void hl_transpose32(const uint32_t *in, uint32_t *out) {
  uint32_t a[32];
  for (int i = 0; i < 32; ++i) a[i] = in[i];
  kvc::transpose32(a);
  for (int i = 0; i < 32; ++i) out[i] = a[i];
}
// The two-thread split of the transpose: each half runs the byte-permute
// exchange against the other half's rows, then the in-half levels.
void hl_transpose32_split(const uint32_t *in, uint32_t *out) {
  uint32_t lo[16], hi[16];
  for (int i = 0; i < 16; ++i) lo[i] = in[i], hi[i] = in[16 + i];
  uint32_t nlo[16], nhi[16];
  for (int i = 0; i < 16; ++i) {
    nlo[i] = kvc::transpose_split_stage16(lo[i], hi[i], 0);
    nhi[i] = kvc::transpose_split_stage16(hi[i], lo[i], 1);
  }
  kvc::transpose_split_rest(nlo);
  kvc::transpose_split_rest(nhi);
  for (int i = 0; i < 16; ++i) out[i] = nlo[i], out[16 + i] = nhi[i];
}
void hl_sign_masks(uint64_t seed, int d, uint32_t *out) { kvc::sign_masks(seed, d, out); }
// Mismatches of the library's division by the quantizers' constant q (its
// host compilation) against the correctly rounded quotient over the fp32
// patterns start, start + stride, ... below 0x7F800000 (every finite x >= 0
// with stride 1). The reference divides in long double (64-bit significand)
// and rounds once more to fp32: exact quotients are exact there, and an
// inexact x / q (q odd) has a periodic binary expansion of period at most 8,
// so its 40 extra bits are never exactly a half-way pattern and the second
// rounding cannot move the result.
uint64_t hl_div_const_mismatches(int q, uint32_t start, uint32_t stride) {
  float (*f)(float) = nullptr;
  switch (q) {
    case 3: f = kvc::div_const<3>; break;
    case 7: f = kvc::div_const<7>; break;
    case 15: f = kvc::div_const<15>; break;
    case 127: f = kvc::div_const<127>; break;
    case 255: f = kvc::div_const<255>; break;
    default: return ~uint64_t(0);
  }
  uint64_t bad = 0;
  for (uint64_t u = start; u < 0x7F800000ull; u += stride) {
    float x;
    const uint32_t b = uint32_t(u);
    memcpy(&x, &b, 4);
    const float ref = float((long double)x / (long double)q);
    const float got = f(x);
    uint32_t rb, gb;
    memcpy(&rb, &ref, 4);
    memcpy(&gb, &got, 4);
    bad += rb != gb;
  }
  return bad;
}
// Mismatches of the library's nonzero-byte mask against a byte-by-byte
// reference over words [start, start + count).
uint64_t hl_nz_nibble_mismatches(uint64_t start, uint64_t count) {
  uint64_t bad = 0;
  for (uint64_t i = 0; i < count; ++i) {
    const uint32_t x = uint32_t(start + i);
    uint32_t ref = 0;
    for (int b = 0; b < 4; ++b) ref |= (((x >> (8 * b)) & 0xFFu) != 0 ? 1u : 0u) << b;
    bad += kvc::nz_nibble(x) != ref;
  }
  return bad;
}
}
