// One decode step of grouped-query attention over a compressed KV cache,
// read straight from the stream: no decoded key or value reaches HBM. The
// design follows the ZipFusion abstract (first page: decode attention that
// consumes the compressed cache) and reading R18 (the keys and values are the
// stream's decoded vectors without the bf16 rounding).
//
// Each decoded vector is x = D H y / d, y the dequantized transformed values
// (the decoder's fp32 y = zf + q sf), D the sign diagonal, H the symmetric
// Walsh-Hadamard matrix. Hence q . x = (H D q) . y / d and
// sum_t p_t x_t = D H (sum_t p_t y_t) / d: a CTA turns each query into
// qt = (scale / d) H D q once, scores every token in the transformed domain,
// accumulates the softmax-weighted transformed values, and one inverse
// transform per query head finishes the output. Per CTA: one (layer,
// request, kv head) and a range of kAttTok tokens (split-K); a second kernel
// combines the splits (running maxima and sums) and inverts the transform.
#pragma once

#include "kvc_decode.cuh"

namespace kvc {

constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttTok = 256;   // tokens per CTA
constexpr int kAttMaxG = 8;    // query heads per kv head



// Header checks shared by the attention kernels: the stream describes this
// cache with the stated bits and group, and stores every code chunk raw (the
// code region is then the plain array of per-vector codes). Flags: bit 0
// (eliminated code chunks) clear; the min/max or absmax quantizer (both
// decode as zero + code * scale) or, as the caller states, FP4 (e2m1(code) *
// s1 * s2); either sign mode (bit 3: per-vector diagonals).
template <int D>
__device__ __forceinline__ bool attn_header_ok(const AttnArgs &a, uint64_t &base, uint32_t &n_code,
                                               uint64_t &seed) {
  constexpr uint32_t kLog2D = D == 64 ? 6 : D == 128 ? 7 : 8;
  const uint8_t *h = a.in;
  if (a.in_bytes < kHeader) return false;
  const uint32_t n_req = ld_u32(h + 48), n_chunks = ld_u32(h + 52);
  const uint64_t cb = uint64_t(D) * a.bits / 8, mbv = uint64_t(D / a.group) * 4;
  const uint64_t nc = (uint64_t(a.V) * cb + kChunk - 1) / kChunk;
  const uint64_t nm = (uint64_t(a.V) * mbv + kChunk - 1) / kChunk;
  base = round16(kHeader + 8ull * n_chunks + 4ull * n_req);
  n_code = uint32_t(nc);
  seed = ld_u64(h + 40);
  return ld_u32(h) == kMagic && (ld_u32(h + 4) & 0xFFFFu) == 1 &&
         (ld_u32(h + 4) >> 16) == kHeader && h[8] == a.bits && h[9] == kLog2D / 2 &&
         (h[11] & 0xF1u) == 0 && ((h[11] >> 1) & 3u) <= 2 &&
         (((h[11] >> 1) & 3u) == 2) == (a.fp4 != 0) && ld_u32(h + 12) == a.group &&
         ld_u32(h + 16) == a.layers &&
         ld_u32(h + 20) == 2 && ld_u32(h + 24) == a.kv_heads && ld_u32(h + 28) == D &&
         ld_u64(h + 32) == a.tokens && n_req == a.n_req && n_chunks == nc + nm &&
         ld_u64(h + 56) <= a.in_bytes && base + uint64_t(a.V) * cb <= ld_u64(h + 56);
}

struct AttnSmem {
  alignas(16) float qt[kAttMaxG][128];            // transformed queries
  float s[kAttTok][kAttMaxG];                     // scores, then weights
  float o[kAttWarps][kAttMaxG][128];              // per-warp partial outputs
  float wmax[kAttWarps][kAttMaxG];
  float m[kAttMaxG], l[kAttMaxG];
  uint32_t ok;
  uint64_t base;
  const uint8_t *mptr[2][2];  // keys, values: meta chunks of the CTA's range
  uint32_t ms0[2];            // index of the first of them
  alignas(16) uint32_t mask[64];
};

// Walsh-Hadamard butterfly of a 128-vector held by a warp, lane j holding
// channels j, j + 32, j + 64, j + 96: strides 1..16 cross lanes (shuffles),
// 32 and 64 stay in registers. Each stage is the pair (a + b, a - b).
__device__ __forceinline__ void warp_fwht128(float (&y)[4], uint32_t lane) {
#pragma unroll
  for (uint32_t s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, y[c], s);
      y[c] = (lane & s) ? __fsub_rn(o, y[c]) : __fadd_rn(y[c], o);
    }
  }
#pragma unroll
  for (int s = 1; s < 4; s <<= 1) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if ((c & s) == 0) {
        const float u = y[c], v = y[c + s];
        y[c] = __fadd_rn(u, v);
        y[c + s] = __fsub_rn(u, v);
      }
    }
  }
}

// Partial record of one CTA and query head: m, l, two pad words, o[D]
// (16-byte aligned, so the combining warps read it in 128-byte lines).
constexpr int kAttRec = 128 + 4;

// QPK: query heads per kv head rounded up to 1, 2, 4 or 8 (a.qpk of them
// are real; the others score a zero query and are not written); G: the
// quantization group.
// kFp4: the stream's FP4 quantizer (reading R22).
template <int D, int BITS, int G, int QPK, bool kFp4 = false>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(const __grid_constant__ AttnArgs a) {
  using C = Cfg<D, BITS, G>;
  static_assert(D == 128, "attention kernel: head_dim 128");
  static_assert(QPK >= 1 && QPK <= kAttMaxG, "query heads per kv head");
  __shared__ AttnSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t qpk = a.qpk;
  const uint32_t H = a.kv_heads;
  const uint32_t unit = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const uint32_t h = unit % H, lr = unit / H, r = lr % a.n_req, l = lr / a.n_req;
  const uint32_t len = a.cum[r + 1] - a.cum[r];
  const uint32_t t_a = split * kAttTok, t_b = min(len, t_a + kAttTok);
  float *part = a.part + (uint64_t(blockIdx.x) * qpk) * kAttRec;
  const uint8_t *in = a.in, *table = in + kHeader;
  const uint32_t T = uint32_t(a.tokens);
  if (tid == 0) {
    uint64_t base, seed;
    uint32_t n_code;
    bool ok = attn_header_ok<D>(a, base, n_code, seed);
    // The table entries this CTA relies on: its code chunks raw and in place
    // (chunk c at c * 16 KB), its meta chunks raw inside the stream or
    // eliminated (then expanded, and checked, by the meta expansion kernel).
    // A range of kAttTok vectors spans at most two chunks of either kind.
    for (uint32_t x = 0; ok && x < 2 && t_a < t_b; ++x) {
      const uint64_t v0 = uint64_t((l * 2 + x) * H + h) * T + a.cum[r];
      const uint64_t va = v0 + t_a, vb = v0 + t_b, code_bytes = uint64_t(a.V) * C::CB;
      for (uint64_t c = va * C::CB / kChunk; c <= (vb * C::CB - 1) / kChunk; ++c) {
        const uint64_t e = ld_u64(table + 8 * c), rest = code_bytes - c * kChunk;
        ok = ok && entry_size(e) == (rest < kChunk ? rest : uint64_t(kChunk)) &&
             entry_pipe(e) == 0 && entry_offset(e) == c * kChunk;
      }
      const uint32_t s0 = uint32_t(va / C::VM), s1 = uint32_t((vb - 1) / C::VM);
      sm.ms0[x] = s0;
      for (uint32_t s = s0; s <= s1; ++s) {
        const uint64_t e = ld_u64(table + 8 * (uint64_t(n_code) + s));
        const uint32_t mlen = min(uint32_t(C::VM), a.V - s * C::VM) * C::MB;
        const bool raw = entry_size(e) == mlen;
        ok = ok && (!raw || (entry_pipe(e) == 0 &&
                             base + entry_offset(e) + mlen <= ld_u64(in + 56)));
        sm.mptr[x][s - s0] = raw ? in + base + entry_offset(e) : a.ws_meta + uint64_t(s) * kChunk;
      }
    }
    sm.ok = ok;
    sm.base = base;
    if (!ok) {
      set_status(a.status, KVC_ERR_CORRUPT);
    } else if (in[11] & 8u) {  // the keys' own diagonal: index (l, 0, h)
      uint32_t S[D / 32];
      vec_sign_words<D>(seed, (l * 2 + 0) * H + h, S);
      for (int k = 0; k < D / 2; ++k) sm.mask[k] = pair_mask<D>(S, 2 * k);
    } else {
      sign_masks(seed, D, sm.mask);
    }
  }
  __syncthreads();
  if (!sm.ok) return;
  if (t_a >= t_b) {  // nothing in this split: an empty partial
    for (uint32_t g = tid; g < qpk; g += kAttThreads) {
      part[g * kAttRec] = -INFINITY;
      part[g * kAttRec + 1] = 0.f;
    }
    return;
  }
  const uint64_t base = sm.base;

  // qt_g = (scale / d) H D q_g, one warp per query head
  for (uint32_t g = warp; g < uint32_t(QPK); g += kAttWarps) {
    const uint16_t *qv = a.q + ((uint64_t(l) * a.n_req + r) * H * qpk + h * qpk + g) * D;
    float y[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t ch = lane + 32 * c;
      const uint32_t sgn = (sm.mask[ch >> 1] >> ((ch & 1) ? 31 : 15)) & 1u;
      y[c] = 0.f;
      if (g < qpk) y[c] = __uint_as_float((uint32_t(qv[ch]) << 16) ^ (sgn << 31));
    }
    warp_fwht128(y, lane);
    const float f = a.scale / float(D);
#pragma unroll
    for (int c = 0; c < 4; ++c) sm.qt[g][lane + 32 * c] = y[c] * f;
  }
  __syncthreads();

  // meta bytes of vector v (x: 0 key, 1 value): a raw meta chunk in place,
  // an eliminated one as the meta expansion kernel left it in the workspace
  auto meta_of = [&](uint32_t v, int x) -> const uint8_t * {
    const uint32_t s = v / C::VM;
    return sm.mptr[x][s - sm.ms0[x]] + uint64_t(v - s * C::VM) * C::MB;
  };
  const uint32_t kv0 = ((l * 2 + 0) * H + h) * T + a.cum[r];  // first key vector
  const uint32_t vv0 = ((l * 2 + 1) * H + h) * T + a.cum[r];  // first value vector
  constexpr int per = 32 / BITS;                               // codes per word
  constexpr uint32_t qmask = (1u << BITS) - 1;

  // ---- scores: lane = token
  const uint32_t qt_s = uint32_t(__cvta_generic_to_shared(&sm.qt[0][0]));
  float mx[QPK];
#pragma unroll
  for (int g = 0; g < QPK; ++g) mx[g] = -INFINITY;
#pragma unroll 1
  for (uint32_t t = t_a + warp * 32 + lane; t < t_b; t += kAttWarps * 32) {
    const uint32_t v = kv0 + t;
    const uint4 *cw = reinterpret_cast<const uint4 *>(in + base + uint64_t(v) * C::CB);
    const uint8_t *mp = meta_of(v, 0);
    float acc[QPK];
#pragma unroll
    for (int g = 0; g < QPK; ++g) acc[g] = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < C::CW / 4; ++q4) {
      const uint4 w4 = cw[q4];
      const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c0 = (q4 * 4 + e) * per;               // first channel of this word
        const uint32_t m = reinterpret_cast<const uint32_t *>(mp)[c0 / G];
        const float sf = __half2float(__ushort_as_half(uint16_t(m))) * float(1 << C::K);
        const float zf = __half2float(__ushort_as_half(uint16_t(m >> 16))) * float(1 << C::K);
        // FP4: the word's channels lie in one half-group (8 of >= 16)
        const float S = kFp4 ? e4m3_value((m >> (16 + 8 * ((c0 % G) / (G / 2)))) & 0xFFu) * sf : 0.f;
#pragma unroll
        for (int k = 0; k < per; k += 4) {
          float y[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t code = (ws[e] >> ((k + i) * BITS)) & qmask;
            y[i] = kFp4 ? e2m1_value(code) * S : fmaf(float(code), sf, zf);
          }
#pragma unroll
          for (int g = 0; g < QPK; ++g) {
            // read per token (a volatile load): kept in registers across
            // tokens, QPK * 128 query values would crowd out the codes
            const uint4 qb = lds128(qt_s + uint32_t((g * 128 + c0 + k) * 4));
            acc[g] = fmaf(__uint_as_float(qb.x), y[0], acc[g]);
            acc[g] = fmaf(__uint_as_float(qb.y), y[1], acc[g]);
            acc[g] = fmaf(__uint_as_float(qb.z), y[2], acc[g]);
            acc[g] = fmaf(__uint_as_float(qb.w), y[3], acc[g]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < QPK; ++g) {
      sm.s[t - t_a][g] = acc[g];
      mx[g] = fmaxf(mx[g], acc[g]);
    }
  }
#pragma unroll
  for (int g = 0; g < QPK; ++g) {
    float x = mx[g];
#pragma unroll
    for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    if (lane == 0) sm.wmax[warp][g] = x;
  }
  __syncthreads();
  if (tid < QPK) {
    float x = sm.wmax[0][tid];
    for (int w = 1; w < kAttWarps; ++w) x = fmaxf(x, sm.wmax[w][tid]);
    sm.m[tid] = x;
  }
  __syncthreads();
  // weights p = exp(s - m) in place, and their sum per query head
  const uint32_t n = t_b - t_a;
  for (uint32_t i = tid; i < n * QPK; i += kAttThreads) {
    const uint32_t t = i / QPK, g = i - t * QPK;
    sm.s[t][g] = expf(sm.s[t][g] - sm.m[g]);
  }
  __syncthreads();
  if (tid < QPK) {
    float x = 0.f;
    for (uint32_t t = 0; t < n; ++t) x += sm.s[t][tid];
    sm.l[tid] = x;
  }

  // ---- values: lane = (token of the step, 8 consecutive channels, which
  // lie in one group and one code word)
  constexpr int CPL = BITS == 8 ? 4 : 8;  // channels per lane (one code word at most)
  constexpr int LPT = D / CPL;        // lanes per token
  constexpr int TPS = 32 / LPT;       // tokens per step
  const int wi = lane % LPT, tp = lane / LPT;
  float o[QPK][CPL];
#pragma unroll
  for (int g = 0; g < QPK; ++g)
#pragma unroll
    for (int k = 0; k < CPL; ++k) o[g][k] = 0.f;
#pragma unroll 1
  for (uint32_t t0 = t_a + warp * TPS; t0 < t_b; t0 += kAttWarps * TPS) {
    const uint32_t t = t0 + tp;
    if (t < t_b) {
      const uint32_t v = vv0 + t;
      const uint32_t word = reinterpret_cast<const uint32_t *>(
          in + base + uint64_t(v) * C::CB)[(wi * CPL * BITS) / 32];
      const uint32_t bits = word >> ((wi * CPL * BITS) % 32);
      const uint32_t m = reinterpret_cast<const uint32_t *>(meta_of(v, 1))[(wi * CPL) / G];
      const float sf = __half2float(__ushort_as_half(uint16_t(m))) * float(1 << C::K);
      const float zf = __half2float(__ushort_as_half(uint16_t(m >> 16))) * float(1 << C::K);
      const float S =
          kFp4 ? e4m3_value((m >> (16 + 8 * (((wi * CPL) % G) / (G / 2)))) & 0xFFu) * sf : 0.f;
      float p[QPK];
#pragma unroll
      for (int g = 0; g < QPK; ++g) p[g] = sm.s[t - t_a][g];
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const uint32_t code = (bits >> (k * BITS)) & qmask;
        const float y = kFp4 ? e2m1_value(code) * S : fmaf(float(code), sf, zf);
#pragma unroll
        for (int g = 0; g < QPK; ++g) o[g][k] = fmaf(p[g], y, o[g][k]);
      }
    }
  }
  // tokens of the same step share channels: sum across them, then warps
#pragma unroll
  for (int g = 0; g < QPK; ++g)
#pragma unroll
    for (int k = 0; k < CPL; ++k)
#pragma unroll
      for (int x = LPT; x < 32; x <<= 1) o[g][k] += __shfl_xor_sync(0xFFFFFFFFu, o[g][k], x);
  if (tp == 0) {
#pragma unroll
    for (int g = 0; g < QPK; ++g)
#pragma unroll
      for (int k = 0; k < CPL; ++k) sm.o[warp][g][wi * CPL + k] = o[g][k];
  }
  __syncthreads();
  for (uint32_t i = tid; i < qpk * D; i += kAttThreads) {
    const uint32_t g = i / D, c = i - g * D;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) x += sm.o[w][g][c];
    part[g * kAttRec + 4 + c] = x;
  }
  if (tid < int(qpk)) {
    part[tid * kAttRec] = sm.m[tid];
    part[tid * kAttRec + 1] = sm.l[tid];
  }
}

// Combines the splits of each (layer, request, query head) and inverts the
// transform: o = sign * H (sum_k e^(m_k - M) o_k / sum_k e^(m_k - M) l_k) / d.
// One warp per output row; lane j holds channels j, j + 32, j + 64, j + 96,
// so the butterfly's strides 1..16 cross lanes (shuffles) and 32, 64 stay in
// registers.
constexpr int kCombWarps = 8;
template <int D>
__global__ void __launch_bounds__(kCombWarps * 32) attend_combine_kernel(const __grid_constant__ AttnArgs a) {
  static_assert(D == 128, "four channels per lane");
  grid_dependency_wait();  // the attention kernel's partials
  const uint32_t lane = threadIdx.x & 31, qpk = a.qpk, H = a.kv_heads;
  const uint32_t n_out = a.layers * a.n_req * H * qpk;
  const uint32_t i = blockIdx.x * kCombWarps + (threadIdx.x >> 5);
  if (i >= n_out) return;
  if (*reinterpret_cast<const volatile uint32_t *>(a.status) != 0) return;
  const uint32_t j = i % (H * qpk), lr = i / (H * qpk), r = lr % a.n_req, l = lr / a.n_req;
  const uint32_t h = j / qpk, g = j % qpk;
  const uint32_t unit = (l * a.n_req + r) * H + h;
  float *out = a.out + uint64_t(i) * D;
  float y[4] = {0.f, 0.f, 0.f, 0.f};
  if (a.cum[r + 1] == a.cum[r]) {  // no tokens: zeros
#pragma unroll
    for (int k = 0; k < 4; ++k) out[lane + 32 * k] = 0.f;
    return;
  }
  const float *p0 = a.part + (uint64_t(unit) * a.splits * qpk + g) * kAttRec;
  const uint64_t step = uint64_t(qpk) * kAttRec;
  float M = -INFINITY;
  for (uint32_t k = lane; k < a.splits; k += 32) M = fmaxf(M, p0[k * step]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
  float L = 0.f;
  for (uint32_t k = 0; k < a.splits; ++k) {
    const float *p = p0 + k * step;
    const float mk = p[0];
    if (mk == -INFINITY) continue;  // an empty split
    const float w = expf(mk - M);
    L = fmaf(w, p[1], L);
#pragma unroll
    for (int c = 0; c < 4; ++c) y[c] = fmaf(w, p[4 + lane + 32 * c], y[c]);
  }
  warp_fwht128(y, lane);
  // sign of channel c: bit c % 64 of the (c / 64 + 1)-th SplitMix64 output
  // of the diagonal (the global one, or the values' own: index (l, 1, h))
  uint64_t st = ld_u64(a.in + 40);
  if (a.in[11] & 8u) st += uint64_t((l * 2 + 1) * H + h) * 2u * 0x9E3779B97F4A7C15ull;
  const uint64_t w0 = splitmix64(st), w1 = splitmix64(st);
  const float f = 1.f / (L * float(D));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t ch = lane + 32 * c;
    const uint32_t sgn = uint32_t(((ch < 64 ? w0 : w1) >> (ch % 64)) & 1u);
    out[ch] = __uint_as_float(__float_as_uint(y[c] * f) ^ (sgn << 31));
  }
}

}  // namespace kvc
