// Attention over a compressed cache with the contractions on tensor cores
// (warp-level mma.sync m16n8k16, fp16 operands, fp32 accumulation), for the
// min/max and absmax quantizers at 2 and 4 bits. Same work and results as
// attend_kernel (kvc_attend.cuh): one CTA per (layer, request, kv head) and
// 256-token split, partial (m, l, o) records for the combining kernel.
//
// Each decoded transformed value is y = zf + q * sf (q the code). With
// qt = (scale / d) H D q (the transformed query):
//   score = sum_groups [ sf * (sum_c qt_c q_c) + zf * (sum_c qt_c) ]
//   sum_t p_t y_t = sum_groups [ sum_t (p_t sf_t) q_t + sum_t p_t zf_t ]
// so both passes contract the integer codes, exact in fp16, with an fp32
// operand split into fp16 hi + lo parts (after scaling by a power of two so
// that the largest magnitude is below 2^15): qt in the score pass, p * sf in
// the value pass. The fp32 accumulators then hold the products to about
// 2^-22 of the largest term. The per-group zero terms are a few FMAs per
// token on the CUDA cores.
//
// Fragments (PTX ISA, mma m16n8k16 .f16): lane = 4 * gq + tq;
//   A (16 x 16, row-major): a0 = A[gq][2tq, 2tq+1], a1 = A[gq+8][2tq, 2tq+1],
//                           a2 = A[gq][2tq+8, +9],  a3 = A[gq+8][2tq+8, +9];
//   B (16 x 8, column n):   b0 = B[2tq, 2tq+1][gq], b1 = B[2tq+8, +9][gq];
//   C (16 x 8):             c0 = C[gq][2tq], c1 = C[gq][2tq+1],
//                           c2 = C[gq+8][2tq], c3 = C[gq+8][2tq+1].
// The reduced dimension (channels in the score pass, tokens in the value
// pass) may be permuted freely as long as both operands agree; the mappings
// below pick, for every lane, slots it can fill from contiguous code bytes
// with one LOP3 per two codes (an fp16 pair 1024 + q, then minus 1024).
#pragma once

#include "kvc_attend.cuh"

namespace kvc {

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two codes (bits 0.. and 16.. of x, `mask` wide) -> fp16 pair of their values.
template <uint32_t kMask>
__device__ __forceinline__ uint32_t codes_f16x2(uint32_t x) {
  uint32_t t, d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(t) : "r"(x), "n"(kMask), "n"(0x64006400));
  asm("sub.f16x2 %0, %1, %2;" : "=r"(d) : "r"(t), "r"(0x64006400));
  return d;
}

// fp32 pair -> fp16 pair (round to nearest), lower element first.
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// The hi and lo fp16 parts of v (v = hi + lo + O(2^-22 |v|) below 2^15).
__device__ __forceinline__ void split_f16(float v, float &hi, float &lo) {
  hi = __half2float(__float2half_rn(v));
  lo = v - hi;
}

struct AttnMmaSmem {
  alignas(16) float qt[kAttMaxG][128];  // transformed queries
  float s[kAttTok][kAttMaxG];            // scores, then weights
  float o[kAttWarps][kAttMaxG][128];     // per-warp partial outputs
  float z[kAttWarps][kAttMaxG][4];       // per-warp sum_t p * zf per group
  float qs[kAttMaxG][4];                 // sum of qt over each group
  float wmax[kAttWarps][kAttMaxG];
  float m[kAttMaxG], l[kAttMaxG];
  float red[kAttWarps];
  float escale_q, escale_w;              // 2^eq, 2^ew
  uint32_t ok;
  uint64_t base;
  const uint8_t *mptr[2][2];
  uint32_t ms0[2];
  alignas(16) uint32_t mask[64];
};

// QPK: query heads per kv head rounded up to 4 or 8 (NT = QPK / 4 column
// tiles of 4 heads x {hi, lo}).
template <int BITS, int G, int QPK>
__global__ void __launch_bounds__(kAttThreads) attend_mma_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int D = 128;
  using C = Cfg<D, BITS, G>;
  static_assert(BITS == 2 || BITS == 4, "2- and 4-bit codes");
  static_assert(QPK == 4 || QPK == 8, "query-head tiles of 4");
  constexpr int NT = QPK / 4;
  constexpr int NG = D / G;
  __shared__ AttnMmaSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t qpk = a.qpk, H = a.kv_heads;
  const uint32_t unit = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const uint32_t h = unit % H, lr = unit / H, r = lr % a.n_req, l = lr / a.n_req;
  const uint32_t len = a.cum[r + 1] - a.cum[r];
  const uint32_t t_a = split * kAttTok, t_b = min(len, t_a + kAttTok);
  float *part = a.part + (uint64_t(blockIdx.x) * qpk) * kAttRec;
  const uint8_t *in = a.in, *table = in + kHeader;
  const uint32_t T = uint32_t(a.tokens);

  // ---- header, this CTA's chunk entries, sign masks (as attend_kernel)
  if (tid == 0) {
    uint64_t base, seed;
    uint32_t n_code;
    bool ok = attn_header_ok<D>(a, base, n_code, seed);
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
  if (t_a >= t_b) {
    for (uint32_t g = tid; g < qpk; g += kAttThreads) {
      part[g * kAttRec] = -INFINITY;
      part[g * kAttRec + 1] = 0.f;
    }
    return;
  }
  const uint64_t base = sm.base;
  const uint32_t n = t_b - t_a;
  auto meta_of = [&](uint32_t v, int x) -> const uint8_t * {
    const uint32_t s = v / C::VM;
    return sm.mptr[x][s - sm.ms0[x]] + uint64_t(v - s * C::VM) * C::MB;
  };
  const uint32_t kv0 = ((l * 2 + 0) * H + h) * T + a.cum[r] + t_a;  // key of token t_a
  const uint32_t vv0 = ((l * 2 + 1) * H + h) * T + a.cum[r] + t_a;  // value of token t_a
  const float kup = float(1 << C::K);  // meta is stored x 2^-K

  // ---- transformed queries (warp-cooperative butterfly), their group sums
  // and the largest magnitude (a power-of-two scale for the fp16 split)
  float qmax = 0.f;
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
    for (int c = 0; c < 4; ++c) {
      y[c] *= f;
      sm.qt[g][lane + 32 * c] = y[c];
      qmax = fmaxf(qmax, fabsf(y[c]));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xFFFFFFFFu, qmax, o));
  if (lane == 0) sm.red[warp] = qmax;
  __syncthreads();
  if (tid < QPK * NG) {
    const int g = tid / NG, gg = tid % NG;
    float x = 0.f;
    for (int c = 0; c < G; ++c) x += sm.qt[g][gg * G + c];
    sm.qs[g][gg] = x;
  }
  if (tid == 0) {
    float mx = fmaxf(fmaxf(sm.red[0], sm.red[1]), fmaxf(sm.red[2], sm.red[3]));
    int e = 0;
    frexpf(mx, &e);  // mx < 2^e
    sm.escale_q = mx > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
  }
  __syncthreads();

  // ---- score pass. Channel of k-slot k of k-block kb for the lane's tq:
  // 4-bit: word w = 4 (kb / 2) + (k % 8) / 2, nibble 2 (kb % 2) + k / 8 +
  // 4 (k % 2); 2-bit: word kb, code (2 ((k % 8) / 2) + k / 8) + 8 (k % 2).
  // Each k-block lies in one group (G >= 32); the lane loads its words.
  auto score_ch = [&](int kb, int k) -> int {
    const int j = (k % 8) / 2, hi8 = k / 8, sub = k % 2;
    if constexpr (BITS == 4) return 8 * (4 * (kb / 2) + j) + 2 * (kb % 2) + hi8 + 4 * sub;
    else return 16 * kb + (2 * j + hi8) + 8 * sub;
  };
  uint32_t qb[8][NT][2];  // B fragments: transformed queries, columns (head, hi / lo)
  {
    const float es = sm.escale_q;
#pragma unroll
    for (int kb = 0; kb < 8; ++kb)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int g = nt * 4 + (gq >> 1), hl = gq & 1;
        float v[4];
        const int ks[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float hi, lo;
          split_f16(sm.qt[g][score_ch(kb, ks[i])] * es, hi, lo);
          v[i] = hl ? lo : hi;
        }
        qb[kb][nt][0] = f16x2(v[0], v[1]);
        qb[kb][nt][1] = f16x2(v[2], v[3]);
      }
  }
  constexpr int kTiles = kAttTok / 16;
  float mx[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) mx[nt] = -INFINITY;
  const float inv_eq = 1.f / sm.escale_q;
#pragma unroll 1
  for (int tile = warp; tile < kTiles && uint32_t(tile) * 16 < n; tile += kAttWarps) {
    const uint32_t tA = uint32_t(tile) * 16 + gq, tB = tA + 8;  // CTA-relative tokens
    const bool okA = tA < n, okB = tB < n;
    // the lane's code words of both tokens
    constexpr int NW = BITS == 4 ? 4 : 8;
    uint32_t wA[NW], wB[NW];
    const uint32_t *rowA = reinterpret_cast<const uint32_t *>(in + base + uint64_t(kv0 + tA) * C::CB);
    const uint32_t *rowB = reinterpret_cast<const uint32_t *>(in + base + uint64_t(kv0 + tB) * C::CB);
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const int w = BITS == 4 ? 4 * i + tq : i;
      wA[i] = okA ? __ldg(rowA + w) : 0u;
      wB[i] = okB ? __ldg(rowB + w) : 0u;
    }
    float acc[NG][NT][4];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[gg][nt][i] = 0.f;
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      uint32_t af[4];
      if constexpr (BITS == 4) {
        const int s = (kb & 1) * 8;
        af[0] = codes_f16x2<0x000F000Fu>(wA[kb / 2] >> s);
        af[1] = codes_f16x2<0x000F000Fu>(wB[kb / 2] >> s);
        af[2] = codes_f16x2<0x000F000Fu>(wA[kb / 2] >> (s + 4));
        af[3] = codes_f16x2<0x000F000Fu>(wB[kb / 2] >> (s + 4));
      } else {
        af[0] = codes_f16x2<0x00030003u>(wA[kb] >> (4 * tq));
        af[1] = codes_f16x2<0x00030003u>(wB[kb] >> (4 * tq));
        af[2] = codes_f16x2<0x00030003u>(wA[kb] >> (4 * tq + 2));
        af[3] = codes_f16x2<0x00030003u>(wB[kb] >> (4 * tq + 2));
      }
      constexpr int kPerG = G / 16;  // k-blocks per group
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma16816(acc[kb / kPerG][nt], af, qb[kb][nt][0], qb[kb][nt][1]);
    }
    // scores of tokens tA, tB for heads nt * 4 + tq (columns 2tq: hi, 2tq + 1: lo)
    const uint32_t *mA = reinterpret_cast<const uint32_t *>(meta_of(kv0 + (okA ? tA : 0), 0));
    const uint32_t *mB = reinterpret_cast<const uint32_t *>(meta_of(kv0 + (okB ? tB : 0), 0));
    float sA[NT], sB[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sA[nt] = sB[nt] = 0.f;
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) {
      const uint32_t ma = mA[gg], mb = mB[gg];
      const float sfa = __half2float(__ushort_as_half(uint16_t(ma))) * kup;
      const float zfa = __half2float(__ushort_as_half(uint16_t(ma >> 16))) * kup;
      const float sfb = __half2float(__ushort_as_half(uint16_t(mb))) * kup;
      const float zfb = __half2float(__ushort_as_half(uint16_t(mb >> 16))) * kup;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float qsum = sm.qs[nt * 4 + tq][gg];
        sA[nt] = fmaf(sfa, (acc[gg][nt][0] + acc[gg][nt][1]) * inv_eq, fmaf(zfa, qsum, sA[nt]));
        sB[nt] = fmaf(sfb, (acc[gg][nt][2] + acc[gg][nt][3]) * inv_eq, fmaf(zfb, qsum, sB[nt]));
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 4 + tq;
      if (okA) {
        sm.s[tA][g] = sA[nt];
        mx[nt] = fmaxf(mx[nt], sA[nt]);
      }
      if (okB) {
        sm.s[tB][g] = sB[nt];
        mx[nt] = fmaxf(mx[nt], sB[nt]);
      }
    }
  }
  // per-head maxima: lanes of equal tq hold the same heads
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float x = mx[nt];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    if (gq == 0) sm.wmax[warp][nt * 4 + tq] = x;
  }
  __syncthreads();
  if (tid < QPK) {
    float x = sm.wmax[0][tid];
    for (int w = 1; w < kAttWarps; ++w) x = fmaxf(x, sm.wmax[w][tid]);
    sm.m[tid] = x;
  }
  __syncthreads();
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

  // ---- value pass. Tokens: lane tq holds k-slots 2tq, 2tq + 1, 2tq + 8,
  // 2tq + 9 = tokens 4tq .. 4tq + 3 of the 16-token step. Channels: the lane
  // (row gq) takes NB = G * BITS / 64 contiguous bytes of every group; byte
  // i of its run in group gg feeds M-tile(s) gg * G / 16 + i (4-bit: low
  // nibble row gq, high nibble row gq + 8) or + 2i, 2i + 1 (2-bit: bit pairs
  // 0, 1 and 2, 3 of the byte for the first, 4, 5 and 6, 7 for the second).
  constexpr int NB = G * BITS / 64;        // bytes per lane and group
  constexpr int NBW = (NB + 3) / 4;        // their words
  // Largest scale of the value rows: the power-of-two scale of p * sf.
  float vsf = 0.f;
  for (uint32_t t = tid; t < n; t += kAttThreads) {
    const uint32_t *mv = reinterpret_cast<const uint32_t *>(meta_of(vv0 + t, 1));
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
      vsf = fmaxf(vsf, __half2float(__ushort_as_half(uint16_t(mv[gg]))) * kup);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) vsf = fmaxf(vsf, __shfl_xor_sync(0xFFFFFFFFu, vsf, o));
  if (lane == 0) sm.red[warp] = vsf;
  __syncthreads();
  if (tid == 0) {
    float m2 = fmaxf(fmaxf(sm.red[0], sm.red[1]), fmaxf(sm.red[2], sm.red[3]));
    int e = 0;
    frexpf(m2, &e);
    sm.escale_w = m2 > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
  }
  __syncthreads();
  const float ew = sm.escale_w;
  float oacc[8][NT][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.f;
  const int hl = gq & 1;
#pragma unroll 1
  for (int step = warp; step < kTiles && uint32_t(step) * 16 < n; step += kAttWarps) {
    const uint32_t t0 = uint32_t(step) * 16 + 4 * tq;  // the lane's four tokens t0 .. t0 + 3
    uint32_t cw[4][NG][NBW];
    float sf4[4][NG], p4[4][NT];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t t = t0 + i;
      const bool ok = t < n;
      const uint8_t *row = in + base + uint64_t(vv0 + (ok ? t : 0)) * C::CB;
      const uint32_t *mv = reinterpret_cast<const uint32_t *>(meta_of(vv0 + (ok ? t : 0), 1));
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const uint8_t *src = row + gg * (G * BITS / 8) + gq * NB;
        if constexpr (NB == 8) {
          const uint2 x = ok ? __ldg(reinterpret_cast<const uint2 *>(src)) : make_uint2(0, 0);
          cw[i][gg][0] = x.x;
          cw[i][gg][1] = x.y;
        } else if constexpr (NB == 4) {
          cw[i][gg][0] = ok ? __ldg(reinterpret_cast<const uint32_t *>(src)) : 0u;
        } else if constexpr (NB == 2) {
          cw[i][gg][0] = ok ? uint32_t(__ldg(reinterpret_cast<const uint16_t *>(src))) : 0u;
        } else {
          cw[i][gg][0] = ok ? uint32_t(__ldg(src)) : 0u;
        }
        sf4[i][gg] = __half2float(__ushort_as_half(uint16_t(mv[gg]))) * kup;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) p4[i][nt] = ok ? sm.s[t][nt * 4 + (gq >> 1)] : 0.f;
    }
    // B fragments per group: column gq = (head nt * 4 + gq / 2, hi / lo)
    uint32_t wb[NG][NT][2];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float hi, lo;
          split_f16(p4[i][nt] * sf4[i][gg] * ew, hi, lo);
          v[i] = hl ? lo : hi;
        }
        wb[gg][nt][0] = f16x2(v[0], v[1]);
        wb[gg][nt][1] = f16x2(v[2], v[3]);
      }
    // A fragments (codes, rows = channels) and the products
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint32_t sel = uint32_t(b % 4) | (uint32_t(4 + b % 4) << 8);
        const uint32_t x01 = __byte_perm(cw[0][gg][b / 4], cw[1][gg][b / 4], sel);
        const uint32_t x23 = __byte_perm(cw[2][gg][b / 4], cw[3][gg][b / 4], sel);
        if constexpr (BITS == 4) {
          const int mt = gg * (G / 16) + b;
          uint32_t af[4];
          af[0] = codes_f16x2<0x000F000Fu>(x01);
          af[1] = codes_f16x2<0x000F000Fu>(x01 >> 4);
          af[2] = codes_f16x2<0x000F000Fu>(x23);
          af[3] = codes_f16x2<0x000F000Fu>(x23 >> 4);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma16816(oacc[mt][nt], af, wb[gg][nt][0], wb[gg][nt][1]);
        } else {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int mt = gg * (G / 16) + 2 * b + hf;
            uint32_t af[4];
            af[0] = codes_f16x2<0x00030003u>(x01 >> (4 * hf));
            af[1] = codes_f16x2<0x00030003u>(x01 >> (4 * hf + 2));
            af[2] = codes_f16x2<0x00030003u>(x23 >> (4 * hf));
            af[3] = codes_f16x2<0x00030003u>(x23 >> (4 * hf + 2));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma16816(oacc[mt][nt], af, wb[gg][nt][0], wb[gg][nt][1]);
          }
        }
      }
  }
  // outputs of the lane: rows gq, gq + 8 of each M-tile, heads nt * 4 + tq
  auto row_channel = [&](int mt, int row8) -> int {  // row8: 0 row gq, 1 row gq + 8
    const int gg = mt / (G / 16), rem = mt % (G / 16);
    if constexpr (BITS == 4) return 2 * (gg * (G / 2) + gq * NB + rem) + row8;
    else return 4 * (gg * (G / 4) + gq * NB + rem / 2) + 2 * (rem % 2) + row8;
  };
  const float inv_ew = 1.f / ew;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 4 + tq;
      sm.o[warp][g][row_channel(mt, 0)] = (oacc[mt][nt][0] + oacc[mt][nt][1]) * inv_ew;
      sm.o[warp][g][row_channel(mt, 1)] = (oacc[mt][nt][2] + oacc[mt][nt][3]) * inv_ew;
    }
  // zero terms sum_t p_t zf_t per (head, group): thread tid takes tokens
  // tid, tid + 128 for every head and group, then a warp reduction
  {
    float z[QPK][NG];
#pragma unroll
    for (int g = 0; g < QPK; ++g)
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) z[g][gg] = 0.f;
    for (uint32_t t = tid; t < n; t += kAttThreads) {
      const uint32_t *mv = reinterpret_cast<const uint32_t *>(meta_of(vv0 + t, 1));
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const float zf = __half2float(__ushort_as_half(uint16_t(mv[gg] >> 16))) * kup;
#pragma unroll
        for (int g = 0; g < QPK; ++g) z[g][gg] = fmaf(sm.s[t][g], zf, z[g][gg]);
      }
    }
#pragma unroll
    for (int g = 0; g < QPK; ++g)
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        float x = z[g][gg];
#pragma unroll
        for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
        if (lane == 0) sm.z[warp][g][gg] = x;
      }
  }
  __syncthreads();
  for (uint32_t i = tid; i < qpk * D; i += kAttThreads) {
    const uint32_t g = i / D, c = i - g * D;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) x += sm.o[w][g][c] + sm.z[w][g][c / G];
    part[g * kAttRec + 4 + c] = x;
  }
  if (tid < int(qpk)) {
    part[tid * kAttRec] = sm.m[tid];
    part[tid * kAttRec + 1] = sm.l[tid];
  }
}

}  // namespace kvc
