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
  float s[kAttTok][kAttMaxG];            // scores, then weights
  float o[kAttWarps][kAttMaxG][128];     // per-warp partial outputs
  float z[kAttWarps][kAttMaxG][4];       // per-warp sum_t p * zf per group
  float vsf[kAttTok][4], vzf[kAttTok][4];  // values' scale and zero per token and group
  float qs[kAttMaxG][4];                 // sum of qt over each group
  float wmax[kAttWarps][kAttMaxG];
  float m[kAttMaxG], l[kAttMaxG];
  float red[kAttWarps];
  float escale_q, escale_w;              // 1 / 2^eq, 2^ew
  const uint8_t *mptr[2][2];
  uint32_t ms0[2];
};

// Results of attend_prep_kernel in the workspace (a.prep):
//   [0, 64)         PrepCtl: the stream's data base and code chunk count
//   [64, ..)        meta chunk s at mptr[s] (raw in the stream or expanded)
//   prep_qfrag(u)   unit u's query fragments: uint4 [8 k-blocks][32 lanes]
//                   = (hi 2tq, 2tq + 1 | hi + 8 | lo | lo + 8) of head lane/4
//   prep_qsx(u)     unit u's group sums qs[8][4] and 1 / 2^eq at [32]
// (PrepCtl, prep_qfrag_off and prep_bytes: kvc_internal.h.)

// Once per call: CTA `units` checks the header and every chunk table entry
// the attention reads (code chunks raw and in place, raw meta chunks inside
// the stream) and records every meta chunk's address; CTA u < units turns
// unit u's queries into qt = (scale / d) H D q (its keys' diagonal), their
// group sums, the power-of-two scale 2^eq of the fp16 split and the lanes'
// B fragments of the score products. The attention CTAs of a unit (one per
// 256-token split) then start from these.
// kPairs (4 query heads per kv head): the score product's 8 columns are
// (head, hi / lo) pairs, column n = 2 * head + part, so one product per
// k-block carries both parts; otherwise the columns are 8 heads and the hi
// and lo parts are two products.
template <int BITS, int G, bool kPairs>
__global__ void __launch_bounds__(kAttThreads) attend_prep_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int D = 128;
  using C = Cfg<D, BITS, G>;
  constexpr int NG = D / G;
  __shared__ alignas(16) float qt[8][128];
  __shared__ uint32_t mask[64];
  __shared__ float red[kAttWarps];
  __shared__ float es_s;
  __shared__ uint32_t hdr_ok;
  grid_dependency_wait();  // the meta expansion
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t H = a.kv_heads, qpk = a.qpk;
  const uint32_t units = a.layers * a.n_req * H;
  const uint8_t *in = a.in, *table = in + kHeader;
  PrepCtl *ctl = reinterpret_cast<PrepCtl *>(a.prep);
  if (blockIdx.x == units) {  // the header and the table
    if (tid == 0) {
      uint64_t base, seed;
      uint32_t n_code;
      const bool ok = attn_header_ok<D>(a, base, n_code, seed);
      hdr_ok = ok;
      if (ok) {
        ctl->base = base;
        ctl->n_code = n_code;
      } else {
        set_status(a.status, KVC_ERR_CORRUPT);
      }
    }
    __syncthreads();
    if (!hdr_ok) return;
    const uint64_t base = ctl->base, sb = ld_u64(in + 56), code_bytes = uint64_t(a.V) * C::CB;
    const uint32_t n_code = ctl->n_code;
    bool bad = false;
    for (uint32_t c = tid; c < n_code; c += kAttThreads) {
      const uint64_t e = ld_u64(table + 8 * uint64_t(c)), rest = code_bytes - uint64_t(c) * kChunk;
      bad |= !(entry_size(e) == (rest < kChunk ? rest : uint64_t(kChunk)) && entry_pipe(e) == 0 &&
               entry_offset(e) == uint64_t(c) * kChunk);
    }
    const uint8_t **mptr = reinterpret_cast<const uint8_t **>(a.prep + 64);
    for (uint32_t s = tid; s < a.n_meta; s += kAttThreads) {
      const uint64_t e = ld_u64(table + 8 * (uint64_t(n_code) + s));
      const uint32_t mlen = min(uint32_t(C::VM), a.V - s * C::VM) * C::MB;
      const bool raw = entry_size(e) == mlen;
      bad |= raw && !(entry_pipe(e) == 0 && base + entry_offset(e) + mlen <= sb);
      mptr[s] = raw ? in + base + entry_offset(e) : a.ws_meta + uint64_t(s) * kChunk;
    }
    if (bad) set_status(a.status, KVC_ERR_CORRUPT);
    return;
  }
  // unit u = (l, r, h): its queries
  if (a.in_bytes < kHeader) return;  // (the header CTA reports it)
  const uint32_t u = blockIdx.x, h = u % H, lr = u / H, r = lr % a.n_req, l = lr / a.n_req;
  if (tid == 0) {
    const uint64_t seed = ld_u64(in + 40);
    if (in[11] & 8u) {  // the keys' own diagonal: index (l, 0, h)
      uint32_t S[D / 32];
      vec_sign_words<D>(seed, (l * 2 + 0) * H + h, S);
      for (int k = 0; k < D / 2; ++k) mask[k] = pair_mask<D>(S, 2 * k);
    } else {
      sign_masks(seed, D, mask);
    }
  }
  __syncthreads();
  float qmax = 0.f;
  for (uint32_t g = warp; g < 8u; g += kAttWarps) {
    const uint16_t *qv = a.q + ((uint64_t(l) * a.n_req + r) * H * qpk + h * qpk + g) * D;
    float y[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t ch = lane + 32 * c;
      const uint32_t sgn = (mask[ch >> 1] >> ((ch & 1) ? 31 : 15)) & 1u;
      y[c] = 0.f;
      if (g < qpk) y[c] = __uint_as_float((uint32_t(qv[ch]) << 16) ^ (sgn << 31));
    }
    warp_fwht128(y, lane);
    const float f = a.scale / float(D);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      y[c] *= f;
      qt[g][lane + 32 * c] = y[c];
      qmax = fmaxf(qmax, fabsf(y[c]));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xFFFFFFFFu, qmax, o));
  if (lane == 0) red[warp] = qmax;
  __syncthreads();
  if (tid == 0) {
    const float mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    int e = 0;
    frexpf(mx, &e);  // mx < 2^e
    es_s = mx > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
  }
  __syncthreads();
  float *qsx = reinterpret_cast<float *>(a.prep + prep_qfrag_off(a.n_meta) + uint64_t(units) * 4096 +
                                         uint64_t(u) * 256);
  for (int pr = warp; pr < 8 * NG; pr += kAttWarps) {  // group sums
    const int g = pr / NG, gg = pr % NG;
    float x = 0.f;
#pragma unroll
    for (int c = lane; c < G; c += 32) x += qt[g][gg * G + c];
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane == 0) qsx[g * 4 + gg] = x;
  }
  if (tid == 0) qsx[32] = 1.f / es_s;
  // B fragments: lane `lane` of an attention warp (head lane / 4, tq =
  // lane % 4); this thread builds k-blocks 2 * warp and 2 * warp + 1
  const int gq = lane >> 2, tq = lane & 3;
  auto score_ch = [&](int kb, int k) -> int {
    const int j = (k % 8) / 2, hi8 = k / 8, sub = k % 2;
    if constexpr (BITS == 4) return 8 * (4 * (kb / 2) + j) + 2 * (kb % 2) + hi8 + 4 * sub;
    else return 16 * kb + (2 * j + hi8) + 8 * sub;
  };
  uint4 *qf = reinterpret_cast<uint4 *>(a.prep + prep_qfrag_off(a.n_meta) + uint64_t(u) * 4096);
  const float es = es_s;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int kb = 2 * warp + i;
    float hi[4], lo[4];
    const int ks[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};
    const int head = kPairs ? gq >> 1 : gq;
#pragma unroll
    for (int k = 0; k < 4; ++k) split_f16(qt[head][score_ch(kb, ks[k])] * es, hi[k], lo[k]);
    if constexpr (kPairs) {  // column gq = (head gq / 2, part gq % 2)
      const float *v = (gq & 1) ? lo : hi;
      qf[kb * 32 + lane] = make_uint4(f16x2(v[0], v[1]), f16x2(v[2], v[3]), 0u, 0u);
    } else {
      qf[kb * 32 + lane] = make_uint4(f16x2(hi[0], hi[1]), f16x2(hi[2], hi[3]), f16x2(lo[0], lo[1]),
                                      f16x2(lo[2], lo[3]));
    }
  }
}

// QPK: query heads per kv head rounded up to 4 or 8 (the heads of the
// softmax; the products always have 8 columns, one per query head).
template <int BITS, int G, int QPK>
__global__ void __launch_bounds__(kAttThreads) attend_mma_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int D = 128;
  using C = Cfg<D, BITS, G>;
  static_assert(BITS == 2 || BITS == 4, "2- and 4-bit codes");
  static_assert(QPK == 4 || QPK == 8, "query-head tiles of 4");
  constexpr bool kPairs = QPK == 4;  // columns (head, hi / lo): see attend_prep_kernel
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
  const uint8_t *in = a.in;
  const uint32_t T = uint32_t(a.tokens);
  grid_dependency_wait();  // the preparation (a dependent launch of it)

  // ---- the preparation's results: header and table checked (the status
  // word), meta chunk addresses, this unit's query fragments and sums
  if (*reinterpret_cast<const volatile uint32_t *>(a.status) != 0) return;
  const PrepCtl *pc = reinterpret_cast<const PrepCtl *>(a.prep);
  const uint32_t units = a.layers * a.n_req * H;
  if (tid < 4 && t_a < t_b) {  // (x, k): keys / values, first / second chunk of the range
    const uint32_t x = tid >> 1, k = tid & 1;
    const uint64_t v0 = uint64_t((l * 2 + x) * H + h) * T + a.cum[r];
    const uint32_t s0 = uint32_t((v0 + t_a) / C::VM), s1 = uint32_t((v0 + t_b - 1) / C::VM);
    const uint8_t *const *mptr = reinterpret_cast<const uint8_t *const *>(a.prep + 64);
    if (k == 0) sm.ms0[x] = s0;
    sm.mptr[x][k] = s0 + k <= s1 ? mptr[s0 + k] : nullptr;
  }
  const float *qsx = reinterpret_cast<const float *>(a.prep + prep_qfrag_off(a.n_meta) +
                                                     uint64_t(units) * 4096 + uint64_t(unit) * 256);
  if (tid < 32) sm.qs[tid / 4][tid % 4] = qsx[tid];
  if (tid == 32) sm.escale_q = qsx[32];  // (here: 1 / 2^eq)
  uint32_t qh[8][2], ql[8][2];  // B fragments of head gq: hi and lo parts
  {
    const uint4 *qf = reinterpret_cast<const uint4 *>(a.prep + prep_qfrag_off(a.n_meta) +
                                                      uint64_t(unit) * 4096);
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      const uint4 v = __ldg(qf + kb * 32 + lane);
      qh[kb][0] = v.x, qh[kb][1] = v.y, ql[kb][0] = v.z, ql[kb][1] = v.w;
    }
  }
  __syncthreads();
  if (t_a >= t_b) {
    for (uint32_t g = tid; g < qpk; g += kAttThreads) {
      part[g * kAttRec] = -INFINITY;
      part[g * kAttRec + 1] = 0.f;
    }
    return;
  }
  const uint64_t base = pc->base;
  const uint32_t n = t_b - t_a;
  auto meta_of = [&](uint32_t v, int x) -> const uint8_t * {
    const uint32_t s = v / C::VM;
    return sm.mptr[x][s - sm.ms0[x]] + uint64_t(v - s * C::VM) * C::MB;
  };
  const uint32_t kv0 = ((l * 2 + 0) * H + h) * T + a.cum[r] + t_a;  // key of token t_a
  const uint32_t vv0 = ((l * 2 + 1) * H + h) * T + a.cum[r] + t_a;  // value of token t_a
  const float kup = float(1 << C::K);  // meta is stored x 2^-K

  constexpr int kTiles = kAttTok / 16;
  float mx[2] = {-INFINITY, -INFINITY};  // heads 2tq, 2tq + 1
  const float inv_eq = sm.escale_q;
#pragma unroll 1
  for (int tile = warp; tile < kTiles && uint32_t(tile) * 16 < n; tile += kAttWarps) {
    const uint32_t tA = uint32_t(tile) * 16 + gq, tB = tA + 8;  // CTA-relative tokens
    const bool okA = tA < n, okB = tB < n;
    // the lane's code words of both tokens
    constexpr int NW = BITS == 4 ? 4 : 8;
    uint32_t wA[NW], wB[NW];
    const uint8_t *rowA = in + base + uint64_t(kv0 + tA) * C::CB;
    const uint8_t *rowB = in + base + uint64_t(kv0 + tB) * C::CB;
    if constexpr (BITS == 4) {
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        wA[i] = okA ? __ldg(reinterpret_cast<const uint32_t *>(rowA) + 4 * i + tq) : 0u;
        wB[i] = okB ? __ldg(reinterpret_cast<const uint32_t *>(rowB) + 4 * i + tq) : 0u;
      }
    } else {  // the whole 32-byte row
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 xa = okA ? __ldg(reinterpret_cast<const uint4 *>(rowA) + i) : make_uint4(0, 0, 0, 0);
        const uint4 xb = okB ? __ldg(reinterpret_cast<const uint4 *>(rowB) + i) : make_uint4(0, 0, 0, 0);
        wA[4 * i] = xa.x, wA[4 * i + 1] = xa.y, wA[4 * i + 2] = xa.z, wA[4 * i + 3] = xa.w;
        wB[4 * i] = xb.x, wB[4 * i + 1] = xb.y, wB[4 * i + 2] = xb.z, wB[4 * i + 3] = xb.w;
      }
    }
    float acc[NG][4];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[gg][i] = 0.f;
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
      mma16816(acc[kb / kPerG], af, qh[kb][0], qh[kb][1]);
      if constexpr (!kPairs) mma16816(acc[kb / kPerG], af, ql[kb][0], ql[kb][1]);
    }
    // scores: c0, c1 = token tA, heads 2tq, 2tq + 1; c2, c3 = token tB
    const uint32_t *mA = reinterpret_cast<const uint32_t *>(meta_of(kv0 + (okA ? tA : 0), 0));
    const uint32_t *mB = reinterpret_cast<const uint32_t *>(meta_of(kv0 + (okB ? tB : 0), 0));
    float sc[4] = {0.f, 0.f, 0.f, 0.f};  // (tA, 2tq), (tA, 2tq + 1), (tB, 2tq), (tB, 2tq + 1)
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) {
      const uint32_t ma = mA[gg], mb = mB[gg];
      const float sfa = __half2float(__ushort_as_half(uint16_t(ma))) * kup;
      const float zfa = __half2float(__ushort_as_half(uint16_t(ma >> 16))) * kup;
      const float sfb = __half2float(__ushort_as_half(uint16_t(mb))) * kup;
      const float zfb = __half2float(__ushort_as_half(uint16_t(mb >> 16))) * kup;
      if constexpr (kPairs) {  // c0 + c1: token tA, head tq; c2 + c3: token tB
        const float q0 = sm.qs[tq][gg];
        sc[0] = fmaf(sfa, (acc[gg][0] + acc[gg][1]) * inv_eq, fmaf(zfa, q0, sc[0]));
        sc[2] = fmaf(sfb, (acc[gg][2] + acc[gg][3]) * inv_eq, fmaf(zfb, q0, sc[2]));
      } else {
        const float q0 = sm.qs[2 * tq][gg], q1 = sm.qs[2 * tq + 1][gg];
        sc[0] = fmaf(sfa, acc[gg][0] * inv_eq, fmaf(zfa, q0, sc[0]));
        sc[1] = fmaf(sfa, acc[gg][1] * inv_eq, fmaf(zfa, q1, sc[1]));
        sc[2] = fmaf(sfb, acc[gg][2] * inv_eq, fmaf(zfb, q0, sc[2]));
        sc[3] = fmaf(sfb, acc[gg][3] * inv_eq, fmaf(zfb, q1, sc[3]));
      }
    }
    if constexpr (kPairs) {
      if (okA) {
        sm.s[tA][tq] = sc[0];
        mx[0] = fmaxf(mx[0], sc[0]);
      }
      if (okB) {
        sm.s[tB][tq] = sc[2];
        mx[0] = fmaxf(mx[0], sc[2]);
      }
    } else {
      if (okA) {
        *reinterpret_cast<float2 *>(&sm.s[tA][2 * tq]) = make_float2(sc[0], sc[1]);
        mx[0] = fmaxf(mx[0], sc[0]);
        mx[1] = fmaxf(mx[1], sc[1]);
      }
      if (okB) {
        *reinterpret_cast<float2 *>(&sm.s[tB][2 * tq]) = make_float2(sc[2], sc[3]);
        mx[0] = fmaxf(mx[0], sc[2]);
        mx[1] = fmaxf(mx[1], sc[3]);
      }
    }
  }
  // per-head maxima: lanes of equal tq hold the same heads (kPairs: head tq)
#pragma unroll
  for (int e = 0; e < (kPairs ? 1 : 2); ++e) {
    float x = mx[e];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    if (gq == 0) sm.wmax[warp][kPairs ? tq : 2 * tq + e] = x;
  }
  __syncthreads();
  if (tid < QPK) {
    float x = sm.wmax[0][tid];
    for (int w = 1; w < kAttWarps; ++w) x = fmaxf(x, sm.wmax[w][tid]);
    sm.m[tid] = x;
  }
  __syncthreads();
  // weights p = exp(s - m) in place (heads < QPK; QPK divides the thread
  // count, so thread tid keeps head tid % QPK), their sums per head; the
  // values' scales and zeros staged per token, and their largest scale
  {
    float x = 0.f;
    const uint32_t g = uint32_t(tid) % QPK;
    for (uint32_t i = tid; i < n * QPK; i += kAttThreads) {
      const uint32_t t = i / QPK;
      const float p = expf(sm.s[t][g] - sm.m[g]);
      sm.s[t][g] = p;
      x += p;
    }
#pragma unroll
    for (int o = 16; o >= QPK; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane < QPK) sm.wmax[warp][lane] = x;  // (reused: per-warp sums)
    float vsf = 0.f;
    for (uint32_t t = tid; t < n; t += kAttThreads) {
      const uint32_t *mv = reinterpret_cast<const uint32_t *>(meta_of(vv0 + t, 1));
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const uint32_t m = mv[gg];
        const float sf = __half2float(__ushort_as_half(uint16_t(m))) * kup;
        sm.vsf[t][gg] = sf;
        sm.vzf[t][gg] = __half2float(__ushort_as_half(uint16_t(m >> 16))) * kup;
        vsf = fmaxf(vsf, sf);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) vsf = fmaxf(vsf, __shfl_xor_sync(0xFFFFFFFFu, vsf, o));
    if (lane == 0) sm.red[warp] = vsf;
  }
  __syncthreads();
  if (tid < QPK) {
    float x = 0.f;
    for (int w = 0; w < kAttWarps; ++w) x += sm.wmax[w][tid];
    sm.l[tid] = x;
  }
  if (tid == 0) {
    float m2 = fmaxf(fmaxf(sm.red[0], sm.red[1]), fmaxf(sm.red[2], sm.red[3]));
    int e = 0;
    frexpf(m2, &e);
    sm.escale_w = m2 > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
  }
  // zero terms sum_t p_t zf_t per (head, group): lane -> pair, warp -> a
  // quarter of the tokens
  {
    const int pr = lane;
    if (pr < QPK * NG) {
      const int g = pr / NG, gg = pr % NG;
      float x = 0.f;
      for (uint32_t t = uint32_t(warp); t < n; t += kAttWarps) x = fmaf(sm.s[t][g], sm.vzf[t][gg], x);
      sm.z[warp][g][gg] = x;
    }
  }
  __syncthreads();

  // ---- value pass. Tokens: lane tq holds k-slots 2tq, 2tq + 1, 2tq + 8,
  // 2tq + 9 = tokens 4tq .. 4tq + 3 of the 16-token step. Channels: the lane
  // (row gq) takes NB = G * BITS / 64 contiguous bytes of every group; byte
  // i of its run in group gg feeds M-tile(s) gg * G / 16 + i (4-bit: low
  // nibble row gq, high nibble row gq + 8) or + 2i, 2i + 1 (2-bit: bit pairs
  // 0, 1 and 2, 3 of the byte for the first, 4, 5 and 6, 7 for the second).
  // Columns: head gq, with the hi and lo parts of p * sf as two products.
  constexpr int NB = G * BITS / 64;        // bytes per lane and group
  constexpr int NBW = (NB + 3) / 4;        // their words
  const float ew = sm.escale_w;
  float oacc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) oacc[mt][i] = 0.f;
#pragma unroll 1
  for (int step = warp; step < kTiles && uint32_t(step) * 16 < n; step += kAttWarps) {
    const uint32_t t0 = uint32_t(step) * 16 + 4 * tq;  // the lane's four tokens t0 .. t0 + 3
    uint32_t cw[4][NG][NBW];
    float x[4][NG];  // p * sf * 2^ew of head gq
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t t = t0 + i;
      const bool ok = t < n;
      const uint8_t *row = in + base + uint64_t(vv0 + (ok ? t : 0)) * C::CB;
      const float p = ok ? sm.s[t][kPairs ? gq >> 1 : gq] * ew : 0.f;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const uint8_t *src = row + gg * (G * BITS / 8) + gq * NB;
        if constexpr (NB == 8) {
          const uint2 v = ok ? __ldg(reinterpret_cast<const uint2 *>(src)) : make_uint2(0, 0);
          cw[i][gg][0] = v.x;
          cw[i][gg][1] = v.y;
        } else if constexpr (NB == 4) {
          cw[i][gg][0] = ok ? __ldg(reinterpret_cast<const uint32_t *>(src)) : 0u;
        } else if constexpr (NB == 2) {
          cw[i][gg][0] = ok ? uint32_t(__ldg(reinterpret_cast<const uint16_t *>(src))) : 0u;
        } else {
          cw[i][gg][0] = ok ? uint32_t(__ldg(src)) : 0u;
        }
        x[i][gg] = ok ? p * sm.vsf[t][gg] : 0.f;
      }
    }
    // B fragments per group: hi parts, and lo = x - hi
    uint32_t wh[NG][2], wl[NG][2];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float x0 = x[2 * k][gg], x1 = x[2 * k + 1][gg];
        const uint32_t hv = f16x2(x0, x1);
        const uint32_t lv = f16x2(x0 - __half2float(__ushort_as_half(uint16_t(hv))),
                                  x1 - __half2float(__ushort_as_half(uint16_t(hv >> 16))));
        if constexpr (kPairs) {  // column gq = (head gq / 2, part gq % 2)
          wh[gg][k] = (gq & 1) ? lv : hv;
        } else {
          wh[gg][k] = hv;
          wl[gg][k] = lv;
        }
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
          mma16816(oacc[mt], af, wh[gg][0], wh[gg][1]);
          if constexpr (!kPairs) mma16816(oacc[mt], af, wl[gg][0], wl[gg][1]);
        } else {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int mt = gg * (G / 16) + 2 * b + hf;
            uint32_t af[4];
            af[0] = codes_f16x2<0x00030003u>(x01 >> (4 * hf));
            af[1] = codes_f16x2<0x00030003u>(x01 >> (4 * hf + 2));
            af[2] = codes_f16x2<0x00030003u>(x23 >> (4 * hf));
            af[3] = codes_f16x2<0x00030003u>(x23 >> (4 * hf + 2));
            mma16816(oacc[mt], af, wh[gg][0], wh[gg][1]);
            if constexpr (!kPairs) mma16816(oacc[mt], af, wl[gg][0], wl[gg][1]);
          }
        }
      }
  }
  // outputs of the lane: rows gq, gq + 8 of each M-tile, heads 2tq, 2tq + 1
  auto row_channel = [&](int mt, int row8) -> int {  // row8: 0 row gq, 1 row gq + 8
    const int gg = mt / (G / 16), rem = mt % (G / 16);
    if constexpr (BITS == 4) return 2 * (gg * (G / 2) + gq * NB + rem) + row8;
    else return 4 * (gg * (G / 4) + gq * NB + rem / 2) + 2 * (rem % 2) + row8;
  };
  const float inv_ew = 1.f / ew;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int c0 = row_channel(mt, 0), c1 = row_channel(mt, 1);
    if constexpr (kPairs) {  // columns 2tq, 2tq + 1: head tq's hi and lo parts
      sm.o[warp][tq][c0] = (oacc[mt][0] + oacc[mt][1]) * inv_ew;
      sm.o[warp][tq][c1] = (oacc[mt][2] + oacc[mt][3]) * inv_ew;
    } else {
      sm.o[warp][2 * tq][c0] = oacc[mt][0] * inv_ew;
      sm.o[warp][2 * tq + 1][c0] = oacc[mt][1] * inv_ew;
      sm.o[warp][2 * tq][c1] = oacc[mt][2] * inv_ew;
      sm.o[warp][2 * tq + 1][c1] = oacc[mt][3] * inv_ew;
    }
  }
  __syncthreads();
  for (uint32_t i = tid; i < qpk * D; i += kAttThreads) {
    const uint32_t g = i / D, c = i - g * D;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) v += sm.o[w][g][c] + sm.z[w][g][c / G];
    part[g * kAttRec + 4 + c] = v;
  }
  if (tid < int(qpk)) {
    part[tid * kAttRec] = sm.m[tid];
    part[tid * kAttRec + 1] = sm.l[tid];
  }
}

}  // namespace kvc
