// Main encode kernel: load/gather -> signs -> fp32 Walsh-Hadamard -> group
// min/max -> fp16 meta -> quantize -> pack. The transformed tensor never
// reaches HBM (the fusion of "Beyond Compression Ratio: High-Throughput KV
// Compression for Disaggregated LLM Serving", Abstract: transform and
// quantization in one kernel with no intermediate tensor).
//
// The stream holds every code chunk before every meta chunk (reading R13), and
// a raw code chunk is just VC consecutive vectors' codes, so the raw code
// region is the plain array of per-vector codes: vector v's codes go straight
// to data base + v * CB. Whether zero-byte elimination pays for a chunk is
// decided from the number of nonzero bytes its bit-plane shuffle would have,
// which this kernel accumulates per chunk (chunk_nnz_part's OR-popcount
// identity); the finishing kernels (kvc_finish.cuh) write the table, the meta
// chunks and the header, and, only when some chunk shrinks and storing it
// eliminated pays for the shift of the later chunks (reading R16), re-encode
// and move code chunks. This kernel therefore has no dependency between threads
// beyond the warp reductions of those counts.
//
// Work: blocks of 32 consecutive vectors, one per lane; warps are fully
// independent and take blocks round-robin over the grid. Each thread holds
// one head_dim vector in registers as head_dim/2 pairs (c, c + d/2), so every
// butterfly stage but the last is a paired f32x2 add/subtract. A warp loads
// its next block's 32 rows into its shared-memory buffer as soon as every
// lane has read the current one: one tensor-map copy per 64-channel half for
// a dense tensor whose blocks are head-row tiles, otherwise a gather of
// 16-byte asynchronous copies, half a warp per row.
#pragma once

#include <type_traits>

#include "kvc_device.cuh"

namespace kvc {

constexpr int kEncWarps = 12;
constexpr int kEncThreads = kEncWarps * 32;

template <int D, int BITS, int G>
struct Cfg {
  static constexpr int ROW = D * 2;              // bytes of one bf16 vector
  static constexpr int CB = D * BITS / 8;        // code bytes per vector
  static constexpr int CW = CB / 4;              // code words per vector
  static constexpr int NG = D / G;               // groups per vector
  static constexpr int MB = NG * 4;              // meta bytes per vector
  static constexpr int VC = kChunk / CB;         // vectors per code chunk
  static constexpr int R = G * BITS / 32;        // code chunks per meta chunk
  static constexpr int VM = VC * R;              // vectors per meta chunk
  static constexpr int SLICE = VC * MB;          // meta bytes per code chunk
  static constexpr int LOG2D = D == 64 ? 6 : D == 128 ? 7 : 8;
  static constexpr int K = LOG2D / 2;            // meta stored x 2^-K
  static constexpr int QMAX = (1 << BITS) - 1;
  static constexpr int QH = (1 << (BITS - 1)) - 1;  // symmetric: codes -QH .. QH
  static_assert(VC % 32 == 0 && VM % 32 == 0, "a block of 32 vectors lies in one chunk");
  static_assert(R >= 2 && R <= 32, "segment size");
  static_assert(SLICE % 32 == 0, "meta slices hold whole 8-word groups");
};

// Shared memory: per-warp row buffers | per-warp mbarriers | request prefix
// (paged).
// A row buffer holds 32 rows (dense input) or 48 (paged input: a block's 32
// tokens start anywhere in a run of at most 16 slots of their pages, and its
// runs come in whole), per 64-channel half.
template <int D, bool kPaged = false>
struct EncSmem {
  static constexpr int ROWS = kPaged ? 48 : 32;
  static constexpr int HALF = ROWS * 128;                   // bytes per 64-channel half
  static constexpr size_t WBUF = size_t(D / 64) * HALF;     // 128-byte swizzled halves
  static constexpr size_t wbars = kEncWarps * WBUF;
  static constexpr size_t cum = wbars + kEncWarps * 8;
  static_assert(WBUF % 1024 == 0, "swizzled buffers stay 1024-byte aligned");
};
template <int D>
constexpr size_t enc_smem_bytes(bool paged) {
  return paged ? EncSmem<D, true>::cum + sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1)
               : EncSmem<D, false>::cum;
}

template <class L>
constexpr bool kIsPaged = std::is_same<L, PagedLayout>::value;

// ------------------------------------------------------------------------
// One vector in registers: pair j holds channels (j, j + d/2).
// ------------------------------------------------------------------------
template <int D>
struct Pairs {
  float2 p[D / 2];
  __device__ __forceinline__ float &at(int c) { return c < D / 2 ? p[c].x : p[c - D / 2].y; }
};

// Reading R2 on the pair layout: strides 1 .. d/4 pair whole pairs (j, j+h),
// both halves at once (f32x2, one rounding per element); stride d/2 is
// inside each pair. Same additions, same order as the scalar butterfly.
template <int D>
__device__ __forceinline__ void fwht_pairs(Pairs<D> &y) {
#pragma unroll
  for (int h = 1; h < D / 2; h <<= 1) {
#pragma unroll
    for (int j = 0; j < D / 2; ++j) {
      if ((j & h) == 0) {
        const float2 a = y.p[j], b = y.p[j + h];
        y.p[j] = add2(a, b);
        y.p[j + h] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < D / 2; ++j) {
    const float a = y.p[j].x, b = y.p[j].y;
    y.p[j].x = __fadd_rn(a, b);
    y.p[j].y = __fsub_rn(a, b);
  }
}

template <int D, int BITS, int G>
struct Enc : Cfg<D, BITS, G> {
  using C = Cfg<D, BITS, G>;

  // E1/E2: widen bf16 exactly and flip the sign bit of negative channels.
  // Word k of the row holds channels 2k (low half) and 2k+1 (high half): one
  // shift-and-add (the flip at bit 31 added) widens the low channel, one
  // three-input logic op the high one.
  template <class SG>
  static __device__ __forceinline__ void unpack(const uint8_t *row, const SG &sg, Pairs<D> &y) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
#pragma unroll
    for (int q = 0; q < D / 16; ++q) {
      const uint4 va = r4[q], vb = r4[q + D / 16];  // words 4q.., 4q + d/4..
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = 4 * q + e;
        y.p[2 * k] = make_float2(__uint_as_float((wa[e] << 16) + sg.lo(k)),
                                 __uint_as_float((wb[e] << 16) + sg.lo(k + D / 4)));
        y.p[2 * k + 1] = make_float2(__uint_as_float((wa[e] ^ sg.word(k)) & 0xFFFF0000u),
                                     __uint_as_float((wb[e] ^ sg.word(k + D / 4)) & 0xFFFF0000u));
      }
    }
  }

  // E1/E2 from a per-warp tensor-load buffer: this lane's row `row` of each
  // 64-channel half (HALF bytes apart), 16-byte chunk c stored at
  // row * 128 + ((c ^ (row % 8)) * 16) (the tensor maps' 128-byte swizzle,
  // which keeps these reads conflict-free for consecutive rows).
  template <int HALF = 4096, class SG>
  static __device__ __forceinline__ void unpack_swz(const uint8_t *wbuf, int row, const SG &sg,
                                                    Pairs<D> &y) {
    const int sw = row & 7;
    auto chunk = [&](int q) {
      return *reinterpret_cast<const uint4 *>(wbuf + (q >> 3) * HALF + row * 128 +
                                              (((q & 7) ^ sw) << 4));
    };
#pragma unroll
    for (int q = 0; q < D / 16; ++q) {
      const uint4 va = chunk(q), vb = chunk(q + D / 16);  // words 4q.., 4q + d/4..
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = 4 * q + e;
        y.p[2 * k] = make_float2(__uint_as_float((wa[e] << 16) + sg.lo(k)),
                                 __uint_as_float((wb[e] << 16) + sg.lo(k + D / 4)));
        y.p[2 * k + 1] = make_float2(__uint_as_float((wa[e] ^ sg.word(k)) & 0xFFFF0000u),
                                     __uint_as_float((wb[e] ^ sg.word(k + D / 4)) & 0xFFFF0000u));
      }
    }
  }

  // Group min / max (exact, order-free), NaN propagating so a non-finite
  // group is always seen: four independent running minima and maxima keep
  // few values live next to the vector.
  static __device__ __forceinline__ void minmax(Pairs<D> &y, int g, float &mn, float &mx) {
    minmax_at<G>(y, g * G, mn, mx);
  }
  // The same over channels c0 .. c0 + N - 1.
  template <int N>
  static __device__ __forceinline__ void minmax_at(Pairs<D> &y, int c0, float &mn, float &mx) {
    float lo[4], hi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) lo[i] = hi[i] = y.at(c0 + i);
#pragma unroll
    for (int c = 4; c < N; ++c) {
      const float u = y.at(c0 + c);
      lo[c & 3] = min2n(lo[c & 3], u);
      hi[c & 3] = max2n(hi[c & 3], u);
    }
    mn = min2n(min2n(lo[0], lo[1]), min2n(lo[2], lo[3]));
    mx = max2n(max2n(hi[0], hi[1]), max2n(hi[2], hi[3]));
  }

  // E4..E7 of the FP4 quantizer (reading R22, 4-bit only): per group an fp16
  // scale s2_h = RU16(fl(max|y| / 2688) * 2^-K) (2688 = 6 * 448), per
  // half-group an e4m3 micro-scale s1 = RU(fl(max_half|y| / (6 * s2))), at
  // most 448; S = s1 * s2 (exact), r = fl(1 / S) (0 for S = 0), code = e2m1
  // nearest to fl(y * r), ties to even. Meta word: s2_h | s1_0 << 16 |
  // s1_1 << 24. The codes are packed here: the conversion turns channels
  // (2k, 2k + 1) into byte k of the vector's codes (LSB first, reading R6),
  // and the -0 codes of a word's eight nibbles become 0 in one step.
  static __device__ __forceinline__ uint32_t quantize_fp4(Pairs<D> &y, uint32_t (&meta)[C::NG],
                                                          uint32_t (&code)[C::CW]) {
    static_assert(BITS == 4, "FP4 codes are 4-bit");
    uint32_t err = 0;
    float rr[2 * C::NG];  // 1 / S per half-group
    const float down = 1.0f / float(1 << C::K), up = float(1 << C::K);
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      float lo[2], hi[2];
      minmax_at<G / 2>(y, g * G, lo[0], hi[0]);
      minmax_at<G / 2>(y, g * G + G / 2, lo[1], hi[1]);
      if (!(isfinite(lo[0]) && isfinite(hi[0]) && isfinite(lo[1]) && isfinite(hi[1]))) err |= 1u;
      const float a0 = fmaxf(fabsf(lo[0]), fabsf(hi[0])), a1 = fmaxf(fabsf(lo[1]), fabsf(hi[1]));
      const __half sh = __float2half_ru(__fmul_rn(__fdiv_rn(fmaxf(a0, a1), 2688.0f), down));
      const uint16_t sb = __half_as_ushort(sh);
      if ((sb & 0x7FFFu) == 0x7C00u) err |= 2u;
      const float s2 = __fmul_rn(__half2float(sh), up);
      uint32_t s1[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        s1[h] = s2 == 0.0f ? 0u : e4m3_ru(__fdiv_rn(h ? a1 : a0, __fmul_rn(6.0f, s2)));
        const float S = __fmul_rn(e4m3_value(s1[h]), s2);
        rr[2 * g + h] = S == 0.0f ? 0.0f : __frcp_rn(S);
      }
      meta[g] = uint32_t(sb) | (s1[0] << 16) | (s1[1] << 24);
    }
#pragma unroll
    for (int j = 0; j < D / 2; ++j) {
      const int ha = j / (G / 2), hb = (j + D / 2) / (G / 2);
      y.p[j] = mul2(y.p[j], make_float2(rr[ha], rr[hb]));
    }
#pragma unroll
    for (int W = 0; W < C::CW; ++W) {  // channels 8W .. 8W + 7
      uint32_t b[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) b[k] = e2m1x2_raw(y.at(8 * W + 2 * k), y.at(8 * W + 2 * k + 1));
      code[W] = e2m1_zero_signs(
          __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410));
    }
    return err;
  }

  // E3..E7. Reading R5: asymmetric min/max group quantization, fp16 zero
  // (round down) and scale (round up), both x 2^-K; t = fl(y - zf),
  // p = fl(t * r), q = nearest integer to p, ties to even, each step rounded
  // on its own (no fused multiply-add). The integer rounding is
  // fl(p * one + 1.5 * 2^23) with `one` = 1.0 passed in at run time: p * 1
  // is exact, so this is the rounded sum p + 1.5 * 2^23, which leaves q in
  // the low bits (the sum lies in [2^23, 2^24), where the fp32 spacing is 1,
  // and 1.5 * 2^23 is even, so ties go to even q). Because that operation is
  // itself a multiply-add whose multiplier the compiler cannot see, the
  // product t * r before it can never be contracted into it. The clamp to
  // [0, 2^b - 1] never acts for a finite group: t >= 0 since zf <= min, and
  // sf >= (max - zf) / (2^b - 1) keeps p below 2^b - 1 + 2^-18. Codes pack
  // LSB first (reading R6).
  template <bool kFp4 = false>
  static __device__ __forceinline__ uint32_t vector(Pairs<D> &y, uint32_t (&code)[C::CW],
                                                    uint32_t (&meta)[C::NG], float one,
                                                    uint32_t sym) {
    fwht_pairs<D>(y);
    return quantize<kFp4>(y, code, meta, one, sym);
  }
  // E4..E7 on the transformed vector. With `sym` (reading R19, symmetric
  // absmax): scale s_h = RU16(fl(max|y| / (2^(b-1) - 1)) * 2^-K), stored zero
  // -2^(b-1) * s_h (exact, so the decoder's zf + q * sf is (q - 2^(b-1)) * sf),
  // p = fl(y * r) and code = nearest integer to p + 2^(b-1): the offset is
  // folded into the rounding constant (1.5 * 2^23 + 2^(b-1) is even, so ties
  // still go to even p) and the clamp to [-(2^(b-1) - 1), 2^(b-1) - 1] never
  // acts for a finite group (|p| <= max|y| / s32 * (1 + 2^-22)).
  template <bool kFp4 = false>
  static __device__ __forceinline__ uint32_t quantize(Pairs<D> &y, uint32_t (&code)[C::CW],
                                                      uint32_t (&meta)[C::NG], float one,
                                                      uint32_t sym) {
    uint32_t err = 0;
    if constexpr (kFp4) return quantize_fp4(y, meta, code);
    float zf[C::NG], rr[C::NG];  // zf: subtracted before the product (0 when symmetric)
    // x * 0 is 0 for finite x and NaN for an infinite or NaN x: nf turns NaN
    // once a group's min or max is not finite, rg once a stored zero or
    // scale overflows fp16
    float nf = 0.0f, rg = 0.0f;
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      float mn, mx;
      minmax(y, g, mn, mx);
      mn = __fadd_rn(mn, 0.0f);  // -0 -> +0
      mx = __fadd_rn(mx, 0.0f);
      nf = __fmaf_rn(mn, 0.0f, __fmaf_rn(mx, 0.0f, nf));
      const float down = 1.0f / float(1 << C::K), up = float(1 << C::K);
      __half zh, sh;
      if (sym) {
        const float am = fmaxf(fabsf(mn), fabsf(mx));
        sh = __float2half_ru(__fmul_rn(div_const<C::QH>(am), down));
        zh = (__half_as_ushort(sh) & 0x7FFFu) == 0
                 ? __ushort_as_half(0)
                 : __float2half_rd(__fmul_rn(__half2float(sh), -float(1 << (BITS - 1))));
        zf[g] = 0.0f;
      } else {
        zh = __float2half_rd(__fmul_rn(mn, down));
        zf[g] = __fmul_rn(__half2float(zh), up);
        const float s32 = div_const<C::QMAX>(__fsub_rn(mx, zf[g]));
        sh = __float2half_ru(__fmul_rn(s32, down));
      }
      const float sf = __fmul_rn(__half2float(sh), up);
      const uint16_t zb = __half_as_ushort(zh), sb = __half_as_ushort(sh);
      rg = __fmaf_rn(__half2float(zh), 0.0f, __fmaf_rn(sf, 0.0f, rg));
      rr[g] = sf == 0.0f ? 0.0f : rcp_scale(sf);
      meta[g] = uint32_t(sb) | (uint32_t(zb) << 16);
    }
    if (nf != 0.0f) err |= 1u;       // (NaN compares unequal)
    else if (rg != 0.0f) err |= 2u;
    const float kMagic = sym ? 12582912.0f + float(1 << (BITS - 1)) : 12582912.0f;  // 1.5 * 2^23
    const float2 mag = make_float2(kMagic, kMagic), one2 = make_float2(one, one);
#pragma unroll
    for (int j = 0; j < D / 2; ++j) {
      const int ga = j / G, gb = (j + D / 2) / G;
      const float2 t = sub2(y.p[j], make_float2(zf[ga], zf[gb]));
      const float2 p = mul2(t, make_float2(rr[ga], rr[gb]));
      y.p[j] = fma2(p, one2, mag);
    }
    pack(y, code);
    return err;
  }
  // E7: each code in the low bits of its float, packed LSB first (reading R6).
  static __device__ __forceinline__ void pack(Pairs<D> &y, uint32_t (&code)[C::CW]) {
    constexpr int per = 8 / BITS;  // codes per byte
#pragma unroll
    for (int W = 0; W < C::CW; ++W) {
      uint32_t b[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < per; ++e)
          acc += __float_as_uint(y.at((W * 4 + k) * per + e)) << (e * BITS);
        b[k] = acc;
      }
      code[W] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    }
  }
};

// E3..E7 (kFwht) or E4..E7 of this lane's vector v of block blk, its stores
// (codes in place, meta to the workspace), and the block's shuffled-byte
// nonzero counts, accumulated per code and meta chunk. With kSearch (the
// lossless search mode, reading R17) also the counts that size the other
// candidate pipelines: nonzero bitmap bytes (a bitmap byte covers 64 words
// of one bit plane, so it is nonzero iff that plane's bit is set in the OR
// of the 64 words) and the meta counts after the XOR of each word with the
// previous one, restarted at every run of 32 vectors (a block is one run).
template <int D, int BITS, int G, bool kFwht, bool kSearch, bool kFp4 = false>
__device__ __forceinline__ void encode_finish_block(const EncArgs &a, uint32_t blk, uint32_t v,
                                                    bool valid, Pairs<D> &y, uint32_t &err) {
  using C = Cfg<D, BITS, G>;
  using E = Enc<D, BITS, G>;
  const int lane = threadIdx.x & 31;
  const uint32_t V = a.V;
  uint32_t code[C::CW], meta[C::NG];
  if (valid) {
    if constexpr (kFwht)
      err |= E::template vector<kFp4>(y, code, meta, a.one, a.sym);
    else
      err |= E::template quantize<kFp4>(y, code, meta, a.one, a.sym);
    uint4 *cd = reinterpret_cast<uint4 *>(a.out + a.data_base + uint64_t(v) * C::CB);
#pragma unroll
    for (int q = 0; q < C::CW / 4; ++q)
      cd[q] = make_uint4(code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
    uint8_t *md = a.ws_meta + uint64_t(v) * C::MB;
    if constexpr (C::NG == 1) {
      *reinterpret_cast<uint32_t *>(md) = meta[0];
    } else if constexpr (C::NG == 2) {
      *reinterpret_cast<uint2 *>(md) = make_uint2(meta[0], meta[1]);
    } else {
      *reinterpret_cast<uint4 *>(md) = make_uint4(meta[0], meta[1], meta[2], meta[3]);
    }
  } else {
#pragma unroll
    for (int w = 0; w < C::CW; ++w) code[w] = 0;
#pragma unroll
    for (int g = 0; g < C::NG; ++g) meta[g] = 0;
  }

  // Shuffled-byte nonzero counts (chunk_nnz_part): 8-word groups of the
  // code region and of the meta region, summed per chunk.
  uint32_t cn = 0;
  if constexpr (C::CW >= 8) {
#pragma unroll
    for (int q = 0; q < C::CW / 8; ++q) {
      uint32_t o = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) o |= code[8 * q + w];
      cn += __popc(o);
    }
  } else {  // 4 words: two lanes form a group
    uint32_t o = code[0] | code[1] | code[2] | code[3];
    o |= __shfl_xor_sync(0xFFFFFFFFu, o, 1);
    cn = (lane & 1) ? 0u : __popc(o);
  }
  if constexpr (kSearch) {  // nonzero bitmap bytes of the code region
    constexpr int L64 = 64 / C::CW;  // vectors per 64-word group
    uint32_t ov = 0;
#pragma unroll
    for (int w = 0; w < C::CW; ++w) ov |= code[w];
#pragma unroll
    for (int o = 1; o < L64; o <<= 1) ov |= __shfl_xor_sync(0xFFFFFFFFu, ov, o);
    cn |= ((lane % L64) ? 0u : uint32_t(__popc(ov))) << 16;
  }
  uint32_t mo = 0;
#pragma unroll
  for (int g = 0; g < C::NG; ++g) mo |= meta[g];
  constexpr int kVecPerGroup = 32 / C::MB;  // vectors per 8-word meta group
#pragma unroll
  for (int o = 1; o < kVecPerGroup; o <<= 1) mo |= __shfl_xor_sync(0xFFFFFFFFu, mo, o);
  uint32_t mcnt = (lane % kVecPerGroup) ? 0u : __popc(mo), mbits = 0;
  if constexpr (kSearch) {
    // the XOR of pipelines 1 and 3 on this run of 32 vectors
    const uint32_t prev = __shfl_up_sync(0xFFFFFFFFu, meta[C::NG - 1], 1);
    uint32_t xo = valid ? meta[0] ^ (lane ? prev : 0u) : 0u;
#pragma unroll
    for (int g = 1; g < C::NG; ++g) xo |= valid ? meta[g] ^ meta[g - 1] : 0u;
#pragma unroll
    for (int o = 1; o < kVecPerGroup; o <<= 1) xo |= __shfl_xor_sync(0xFFFFFFFFu, xo, o);
    mcnt |= ((lane % kVecPerGroup) ? 0u : uint32_t(__popc(xo))) << 16;
    if constexpr (C::NG >= 2) {  // 64-word groups lie inside the block
      constexpr int L64 = 64 / C::NG;
      uint32_t b0 = mo, b1 = xo;
#pragma unroll
      for (int o = kVecPerGroup; o < L64; o <<= 1) {
        b0 |= __shfl_xor_sync(0xFFFFFFFFu, b0, o);
        b1 |= __shfl_xor_sync(0xFFFFFFFFu, b1, o);
      }
      mbits = (lane % L64) ? 0u : uint32_t(__popc(b0)) | (uint32_t(__popc(b1)) << 16);
    }
  }
  const uint32_t cs = __reduce_add_sync(0xFFFFFFFFu, cn);
  const uint32_t ms = __reduce_add_sync(0xFFFFFFFFu, mcnt);
  uint32_t mb = 0;
  if constexpr (kSearch && C::NG >= 2) mb = __reduce_add_sync(0xFFFFFFFFu, mbits);
  if (lane == 0) {
    // The block that completes a full code chunk sees its final counts and
    // flags the chunk if a lossless pipeline makes it shorter (reading R11,
    // R17), adding the padded bytes it would save (reading R16 weighs them).
    const uint32_t c = blk * 32 / C::VC;
    const unsigned long long old = atomicAdd(a.code_nnz + c, (1ull << 32) | cs);
    const uint32_t blocks = (min(uint32_t(C::VC), V - c * C::VC) + 31) / 32;
    const uint32_t nnz = (uint32_t(old) & 0xFFFFu) + (cs & 0xFFFFu);
    uint32_t size = kBitmap + nnz;
    if constexpr (kSearch) size = min(size, kBitmap2 + ((uint32_t(old) >> 16) + (cs >> 16)) + nnz);
    if (uint32_t(old >> 32) + 1 == blocks && blocks * 32 == uint32_t(C::VC) &&
        size < uint32_t(kChunk) && a.mode != KVC_LOSSLESS_NONE) {
      atomicOr(a.flags, 1u);
      atomicMax(a.first_inv, ~c);
      atomicAdd(a.saved, (unsigned long long)(uint32_t(kChunk) - uint32_t(round16(size))));
    }
    atomicAdd(a.meta_nnz + blk * 32 / C::VM, (unsigned long long)ms | ((unsigned long long)mb << 32));
  }
}

// ------------------------------------------------------------------------
// Load plans of a paged pool's blocks (before the encoder, in the encode
// step's interval). Block b (32 vectors, every full block but the last) gets
// 8 words at ws_meta + b * 32 * MB, the start of its own meta slot:
//   word 0: kind (bits 0-1: 1 = tensor-map runs, 2 = row gather), t0 % run
//           (bits 2-5), runs (6-8), kv * kv_heads + head (9-19), layer (20-31)
//   word 1 + j: run j's page << 5 | the run's position in its page.
// Runs need the block inside one request and every page inside the pool.
// Host conditions (add_tensor_map_paged): 2 * kv_heads <= 2048,
// layers <= 4096, num_pages < 2^27.
// ------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    paged_plan_kernel(const __grid_constant__ EncArgs a, const __grid_constant__ PagedLayout lay,
                      uint32_t slot_bytes) {
  __shared__ uint32_t cum[KVC_MAX_REQUESTS + 1];
  for (uint32_t r = threadIdx.x; r <= lay.n_req; r += blockDim.x) cum[r] = lay.cum[r];
  __syncthreads();
  // the meta slots' previous users (the last call's finishing kernels) are
  // done: the clear before this waited for them
  grid_dependency_wait();
  const uint32_t n_blocks = (a.V + 31) / 32;
  const uint32_t rlg = lay.run_lg, plg = lay.page_lg;
  const uint32_t rmask = (1u << rlg) - 1u, qmask = (1u << (plg - rlg)) - 1u;
  for (uint32_t b = blockIdx.x * blockDim.x + threadIdx.x; b + 1 < n_blocks;
       b += gridDim.x * blockDim.x) {
    const uint32_t v0 = b * 32, lkh = fdiv(lay.T, v0), u0 = v0 - lkh * lay.T.d;
    uint32_t w[8] = {2u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (u0 + 32 <= lay.T.d) {
      uint32_t lo = 0, hi = lay.n_req;  // cum[lo] <= u0 < cum[hi]
      while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) / 2;
        if (cum[mid] <= u0) lo = mid; else hi = mid;
      }
      const uint32_t t0 = u0 - cum[lo];
      if (u0 + 32 <= cum[lo + 1]) {
        const uint32_t runs = ((t0 + 31) >> rlg) - (t0 >> rlg) + 1;  // 2 or 3 (runs of 16)
        const int32_t *row = lay.page_table + int64_t(lo) * lay.pt_stride;
        bool ok = true;
#pragma unroll
        for (uint32_t j = 0; j < 5; ++j) {  // (at most 5 runs: runs of 8)
          if (j < runs) {
            const uint32_t hp = (t0 >> rlg) + j;  // the run's index in the request
            const int32_t pg = __ldg(row + (hp >> (plg - rlg)));
            ok &= pg >= 0 && int64_t(pg) < lay.num_pages;
            w[1 + j] = (uint32_t(pg) << 5) | (hp & qmask);
          }
        }
        if (ok) {
          const uint32_t lk = fdiv(lay.H, lkh), h = lkh - lk * lay.H.d;
          w[0] = 1u | ((t0 & rmask) << 2) | (runs << 6) | (((lk & 1u) * lay.H.d + h) << 9) |
                 ((lk >> 1) << 20);
        }
      }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(a.ws_meta + uint64_t(b) * slot_bytes);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// ------------------------------------------------------------------------
// The kernel.
// ------------------------------------------------------------------------
// kVar bit 0: per-(layer, kv, head) sign diagonals (each lane derives its
// vector's diagonal from the seed) instead of the one in the kernel's
// parameters; bit 1: the FP4 quantizer (reading R22).
template <int D, int BITS, int G, class Layout, bool kNarrow, bool kSearch, int kVar>
__global__ void __launch_bounds__(kEncThreads, 1)
    encode_kernel(const __grid_constant__ EncArgs a, const __grid_constant__ Layout lay) {
  using C = Cfg<D, BITS, G>;
  using E = Enc<D, BITS, G>;
  constexpr bool kPaged = kIsPaged<Layout>;
  constexpr bool kVec = (kVar & 1) != 0, kFp4 = (kVar & 2) != 0;
  using S = EncSmem<D, kPaged>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t *wbuf = smem + warp * S::WBUF;
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem + S::wbars) + warp;
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(smem + S::cum);

  if (lane == 0) {
    mbar_init(wbar, 1);
    mbar_fence_init();
  }
  __syncwarp();  // the warp's barrier is initialized before any lane waits on it
  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
    __syncthreads();
  }

  const uint32_t V = a.V;
  const uint32_t n_blocks = (V + 31) / 32;
  const uint32_t stride = gridDim.x * kEncWarps;
  uint32_t blk = blockIdx.x * kEncWarps + (tid >> 5);

  // Source row of vector v for the gather path (null past the end or for a
  // page outside the pool, which is recorded).
  auto src_of = [&](uint32_t v) -> const uint8_t * {
    if (v >= V) return nullptr;
    bool ok;
    const uint8_t *p = vec_addr(lay, s_cum, v, ok);
    if (!ok) {
      set_status(a.status, KVC_ERR_CORRUPT);
      return nullptr;
    }
    return p;
  };

  uint32_t phase = 0, err = 0;
  auto finish_block = [&](uint32_t blk, uint32_t v, bool valid, Pairs<D> &y) {
    encode_finish_block<D, BITS, G, true, kSearch, kFp4>(a, blk, v, valid, y, err);
  };
  // E1/E2 of vector v from row `row` of the warp's buffer.
  auto unpack = [&](int row, uint32_t v, Pairs<D> &y) {
    if constexpr (kVec) {
      VectorSigns<D> sg;
      vec_sign_words<D>(a.seed, fdiv(a.tdiv, v), sg.S);
      E::template unpack_swz<S::HALF>(wbuf, row, sg, y);
    } else {
      E::template unpack_swz<S::HALF>(wbuf, row, GlobalSigns{a.sign_mask, a.sign_lo}, y);
    }
  };

  bool use_tma = false;
  if constexpr (!kPaged) use_tma = lay.tma != 0;
  if constexpr (!kPaged) {
    if (use_tma) {
      // Per-warp tensor loads: every block is 32 vectors of one head row
      // (tokens % 32 == 0, so V % 32 == 0 and no block is partial).
      auto issue_tma = [&](uint32_t b) {
        if (lane == 0) {
          const uint32_t v0 = b * 32, lkh = fdiv(lay.T, v0), t0 = v0 - lkh * lay.T.d;
          const uint32_t lk = fdiv(lay.H, lkh), h = lkh - lk * lay.H.d;
          mbar_arrive_expect_tx(wbar, uint32_t(D / 64) * 4096u);  // two 32-row boxes
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(wbuf + hh * 4096, &lay.tmap, hh * 64, int(t0), int(h), int(lk & 1u),
                        int(lk >> 1), wbar);
        }
      };
      if (blk < n_blocks) issue_tma(blk);
      // The launch may overlap the workspace clear before it: the first
      // rows load meanwhile; counts and status are touched only after this.
      grid_dependency_wait();
#pragma unroll 1
      for (; blk < n_blocks; blk += stride) {
        if (!mbar_wait(wbar, phase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
        phase ^= 1;
        Pairs<D> y;
        unpack(lane, blk * 32 + lane, y);
        // every lane has read the buffer; the next load may overwrite it
        fence_proxy_async_smem();
        __syncwarp();
        if (blk + stride < n_blocks) issue_tma(blk + stride);
        finish_block(blk, blk * 32 + lane, true, y);
      }
    }
  }
  auto gather = [&](const uint8_t *rowp) {
    if constexpr (kNarrow)
      gather_rows_narrow<D / 8, S::HALF>(wbuf, lay.base,
                                         rowp ? uint32_t((rowp - lay.base) >> 4) : 0u);
    else
      gather_rows<D, S::HALF>(wbuf, rowp, a.out);
  };
  if constexpr (kPaged) {
    grid_dependency_wait();  // the plans (paged_plan_kernel)
    // A block whose 32 tokens lie in one request (all but about one in a
    // hundred of a batch of long requests) loads as the runs of its pages (a
    // run: 2^run_lg slots, 16 or, for pages of 8, 8): lane j < runs issues
    // one tensor box of run j per 64-channel half into slot j of the buffer,
    // so lane i's row is row (t0 % run) + i. Other blocks (a request
    // boundary, a page outside the pool, no tensor map, the last block) are
    // gathered row by row, lane i's row at row i, which records a bad page.
    // paged_plan_kernel wrote each full block's plan into the first 32 bytes
    // of the block's own meta slot, which only this warp writes, and only
    // after reading the plan (two blocks ahead of its use).
    const uint32_t rlg = lay.run_lg;
    const uint8_t *plans = a.ws_meta;
    auto plan = [&](uint32_t b, uint32_t &own) -> uint32_t {
      own = 0;
      if (b >= n_blocks) return 0u;
      if (!lay.tma || b + 1 == n_blocks) return 2u;
      const uint32_t *pw = reinterpret_cast<const uint32_t *>(plans + uint64_t(b) * (32 * C::MB));
      own = __ldcg(pw + 1 + min(lane, 4));
      return __ldcg(pw);
    };
    // Issues block b's loads; returns the kind and the row shift.
    auto issue = [&](uint32_t b, uint32_t p, uint32_t own) -> uint32_t {
      if ((p & 3u) == 1u) {
        const uint32_t runs = (p >> 6) & 7u;
        if (lane == 0) mbar_arrive_expect_tx(wbar, (runs << rlg) * uint32_t(D / 64) * 128u);
        __syncwarp();
        if (uint32_t(lane) < runs) {
          const int kvh = int((p >> 9) & 2047u), layer = int(p >> 20);
          const int slot = int((own & 31u) << rlg), pg = int(own >> 5);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(wbuf + hh * S::HALF + (lane << (rlg + 7)), &lay.tmap, hh * 64, slot, kvh,
                        pg, layer, wbar);
        }
        return p & 63u;
      }
      if ((p & 3u) == 2u) gather(src_of(b * 32 + lane));
      return p & 3u;
    };
    uint32_t npg;
    uint32_t cur = issue(blk, plan(blk, npg), npg);
    uint32_t next = plan(blk + stride, npg);
#pragma unroll 1
    for (; blk < n_blocks; blk += stride) {
      const uint32_t v = blk * 32 + lane;
      if ((cur & 3u) == 1u) {
        if (!mbar_wait(wbar, phase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
        phase ^= 1;
      } else {
        cp_async_wait_all();
        __syncwarp();  // every lane's copies have landed
      }
      Pairs<D> y;
      unpack(lane + int((cur >> 2) & 15u), v, y);
      // every lane has read the buffer; the next load may overwrite it
      fence_proxy_async_smem();
      __syncwarp();
      cur = issue(blk + stride, next, npg);
      next = plan(blk + 2 * stride, npg);
      finish_block(blk, v, v < V, y);
    }
  } else if (!use_tma) {
    grid_dependency_wait();  // the workspace clear (src_of may record a status)
    // Row addresses are looked up one block ahead of their gather.
    if (blk < n_blocks) gather(src_of(blk * 32 + lane));
    const uint8_t *next = src_of((blk + stride) * 32 + lane);
#pragma unroll 1
    for (; blk < n_blocks; blk += stride) {
      const uint32_t v = blk * 32 + lane;
      cp_async_wait_all();
      __syncwarp();  // every lane's copies have landed
      Pairs<D> y;
      unpack(lane, v, y);
      __syncwarp();  // every lane has read the buffer; the next gather may overwrite it
      if (blk + stride < n_blocks) gather(next);
      next = src_of((blk + 2 * stride) * 32 + lane);
      finish_block(blk, v, v < V, y);
    }
  }
  err = __reduce_or_sync(0xFFFFFFFFu, err);
  if (lane == 0) {
    if (err & 1u) set_status(a.status, KVC_ERR_NONFINITE);
    if (err & 2u) set_status(a.status, KVC_ERR_RANGE);
  }
}

}  // namespace kvc
