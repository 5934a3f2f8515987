// Definitions shared by the host launcher and the sm_100a kernels of libkvc.
//
// Stream format and arithmetic follow the readings stated in include/kvc.h:
// stage list from "Beyond Compression Ratio: High-Throughput KV Compression
// for Disaggregated LLM Serving" (Abstract, Methodology) and the podcast page
// "FastKVComp: checking whether high-throughput KV compression pays off"
// (episode notes); exact rules are this library's readings.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cmath>

#include "../../include/kvc.h"

#if defined(__CUDACC__)
#define KVC_HD __host__ __device__ __forceinline__
#else
#define KVC_HD inline
#endif

namespace kvc {

constexpr int kChunk = 16384;   // lossless chunk bytes
constexpr int kBitmap = 2048;   // zero-byte-elimination bitmap bytes
constexpr int kBitmap2 = 256;   // second-level bitmap bytes (pipelines 2 and 3)
constexpr int kHeader = 64;     // stream header bytes
constexpr uint32_t kMagic = 0x3143564Bu;  // "KVC1"
constexpr int kThreads = 256;   // compute threads per CTA (one vector each)
constexpr uint32_t kNoTile = 0xFFFFFFFFu;

// Every device wait is bounded: after this many nanoseconds of %globaltimer
// (or the iteration cap) the waiter records KVC_ERR_TIMEOUT and goes on. A
// recorded timeout is sticky: every other wait of the call sees it in the
// status word and gives up at once, so a failed call ends within about one
// wait limit.
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kWaitIters = 1u << 26;

// Workspace of kvc_compress, in this order (each part 256-byte aligned):
//   control   status word, flags word (bit 0: some code chunk shrank),
//             compaction ticket, compaction read count, ~(first shrinking
//             code chunk), (u64 at byte 24) padded bytes the shrinking code
//             chunks save
//   meta_nnz  u64 per meta chunk, accumulated 16-bit fields: shuffled-byte
//             nonzero count (bits 0..15), the same after the XOR of
//             pipelines 1 and 3 (16..31), nonzero bytes of the 2048-byte
//             bitmap (32..47) and of the bitmap after the XOR (48..63); all
//             but the first only in the search mode
//   code_nnz  u64 per code chunk: shuffled-byte nonzero count (bits 0..15),
//             nonzero bitmap bytes (16..31, search mode) and the number of
//             32-vector blocks accumulated so far (32..63)
//   done      u32 per code chunk: compaction read flags
//   code_size u32 per code chunk: stored size
//   meta_size u32 per meta chunk: stored size
//   code_off  u64 per code chunk: final offsets (compaction only)
//   meta      raw meta of every vector (meta chunk s at s * 16 KB), then
//             (compaction only) each meta chunk as stored
// Only control, meta_nnz, code_nnz and done need zeroing per call.
constexpr size_t kWsCtl = 256;
struct WsLayout {
  size_t meta_nnz, code_nnz, done, code_size, meta_size, code_off, meta, total, zero_bytes;
};

KVC_HD uint64_t round16(uint64_t x) { return (x + 15u) & ~uint64_t(15); }

// Chunk table entry (readings R12, R17): bits 0..15 unpadded size, 16..59
// offset from the data base in 16-byte units, 60..63 lossless pipeline id.
KVC_HD uint32_t entry_size(uint64_t e) { return uint32_t(e & 0xFFFFu); }
KVC_HD uint64_t entry_offset(uint64_t e) { return ((e >> 16) & 0xFFFFFFFFFFFull) << 4; }
KVC_HD uint32_t entry_pipe(uint64_t e) { return uint32_t(e >> 60); }
KVC_HD uint64_t make_entry(uint64_t off, uint32_t size, uint32_t pipe) {
  return (uint64_t(pipe) << 60) | ((off >> 4) << 16) | size;
}
KVC_HD uint64_t round256(uint64_t x) { return (x + 255u) & ~uint64_t(255); }

inline WsLayout ws_layout(uint64_t n_code, uint64_t n_meta) {
  WsLayout w{};
  w.meta_nnz = kWsCtl;
  w.code_nnz = w.meta_nnz + round256(8 * n_meta);
  w.done = w.code_nnz + round256(8 * n_code);
  w.code_size = w.done + round256(4 * n_code);
  w.meta_size = w.code_size + round256(4 * n_code);
  w.code_off = w.meta_size + round256(4 * n_meta);
  w.meta = w.code_off + round256(8 * n_code);
  w.total = w.meta + n_meta * uint64_t(kChunk);
  w.zero_bytes = w.code_size;
  return w;
}

// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): sign words of the +-1
// diagonal are its outputs counted from state = seed.
KVC_HD uint64_t splitmix64(uint64_t &state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// XOR masks that flip the bf16 sign bits of channel pair (2j, 2j+1).
KVC_HD void sign_masks(uint64_t seed, int d, uint32_t *mask) {
  uint64_t st = seed, w = 0;
  for (int c = 0; c < d; c += 2) {
    if (c % 64 == 0) w = splitmix64(st);
    uint32_t lo = uint32_t((w >> (c % 64)) & 1u), hi = uint32_t((w >> (c % 64 + 1)) & 1u);
    mask[c / 2] = (lo << 15) | (hi << 31);
  }
}

// Per-(layer, kv, head) diagonals (the FP4Quant abstract's variant of the
// randomized transform): vector index i takes SplitMix64 outputs number
// i*W .. i*W + W - 1 (W = d / 64) from state = seed, i.e. the generator
// advanced by i*W steps; index 0 is the global diagonal. S receives them as
// 32-bit words, S[j] holding channels 32j .. 32j + 31.
template <int D>
KVC_HD void vec_sign_words(uint64_t seed, uint32_t index, uint32_t (&S)[D / 32]) {
  uint64_t st = seed + uint64_t(index) * uint64_t(D / 64) * 0x9E3779B97F4A7C15ull;
#pragma unroll
  for (int j = 0; j < D / 64; ++j) {
    const uint64_t w = splitmix64(st);
    S[2 * j] = uint32_t(w);
    S[2 * j + 1] = uint32_t(w >> 32);
  }
}

// The XOR mask of channel pair (c, c + 1) (c even) from such words: bit 15
// flips channel c's bf16 sign, bit 31 channel c + 1's.
template <int D>
KVC_HD uint32_t pair_mask(const uint32_t (&S)[D / 32], int c) {
  const uint32_t w = S[c / 32] >> (c % 32);
  return ((w & 1u) << 15) | ((w & 2u) << 30);
}

// x / Q, correctly rounded, for a constant Q and x >= 0 (the quantizers'
// 2^b - 1 and 2^(b-1) - 1): Markstein's correction of the product with the
// rounded reciprocal (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990):
// q = RN(x * RN(1/Q)), the remainder x - q * Q exactly by one fused
// multiply-add, then RN(q + remainder * RN(1/Q)). The result equals the
// correctly rounded quotient for every finite x >= 0 and Q in {3, 7, 15, 127,
// 255}: checked over all of them on the host (this function compiled for
// the host), and on the GPU over samples of every binade through
// kvc_test_div_const.
template <int Q>
KVC_HD float div_const(float x) {
  if constexpr (Q == 1) {
    return x;
  } else {
    constexpr float c = 1.0f / float(Q);
#ifdef __CUDA_ARCH__
    const float q = __fmul_rn(x, c);
    return __fmaf_rn(__fmaf_rn(-q, float(Q), x), c, q);
#else
    const float q = x * c;
    return std::fmaf(std::fmaf(-q, float(Q), x), c, q);
#endif
  }
}

#ifdef __CUDACC__
// 1 / s for the encoder's scales s = h * 2^K (h a positive finite fp16
// value, K = 3 or 4): the hardware's approximate reciprocal y, then one
// Newton step with its residual fused, y + y * (1 - s * y) (Markstein's
// method, P. Markstein, IBM J. Res. Develop. 34(1), 1990). It equals the
// correctly rounded 1 / s for every such s: checked on the GPU over all of
// them through kvc_test_rcp_scale. (s is normal and so is 1 / s, so the
// approximation's flush of subnormals never acts.)
__device__ __forceinline__ float rcp_scale(float s) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(s));
  return __fmaf_rn(__fmaf_rn(-s, y, 1.0f), y, y);
}
#endif

// Sign sources of the transform kernels: the diagonal shared by every vector
// (masks in the kernel's parameters) or the vector's own (its words in
// registers). word(k) is the mask of channel pair (2k, 2k + 1).
// lo(k) is word(k) << 16: channel 2k's flip moved to bit 31, where adding it
// to the widened channel (an integer add) is the same as XOR-ing it in.
struct GlobalSigns {
  const uint32_t *mask;
  const uint32_t *lo_mask = nullptr;  // words << 16 (the encoder's widening)
  __device__ __forceinline__ uint32_t word(int k) const { return mask[k]; }
  __device__ __forceinline__ uint32_t lo(int k) const { return lo_mask[k]; }
  __device__ __forceinline__ uint4 quad(int q) const {  // words 4q .. 4q + 3
    return reinterpret_cast<const uint4 *>(mask)[q];
  }
};
template <int D>
struct VectorSigns {
  uint32_t S[D / 32];
  __device__ __forceinline__ uint32_t word(int k) const { return pair_mask<D>(S, 2 * k); }
  __device__ __forceinline__ uint32_t lo(int k) const { return ((S[k / 16] >> (2 * k % 32)) & 1u) << 31; }
  __device__ __forceinline__ uint4 quad(int q) const {
    return make_uint4(word(4 * q), word(4 * q + 1), word(4 * q + 2), word(4 * q + 3));
  }
};

#ifdef __CUDACC__
// FP4 helpers (the dual-scale e2m1 quantizer). e4m3 (fn variant: bias 7,
// 3 mantissa bits, largest finite 448, no inf) and e2m1 (bias 1, 1 mantissa
// bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6) from their bit patterns.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * (1.0f / 512.0f);
  return (b & 0x80u) ? -v : v;
}
// The smallest e4m3 value >= x (0 <= x, finite), at most 448: normals round
// the fp32 mantissa up to 3 bits (an integer add on the bit pattern),
// subnormals (x < 2^-6) to a multiple of 2^-9; the byte is returned.
__device__ __forceinline__ uint32_t e4m3_ru(float x) {
  if (x < 0.015625f) return uint32_t(ceilf(x * 512.0f));  // 0..8 (8 = 2^-6, code 0x08)
  const uint32_t u = (__float_as_uint(x) + 0xFFFFFu) & ~0xFFFFFu;
  if (__uint_as_float(u) > 448.0f) return 0x7Eu;
  return ((((u >> 23) & 255u) - 120u) << 3) | ((u >> 20) & 7u);
}
// e2m1 code -> fp32: magnitude index i = 2e + m, value 2^(e-1) (1 + m/2) for
// e > 0, m/2 for e = 0; bit 3 is the sign.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t i = c & 7u, e = i >> 1, m = i & 1u;
  const uint32_t mag = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  return __uint_as_float(mag | ((c & 8u) << 28));
}
// The e2m1 codes nearest to lo and hi (bits 0-3 and 4-7), ties to the even
// magnitude index, magnitudes above 6 to 6: the sm_100a conversion
// cvt.rn.satfinite.e2m1x2.f32, whose rounding is the rule of the FP4
// quantizer (a test compares it with the rule at every tie); a magnitude-0
// code loses its sign bit (no negative zero).
// The conversion's byte (lo in the low nibble) as it comes, -0 codes included.
__device__ __forceinline__ uint32_t e2m1x2_raw(float lo, float hi) {
  uint32_t d;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
      : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// Every nibble of w whose magnitude is 0 loses its sign bit (-0 -> code 0).
__device__ __forceinline__ uint32_t e2m1_zero_signs(uint32_t w) {
  const uint32_t m = w & 0x77777777u;                            // magnitudes
  const uint32_t nz = (m | (m >> 1) | (m >> 2)) & 0x11111111u;   // a nonzero magnitude per nibble
  return m | (w & (nz << 3));
}
__device__ __forceinline__ uint32_t e2m1x2_rne(float lo, float hi) {
  return e2m1_zero_signs(e2m1x2_raw(lo, hi));
}
__device__ __forceinline__ uint32_t e2m1_rne(float p) { return e2m1x2_rne(p, 0.f) & 0xFu; }
// Two e2m1 codes (the low byte of b: the low nibble first) as their values,
// by the hardware conversion to f16 (exact: every e2m1 value is an f16).
__device__ __forceinline__ float2 e2m1x2_to_float2(uint32_t b) {
  float lo, hi;
  asm("{\n .reg .b8 t;\n .reg .b16 a, c;\n .reg .b32 h;\n cvt.u8.u32 t, %2;\n"
      " cvt.rn.f16x2.e2m1x2 h, t;\n mov.b32 {a, c}, h;\n cvt.f32.f16 %0, a;\n"
      " cvt.f32.f16 %1, c;\n}"
      : "=f"(lo), "=f"(hi) : "r"(b));
  return make_float2(lo, hi);
}
#endif

// Unsigned 32-bit division by a run-time constant (Granlund and Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, the
// round-up variant): q = (umulhi(n, m) + n) >> s, exact for every n < 2^32.
struct FastDiv {
  uint32_t d, m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0, 0};
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) l++;
  f.s = l;
  f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  return f;
}
KVC_HD uint32_t fdiv(const FastDiv &f, uint32_t n) {
  uint32_t hi = uint32_t((uint64_t(n) * f.m) >> 32);
  return uint32_t((uint64_t(hi) + n) >> f.s);
}

// Vector addressing. Vector v (logical order [layer][kv][head][request]
// [token]) -> byte address of its head_dim contiguous bf16 values.
struct DenseLayout {
  // Tensor map of the input as 5-D [layers][2][kv_heads][tokens][head_dim]
  // (boxes of 32 tokens x 64 channels, 128-byte swizzle), valid iff tma != 0:
  // set by the host when tokens % 32 == 0, so a 32-vector block lies in one
  // head row.
  alignas(64) CUtensorMap tmap;
  uint8_t *base;
  int64_t s_l, s_kv, s_h, s_t;  // bytes
  FastDiv T, H;                 // tokens, kv_heads
  uint32_t tokens;
  uint32_t tma;
  uint32_t narrow;  // 1: every row at a non-negative offset below 64 GB from base
};

struct PagedLayout {
  // Tensor map of the pool as 5-D [layers][pages][2 * kv_heads][page_tokens]
  // [head_dim] (boxes of one run of 2^run_lg slots x 64 channels, 128-byte
  // swizzle), valid iff tma != 0: set by the host when kv and head merge into
  // one dimension (stride_kv == kv_heads * stride_head) and page_tokens is a
  // power of two 2^page_lg from 8 to 512 (runs of 16 slots, of 8 for pages
  // of 8).
  alignas(64) CUtensorMap tmap;
  uint32_t tma;
  uint32_t run_lg, page_lg;
  uint8_t *base;
  int64_t s_l, s_p, s_kv, s_h, s_slot;  // bytes
  const int32_t *page_table;
  int64_t pt_stride;
  int64_t num_pages;
  FastDiv T, H, PT;                     // total tokens, kv_heads, page tokens
  uint32_t n_req;
  uint32_t narrow;  // 1: every row at a non-negative offset below 64 GB from base
  uint32_t cum[KVC_MAX_REQUESTS + 1];   // token prefix per request
};

// Main encode kernel: codes of vector v to data base + v * CB (the raw code
// region), raw meta to the workspace, nonzero counts per chunk.
struct EncArgs {
  uint32_t V;          // vectors
  uint8_t *out;
  uint64_t data_base;
  uint32_t *status;
  uint32_t *flags;     // bit 0: some code chunk shrinks
  uint32_t *first_inv; // max over shrinking code chunks c of ~c (0: none)
  unsigned long long *saved;  // padded bytes the shrinking code chunks save
  unsigned long long *code_nnz;
  unsigned long long *meta_nnz;
  uint8_t *ws_meta;
  float *ymid;         // unfused baseline only: transformed vectors, d fp32 each
  float one;           // 1.0: the quantizer's integer rounding multiplies by it
  uint32_t mode;       // KVC_LOSSLESS_*
  uint32_t sym;        // 1: symmetric absmax quantizer (KVC_QUANT_SYM)
  uint32_t vec_signs;  // 1: per-(layer, kv, head) sign diagonals
  uint32_t fp4;        // 1: the FP4 quantizer (KVC_QUANT_FP4, 4-bit codes)
  uint64_t seed;       // sign seed (per-vector diagonals)
  FastDiv tdiv;        // tokens per (layer, kv, head): vector index = v / tokens
  uint32_t sign_mask[128];
  uint32_t sign_lo[128];  // sign_mask[k] << 16
};

// Finishing kernels: sizes and offsets of every chunk, meta chunks,
// chunk table, header; compaction when a code chunk shrank.
struct FinArgs {
  uint32_t V, n_code, n_meta, n_chunks;
  uint32_t cb, mb, vc, vm;  // code / meta bytes per vector, vectors per code / meta chunk
  uint8_t *out;
  uint64_t out_capacity;
  uint64_t data_base;
  uint64_t *out_bytes_dev;
  uint32_t *status;
  uint32_t *flags;
  uint32_t *first_inv;  // ~(first shrinking code chunk), 0 if none
  const unsigned long long *saved;  // padded bytes the shrinking code chunks save
  uint32_t *ticket;
  const unsigned long long *code_nnz;
  const unsigned long long *meta_nnz;
  uint32_t *code_size;
  uint32_t *done;
  uint32_t *meta_size;
  uint64_t *code_off;
  uint8_t *ws_meta;
  // header fields
  uint32_t layers, kv_heads, head_dim, group, bits, k, origin, n_req;
  uint64_t tokens, seed;
  // compaction waits give up after wait_ns (kWaitNs in every product call);
  // ticket_skip > 0 (a test of that limit only) starts the compaction's
  // tickets that many chunks late, so those chunks' read flags are never set
  uint64_t wait_ns;
  uint32_t ticket_skip;
  uint32_t mode;  // KVC_LOSSLESS_*
  uint32_t quant, signs;  // KVC_QUANT_*, KVC_SIGNS_* (header flags bits 1..3)
};

struct DecArgs {
  const uint8_t *in;
  uint64_t in_bytes;
  uint32_t *status;
  uint32_t layers, kv_heads, head_dim, n_req;
  uint64_t tokens;
  uint32_t V;
  uint32_t paged_receiver;   // 1: request count and lengths must match
  FastDiv tdiv;              // tokens: a vector's (layer, kv, head) index = v / tokens
  uint8_t *ws_meta;          // expanded meta chunks, 16 KB each
  uint32_t ws_meta_chunks;   // slots in ws_meta
};

// Per-kernel timing of the measurement entry points (kvc_compress_timed,
// kvc_decompress_timed): while such a call runs on this host thread, the
// launchers record timing_events[i] after the i-th kernel of the call
// (timing_events[0] before the first) and launch without programmatic
// dependence, so that each pair of events brackets exactly one kernel.
struct KernelTiming {
  const cudaEvent_t *events = nullptr;  // null: an ordinary call
  int next = 0;
};
KernelTiming &kernel_timing();  // this host thread's state
inline void timing_mark(cudaStream_t st) {
  KernelTiming &t = kernel_timing();
  if (t.events) cudaEventRecord(t.events[t.next++], st);
}

// Launchers, one translation unit per (head_dim, layout).
#define KVC_DECLARE_LAUNCHERS(D)                                                          \
  cudaError_t launch_encode_dense_d##D(int bits, int group, const EncArgs &a,             \
                                       const DenseLayout &lay, int sms, cudaStream_t st); \
  cudaError_t launch_encode_paged_d##D(int bits, int group, const EncArgs &a,             \
                                       const PagedLayout &lay, int sms, cudaStream_t st); \
  cudaError_t launch_encode_dense_d##D##_var(int bits, int group, const EncArgs &a,       \
                                             const DenseLayout &lay, int sms,             \
                                             cudaStream_t st);                            \
  cudaError_t launch_encode_paged_d##D##_var(int bits, int group, const EncArgs &a,       \
                                             const PagedLayout &lay, int sms,             \
                                             cudaStream_t st);                            \
  cudaError_t launch_decode_dense_d##D(const DecArgs &a, const DenseLayout &lay, int sms, \
                                       cudaStream_t st);                                  \
  cudaError_t launch_decode_paged_d##D(const DecArgs &a, const PagedLayout &lay, int sms, \
                                       cudaStream_t st);
KVC_DECLARE_LAUNCHERS(128)
KVC_DECLARE_LAUNCHERS(64)
#undef KVC_DECLARE_LAUNCHERS
// Unfused baseline: transform kernel (per layout), quantize kernel.
cudaError_t launch_transform_dense(int d, const EncArgs &a, const DenseLayout &lay, int sms,
                                   cudaStream_t st);
cudaError_t launch_transform_paged(int d, const EncArgs &a, const PagedLayout &lay, int sms,
                                   cudaStream_t st);
cudaError_t launch_quantize(int d, int bits, int group, const EncArgs &a, int sms, cudaStream_t st);
cudaError_t launch_finish_dense(const FinArgs &a, const DenseLayout &lay, int sms, cudaStream_t st);
// Attention over the compressed cache (kvc_attend).
struct AttnArgs {
  const uint8_t *in;
  uint64_t in_bytes;
  uint32_t *status;
  uint32_t layers, kv_heads, n_req, qpk;  // qpk: query heads per kv head
  uint32_t bits, group;                   // as the caller states them (checked)
  uint32_t fp4;                           // 1: the FP4 quantizer (checked)
  uint32_t cuda_cores;                    // 1: the CUDA-core kernel (measurement)
  uint64_t tokens;                        // all requests
  uint32_t V, splits;                     // vectors; CTAs per (layer, request, kv head)
  const uint16_t *q;                      // bf16 [layers][n_req][kv_heads * qpk][D]
  float scale;
  float *out;                             // fp32, the shape of q
  float *part;                            // per CTA and query head: m, l, o[D]
  const uint8_t *ws_meta;                 // meta chunks expanded by meta_expand_kernel
  uint8_t *prep;                          // tensor-core path: attend_prep_kernel's results
  uint32_t n_meta;                        // meta chunks
  uint32_t cum[KVC_MAX_REQUESTS + 1];     // token prefix per request
};
cudaError_t launch_attend(const AttnArgs &a, const DecArgs &d, int sms, cudaStream_t st);
// The tensor-core attention's preparation area (kvc_attend_mma.cuh).
struct PrepCtl {
  uint64_t base;
  uint32_t n_code;
};
KVC_HD uint64_t prep_qfrag_off(uint32_t n_meta) {
  return (64 + 8 * uint64_t(n_meta) + 255) & ~uint64_t(255);
}
KVC_HD uint64_t prep_bytes(uint32_t n_meta, uint32_t units) {
  return prep_qfrag_off(n_meta) + uint64_t(units) * (4096 + 256);
}
cudaError_t launch_finish_paged(const FinArgs &a, const PagedLayout &lay, int sms, cudaStream_t st);

}  // namespace kvc
