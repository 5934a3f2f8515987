// Device building blocks of libkvc (sm_100a): mbarriers and bulk-async copies,
// memory-model helpers, paired fp32 arithmetic, the register Walsh-Hadamard
// butterfly, the 32x32 bit transpose, block scans and vector addressing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvc_internal.h"

namespace kvc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: a kernel launched with launch_after() is
// set up while the previous kernel on the stream runs; it calls
// grid_dependency_wait() before anything else, which returns once that
// kernel has completed and its writes are visible. (No kernel triggers its
// dependents early: measured slower, their CTAs then wait on busy SMs.)
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// First error of a call wins.
__device__ __forceinline__ void set_status(uint32_t *status, uint32_t code) {
  atomicCAS(status, 0u, code);
}
__device__ __forceinline__ bool timed_out(const uint32_t *status) {
  return *reinterpret_cast<const volatile uint32_t *>(status) == KVC_ERR_TIMEOUT;
}
// Poll step of a bounded spin: true means give up (time, iterations, or a
// timeout already recorded by another waiter). Checks every 64 iterations.
__device__ __forceinline__ bool spin_expired(uint32_t it, uint64_t t0, const uint32_t *status,
                                             uint64_t limit_ns = kWaitNs) {
  if (it >= kWaitIters) return true;
  if ((it & 63u) != 63u) return false;
  return globaltimer() - t0 > limit_ns || timed_out(status);
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (spin_expired(i, t0, status)) return false;
  }
}

// ---------------------------------------------------- bulk-async copies --
// Tensor-map load of a 5-D box into shared memory, completion counted in
// bytes on `bar` (this CTA's buffer only). c0 is the innermost coordinate.
__device__ __forceinline__ void tma_load_5d(void *sdst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, int c4, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(sdst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar))
      : "memory");
}

// Tensor-map store of a 5-D box from shared memory (bulk group completion).
__device__ __forceinline__ void tma_store_5d(const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                             int c4, const void *ssrc) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group"
      " [%0, {%1, %2, %3, %4, %5}], [%6];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(ssrc))
      : "memory");
}

// global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *sdst, const void *gsrc, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(sdst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// shared -> global, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_s2g(void *gdst, const void *ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// 16-byte asynchronous global -> shared copy issued by this thread (L2 only);
// src_bytes 0 zero-fills the destination and reads nothing.
__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sdst)), "l"(gsrc),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Waits for all of this thread's committed 16-byte copies.
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// bulk-async reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// ------------------------------------------------------- memory model --
__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Invalidates an L2 line without writing it back (its content is dead).
__device__ __forceinline__ void discard_l2(const void *p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// ---------------------------------------------------- fp32 arithmetic --
// Paired fp32 ops (sm_100 f32x2): each lane is one IEEE round-to-nearest-even
// operation. Written as PTX with an explicit .rn modifier, which the compiler
// never contracts into a fused multiply-add (the codec's bit-exactness
// depends on every product and sum being rounded separately).
__device__ __forceinline__ uint64_t f2_bits(float2 a) { return *reinterpret_cast<uint64_t *>(&a); }
__device__ __forceinline__ float2 bits_f2(uint64_t r) { return *reinterpret_cast<float2 *>(&r); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
// a*b + c with one rounding. Used only where a*b is exact (a small integer
// times an fp16 value, or a value times 1.0), so the result equals the
// separately rounded product-then-sum.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(r);
}
// Measured on sm_100a: a paired multiply followed by a paired add can be
// fused, so no product that needs its own rounding feeds an add here; the
// quantizer rounds its product to an integer with a multiply-add by a
// run-time 1.0 instead (kvc_encode.cuh).
// min / max that return NaN if any input is NaN.
__device__ __forceinline__ float min3n(float a, float b, float c) {
  float d;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3n(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min2n(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float max2n(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Walsh-Hadamard butterfly of one head_dim vector in registers (reading R2):
// strides h = 1, 2, ..., d/2 in ascending order; each pair (i, i+h) with
// (i & h) == 0 becomes (a+b, a-b), one rounding each.
template <int D>
__device__ __forceinline__ void fwht(float (&y)[D]) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; ++i) {
      if ((i & h) == 0) {
        const float a = y[i], b = y[i + h];
        y[i] = __fadd_rn(a, b);
        y[i + h] = __fsub_rn(a, b);
      }
    }
  }
}

// In-register transpose of a 32x32 bit matrix: afterwards bit l of a[p] is
// bit p of the original a[l]. Recursive exchange of off-diagonal blocks of
// 16, 8, 4, 2 and 1 bits.
KVC_HD void transpose32(uint32_t (&a)[32]) {
  const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int j = 16 >> lvl;
    const uint32_t m = masks[lvl];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if ((k & j) == 0) {
        const uint32_t t = ((a[k] >> j) ^ a[k + j]) & m;
        a[k] ^= t << j;
        a[k + j] ^= t;
      }
    }
  }
}

// Byte permute (PRMT semantics: selector nibble i picks byte i of the result
// from the eight bytes y:x, x being bytes 0..3), usable on the host as well.
KVC_HD uint32_t prmt(uint32_t x, uint32_t y, uint32_t sel) {
#ifdef __CUDA_ARCH__
  return __byte_perm(x, y, sel);
#else
  const uint64_t v = (uint64_t(y) << 32) | x;
  uint32_t r = 0;
  for (int i = 0; i < 4; ++i) r |= uint32_t((v >> (8 * ((sel >> (4 * i)) & 7))) & 0xFFu) << (8 * i);
  return r;
#endif
}

// transpose32 split between two threads. Half h holds rows 16h .. 16h+15 of
// the 32x32 bit matrix (a[i] = row 16h + i), `other` the partner's a[i].
// The 16-bit block exchange is one byte permute per row:
//   row i      keeps its low half and takes the low half of row i + 16 on top,
//   row i + 16 keeps its high half and takes the high half of row i below.
KVC_HD uint32_t transpose_split_stage16(uint32_t mine, uint32_t other, int h) {
  return prmt(mine, other, h ? 0x3276u : 0x5410u);
}
// The remaining levels (8, 4, 2, 1 bits) act within each half. The 8-bit
// level is a byte permute too.
KVC_HD void transpose_split_rest(uint32_t (&a)[16]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t x = a[k], y = a[k + 8];
    a[k] = prmt(x, y, 0x6240u);      // bytes x0 y0 x2 y2
    a[k + 8] = prmt(x, y, 0x7351u);  // bytes x1 y1 x3 y3
  }
  const uint32_t masks[3] = {0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int lvl = 0; lvl < 3; ++lvl) {
    const int j = 4 >> lvl;
    const uint32_t m = masks[lvl];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if ((k & j) == 0) {
        const uint32_t t = ((a[k] >> j) ^ a[k + j]) & m;
        a[k] ^= t << j;
        a[k + j] ^= t;
      }
    }
  }
}

// -------------------------------------------------------------- scans --
// Exclusive sum over the first NT threads of the block (named barrier 1);
// also returns the total. `red` holds NT/32 words of shared memory.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t *red, uint32_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  named_bar_sync(1, NT);
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t r = red[w];
    before += (w < warp) ? r : 0u;
    all += r;
  }
  named_bar_sync(1, NT);
  total = all;
  return before + incl - x;
}
template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t x, uint32_t *red) {
  uint32_t total;
  block_excl_scan<NT>(x, red, total);
  return total;
}

// ------------------------------------------- lossless stage (16 KB chunk) --
// Reading R10 (bit planes of 32-bit little-endian words) and R11 (zero-byte
// elimination: 2048-byte bitmap + nonzero bytes), on a chunk in shared
// memory, by the first 256 threads.

// Nonzero bytes the bit-plane shuffle of the chunk would have: byte i of
// plane p is nonzero iff bit p of (w[8i] | ... | w[8i+7]) is set, so the
// count is the sum of popcounts of 8-word ORs; no shuffle is needed to
// decide between raw and eliminated storage. This thread's part.
template <int NT>
__device__ __forceinline__ uint32_t chunk_nnz_part(const uint8_t *buf) {
  constexpr int kGroups = kChunk / 32 / NT;  // 8-word groups per thread
  const uint4 *s = reinterpret_cast<const uint4 *>(buf) + threadIdx.x * 2 * kGroups;
  uint32_t n = 0;
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    const uint4 a = s[2 * q], b = s[2 * q + 1];
    n += __popc(a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w);
  }
  return n;
}

// Plane words: the shuffled chunk as 4096 little-endian words, word
// p * 128 + m holding bit p of words 32m .. 32m+31 (bytes p*512 + 4m ..).
// Their shared-memory image (scratch between the transpose and the byte
// compaction) keeps word (p, m) at p * 128 + (m ^ 16 * (p >> 4)).
__device__ __forceinline__ uint32_t pw_index(uint32_t p, uint32_t m) {
  return p * 128 + (m ^ ((p >> 4) << 4));
}

// The 128 groups of 32 words are transposed by thread pairs (the first 256
// threads): lane l of warp w takes group m = 16w + 4(l >> 3) + (l & 3) and
// half h = (l >> 2) & 1; its partner is lane l ^ 4. The pair transposes the
// group's rows rotated by r = 4s, s = l & 3 (half h reads its four 16-byte
// pieces from piece 4h + s on, so the eight lanes of a shared-memory phase
// hit eight different bank groups); rotating the rows rotates every
// transposed word by r bits, which a funnel shift undoes. In the image the
// partners' words (same m, planes p and p + 16) fall in different banks.
struct PairLane {
  int m, h, s;
};
__device__ __forceinline__ PairLane pair_lane() {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  return {16 * warp + 4 * (lane >> 3) + (lane & 3), (lane >> 2) & 1, lane & 3};
}

__device__ __forceinline__ void planes_from_words(const uint8_t *buf, uint32_t *pw) {
  const PairLane L = pair_lane();
  const uint4 *src = reinterpret_cast<const uint4 *>(buf + L.m * 128);
  uint32_t a[16];  // rows 16h .. 16h+15 of the rotated group
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = src[(4 * L.h + q + L.s) & 7];
    a[4 * q] = v.x, a[4 * q + 1] = v.y, a[4 * q + 2] = v.z, a[4 * q + 3] = v.w;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i)
    a[i] = transpose_split_stage16(a[i], __shfl_xor_sync(0xFFFFFFFFu, a[i], 4), L.h);
  transpose_split_rest(a);
  const int r = 4 * L.s;
#pragma unroll
  for (int i = 0; i < 16; ++i) pw[pw_index(16 * L.h + i, L.m)] = __funnelshift_l(a[i], a[i], r);
}
__device__ __forceinline__ void words_from_planes(const uint32_t *pw, uint8_t *buf) {
  const PairLane L = pair_lane();
  const int r = 4 * L.s;
  uint32_t a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t x = pw[pw_index(16 * L.h + i, L.m)];
    a[i] = __funnelshift_r(x, x, r);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i)
    a[i] = transpose_split_stage16(a[i], __shfl_xor_sync(0xFFFFFFFFu, a[i], 4), L.h);
  transpose_split_rest(a);  // a[i] = word (16h + i + r) mod 32 of the group
  uint4 *dst = reinterpret_cast<uint4 *>(buf + L.m * 128);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    dst[(4 * L.h + q + L.s) & 7] = make_uint4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
}

// Nonzero-byte mask of a word: bit b set iff byte b is nonzero. The top bit
// of each byte of ((x & 0x7F..) + 0x7F..) | x is set iff the byte is
// nonzero (the add cannot carry out of a byte); one multiply then gathers
// bits 7, 15, 23, 31 into bits 28..31 (the other partial products land on
// distinct bits below 28 or above 31, so nothing carries into 28..31).
KVC_HD uint32_t nz_nibble(uint32_t x) {
  const uint32_t m = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x) & 0x80808080u;
  return (m * 0x00204081u) >> 28;
}

// Inclusive prefix sum over the warp.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Byte-permute selectors, indexed by a 4-bit nonzero-byte mask n:
// expand: byte b takes source byte #(set bits of n below b) if bit b is set,
//         zero otherwise;
// compact: byte i takes the position of the i-th set bit of n, zero beyond.
__device__ __forceinline__ uint32_t expand_selector(uint32_t n) {
  uint32_t sel = 0, j = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const bool on = (n >> b) & 1u;
    sel |= (on ? j : 4u) << (4 * b);
    j += on;
  }
  return sel;
}
__device__ __forceinline__ uint32_t compact_selector(uint32_t n) {
  uint32_t sel = 0x4444u, j = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    if ((n >> b) & 1u) {
      sel = (sel & ~(0xFu << (4 * j))) | (uint32_t(b) << (4 * j));
      ++j;
    }
  }
  return sel;
}

// Byte positions of the compaction. Warp w covers plane words 512w ..
// 512w + 511 in four rounds; in round k lane l takes the four words
// j = 512w + 128k + 4l .. + 3 (plane 4w + k), whose bitmap bits are the
// 16-bit bitmap word j / 4. cnt[k] is the lane's nonzero-byte count in round
// k; q[k] receives the exclusive prefix over all words before its first one
// (plus the bitmap), `total` the chunk's count. Two rounds share one warp
// scan (a round's warp total is at most 512, so 16-bit halves cannot
// overflow); warp totals go through red[] (named barrier 1, first NT
// threads). The caller passes another barrier before red is reused.
template <int NT>
__device__ __forceinline__ void ze_positions(const uint32_t (&cnt)[4], uint32_t *red,
                                             uint32_t (&q)[4], uint32_t &total,
                                             uint32_t data_base = kBitmap) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t i01 = warp_incl_scan(cnt[0] | (cnt[1] << 16));
  const uint32_t i23 = warp_incl_scan(cnt[2] | (cnt[3] << 16));
  const uint32_t t01 = __shfl_sync(0xFFFFFFFFu, i01, 31), t23 = __shfl_sync(0xFFFFFFFFu, i23, 31);
  const uint32_t r0 = t01 & 0xFFFFu, r1 = t01 >> 16, r2 = t23 & 0xFFFFu, r3 = t23 >> 16;
  if (lane == 0) red[warp] = r0 + r1 + r2 + r3;
  named_bar_sync(1, NT);
  uint32_t base = data_base, all = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t v = red[w];
    base += (w < warp) ? v : 0u;
    all += v;
  }
  total = all;
  q[0] = base + (i01 & 0xFFFFu) - cnt[0];
  q[1] = base + r0 + (i01 >> 16) - cnt[1];
  q[2] = base + r0 + r1 + (i23 & 0xFFFFu) - cnt[2];
  q[3] = base + r0 + r1 + r2 + (i23 >> 16) - cnt[3];
}

// buf holds a full chunk (first 256 threads); on return it holds bitmap + nonzero bytes (the
// caller knows their count from chunk_nnz_part). scr: 16 KB scratch. Each
// word's nonzero bytes are packed by one byte permute and stored at its
// position; the lanes of a warp store next to one another. The bitmap goes
// to `bitmap` (buf itself for the one-level form) and the nonzero bytes to
// buf from `data_base` on.
template <int NT>
__device__ __forceinline__ bool ze_encode(uint8_t *buf, uint8_t *scr, uint32_t *red,
                                          uint8_t *bitmap = nullptr, uint32_t data_base = kBitmap) {
  static_assert(NT == 256, "eight warps of 512 plane words");
  __shared__ uint32_t lut[16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t *pw = reinterpret_cast<uint32_t *>(scr);
  if (tid < 16) lut[tid] = compact_selector(tid);
  planes_from_words(buf, pw);
  named_bar_sync(1, NT);  // buf is free from here on
  uint32_t x[4][4], nib[4], cnt[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 v = *reinterpret_cast<const uint4 *>(pw + pw_index(4 * warp + k, 4 * lane));
    x[k][0] = v.x, x[k][1] = v.y, x[k][2] = v.z, x[k][3] = v.w;
    nib[k] = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) nib[k] |= nz_nibble(x[k][e]) << (4 * e);
    cnt[k] = __popc(nib[k]);
    reinterpret_cast<uint16_t *>(bitmap ? bitmap : buf)[128 * warp + 32 * k + lane] =
        uint16_t(nib[k]);
  }
  uint32_t q[4], total;
  ze_positions<NT>(cnt, red, q, total, data_base);
  if (data_base + total > uint32_t(kChunk)) {  // counts and data disagree: write nothing
    named_bar_sync(1, NT);
    return false;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t n = (nib[k] >> (4 * e)) & 0xFu;
      const uint32_t c = __byte_perm(x[k][e], 0, lut[n]), nb = __popc(n);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (uint32_t(i) < nb) buf[q[k] + i] = uint8_t(c >> (8 * i));
      q[k] += nb;
    }
  }
  named_bar_sync(1, NT);
  return true;
}

// Inverse: buf holds bitmap + nonzero bytes (`size` bytes); on return it
// holds the 16 KB chunk. Returns false (for every thread) if the bitmap's
// popcount disagrees with the size; then buf is unspecified. Each plane word
// takes the next popcount(n) source bytes (an unaligned 4-byte window) and
// spreads them with one byte permute.
template <int NT>
__device__ __forceinline__ bool ze_decode(uint8_t *buf, uint8_t *scr, uint32_t *red, uint32_t size,
                                          const uint8_t *bitmap = nullptr,
                                          uint32_t data_base = kBitmap) {
  static_assert(NT == 256, "eight warps of 512 plane words");
  __shared__ uint32_t lut[16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t *pw = reinterpret_cast<uint32_t *>(scr);
  if (tid < 16) lut[tid] = expand_selector(tid);
  uint32_t nib[4], cnt[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    nib[k] = reinterpret_cast<const uint16_t *>(bitmap ? bitmap : buf)[128 * warp + 32 * k + lane];
    cnt[k] = __popc(nib[k]);
  }
  uint32_t q[4], total;
  ze_positions<NT>(cnt, red, q, total, data_base);  // lut visible after its barrier
  if (total != size - data_base) {
    named_bar_sync(1, NT);  // red read by all before anyone reuses it
    return false;
  }
  // the window's words are clamped to the buffer: a byte it needs lies below
  // `size` <= 16384, so a clamped word is never one whose bytes are used
  const uint32_t *b32 = reinterpret_cast<const uint32_t *>(buf);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t o[4], p = q[k];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t n = (nib[k] >> (4 * e)) & 0xFu;
      const uint32_t a = min(p >> 2, 4095u), a1 = min((p >> 2) + 1, 4095u);
      const uint32_t win = __funnelshift_r(b32[a], b32[a1], 8 * (p & 3));
      o[e] = __byte_perm(win, 0, lut[n]);
      p += __popc(n);
    }
    *reinterpret_cast<uint4 *>(pw + pw_index(4 * warp + k, 4 * lane)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  named_bar_sync(1, NT);
  words_from_planes(pw, buf);
  named_bar_sync(1, NT);
  return true;
}

// ------------------------------------ composable pipelines (reading R17) --
// A stored chunk's pipeline id: bit 0 = the XOR of each word with the
// previous one, restarting every `run` words (32 vectors), before the
// bit-plane shuffle; bit 1 = the two-level form of zero-byte elimination
// (the 2048-byte bitmap reduced to a 256-byte map and its nonzero bytes).

// Forward XOR over the 4096 words of buf: w'[j] = w[j] ^ w[j - 1] unless j
// starts a run. Thread t (first 256) rewrites words 16t .. 16t+15.
template <int NT>
__device__ __forceinline__ void xor_runs_forward(uint8_t *buf, uint32_t run) {
  static_assert(NT == 256, "16 words per thread");
  uint32_t *w = reinterpret_cast<uint32_t *>(buf);
  const uint32_t t = threadIdx.x;
  uint32_t v[17];
  v[0] = t ? w[16 * t - 1] : 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 x = reinterpret_cast<const uint4 *>(w + 16 * t)[q];
    v[4 * q + 1] = x.x, v[4 * q + 2] = x.y, v[4 * q + 3] = x.z, v[4 * q + 4] = x.w;
  }
  named_bar_sync(1, NT);  // every thread has read its predecessor's last word
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = ((16 * t + i) % run) ? v[i + 1] ^ v[i] : v[i + 1];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    reinterpret_cast<uint4 *>(w + 16 * t)[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2],
                                                          o[4 * q + 3]);
  named_bar_sync(1, NT);
}

// Inverse: each word becomes the XOR of its run's words up to itself. A run
// of 32, 64 or 128 words spans 2, 4 or 8 consecutive threads (aligned in the
// warp), which exchange their partial XORs by shuffles.
template <int NT>
__device__ __forceinline__ void xor_runs_inverse(uint8_t *buf, uint32_t run) {
  static_assert(NT == 256, "16 words per thread");
  uint32_t *w = reinterpret_cast<uint32_t *>(buf);
  const uint32_t t = threadIdx.x, gs = run / 16, gl = t % gs;
  uint32_t p[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 x = reinterpret_cast<const uint4 *>(w + 16 * t)[q];
    p[4 * q] = x.x, p[4 * q + 1] = x.y, p[4 * q + 2] = x.z, p[4 * q + 3] = x.w;
  }
#pragma unroll
  for (int i = 1; i < 16; ++i) p[i] ^= p[i - 1];
  uint32_t incl = p[15];
#pragma unroll
  for (uint32_t o = 1; o < 8; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (o < gs && gl >= o) incl ^= y;
  }
  const uint32_t ex = incl ^ p[15];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    reinterpret_cast<uint4 *>(w + 16 * t)[q] =
        make_uint4(p[4 * q] ^ ex, p[4 * q + 1] ^ ex, p[4 * q + 2] ^ ex, p[4 * q + 3] ^ ex);
  named_bar_sync(1, NT);
}

// Two-level form, encode side: the 2048-byte bitmap in bm becomes, at the
// start of buf, a 256-byte map (bit i: bitmap byte i is nonzero) followed by
// the nonzero bitmap bytes in order. Returns their count (every thread).
template <int NT>
__device__ __forceinline__ uint32_t ze2_pack_bitmap(const uint8_t *bm, uint8_t *buf,
                                                    uint32_t *red) {
  static_assert(NT == 256, "8 bitmap bytes per thread");
  const uint32_t t = threadIdx.x;
  const uint2 v = *reinterpret_cast<const uint2 *>(bm + 8 * t);
  const uint32_t m = nz_nibble(v.x) | (nz_nibble(v.y) << 4);
  uint32_t total;
  const uint32_t ex = block_excl_scan<NT>(__popc(m), red, total);
  buf[t] = uint8_t(m);
  uint32_t pos = kBitmap2 + ex;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if ((m >> i) & 1u) buf[pos++] = uint8_t((i < 4 ? v.x : v.y) >> (8 * (i & 3)));
  named_bar_sync(1, NT);
  return total;
}

// Two-level form, decode side: expands the map and bitmap bytes at the start
// of buf into the 2048-byte bitmap bm. Returns the number of bitmap bytes
// (every thread); the caller checks it against the chunk's size.
template <int NT>
__device__ __forceinline__ uint32_t ze2_unpack_bitmap(const uint8_t *buf, uint8_t *bm,
                                                      uint32_t *red) {
  static_assert(NT == 256, "8 bitmap bytes per thread");
  const uint32_t t = threadIdx.x, m = buf[t];
  uint32_t total;
  const uint32_t ex = block_excl_scan<NT>(__popc(m), red, total);
  uint32_t pos = kBitmap2 + ex, lo = 0, hi = 0;  // pos < 256 + 2048 < 16384: inside buf
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if ((m >> i) & 1u) {
      const uint32_t b = buf[pos++];
      if (i < 4) lo |= b << (8 * i); else hi |= b << (8 * (i - 4));
    }
  }
  *reinterpret_cast<uint2 *>(bm + 8 * t) = make_uint2(lo, hi);
  named_bar_sync(1, NT);
  return total;
}

// A full chunk in buf through pipeline `pipe` into buf[0, size). run: words
// per 32 vectors; bnz: the nonzero bitmap bytes of the two-level form (from
// the encoder's counts; a mismatch records KVC_ERR_CORRUPT). bm: 2 KB.
template <int NT>
__device__ __forceinline__ void lossless_encode(uint8_t *buf, uint8_t *scr, uint8_t *bm,
                                                uint32_t *red, uint32_t pipe, uint32_t run,
                                                uint32_t bnz, uint32_t *status) {
  if (pipe & 1u) xor_runs_forward<NT>(buf, run);
  bool ok;
  if (pipe & 2u) {
    ok = ze_encode<NT>(buf, scr, red, bm, kBitmap2 + bnz) &&
         ze2_pack_bitmap<NT>(bm, buf, red) == bnz;
  } else {
    ok = ze_encode<NT>(buf, scr, red);
  }
  if (!ok && threadIdx.x == 0) set_status(status, KVC_ERR_CORRUPT);
}

// Inverse of any pipeline on a full chunk of `size` stored bytes in buf;
// false (every thread) if the chunk is inconsistent.
template <int NT>
__device__ __forceinline__ bool lossless_decode(uint8_t *buf, uint8_t *scr, uint8_t *bm,
                                                uint32_t *red, uint32_t size, uint32_t pipe,
                                                uint32_t run) {
  bool ok;
  if (pipe & 2u) {
    const uint32_t nb = ze2_unpack_bitmap<NT>(buf, bm, red);
    ok = kBitmap2 + nb <= size && ze_decode<NT>(buf, scr, red, size, bm, kBitmap2 + nb);
  } else {
    ok = size >= kBitmap && ze_decode<NT>(buf, scr, red, size);
  }
  if (ok && (pipe & 1u)) xor_runs_inverse<NT>(buf, run);
  return ok;
}

// ------------------------------------------- warp row blocks (32 rows) --
// A per-warp buffer of 32 rows in column blocks of 32 x 128 bytes (64 bf16
// channels, or 32 fp32), 16-byte piece c of row r at (c / 8) * 4096 +
// r * 128 + ((c % 8) ^ (r % 8)) * 16: the tensor maps' 128-byte swizzle, in
// which lane r reading its own row, or a group of lanes reading one row, hits
// distinct bank groups.
// HALF: bytes between column blocks (4096 for 32 rows; the paged encoder's
// buffers hold 40 rows, 5120).
template <int HALF = 4096>
__device__ __forceinline__ uint32_t swz_offset(int r, int c) {
  return uint32_t((c >> 3) * HALF + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Gathers the 32 rows whose global addresses the lanes hold (lane r: row r;
// null: zeros) into the buffer with 16-byte asynchronous copies. Each copy
// instruction covers D/8-lane groups, one whole row per group, so every
// group reads 2*D contiguous bytes. `dummy` is any valid global address
// (passed with zero-fill copies). Completion: cp_async_wait_all + __syncwarp.
template <int P, int HALF = 4096>  // 16-byte pieces per row: 8, 16 or 32
__device__ __forceinline__ void gather_rows_p(uint8_t *wbuf, const uint8_t *row, const void *dummy) {
  constexpr int RPI = 32 / P;  // rows per instruction
  const int lane = threadIdx.x & 31, c = lane % P, rs = lane / P;
  const uint64_t me = reinterpret_cast<uint64_t>(row);
#pragma unroll
  for (int i = 0; i < 32 / RPI; ++i) {
    const int r = i * RPI + rs;
    const uint64_t s = __shfl_sync(0xFFFFFFFFu, me, r);
    const void *src = s ? reinterpret_cast<const void *>(s + 16u * c) : dummy;
    cp_async16(wbuf + swz_offset<HALF>(r, c), src, s ? 16u : 0u);
  }
  cp_async_commit();
}

// The inverse move: the buffer's rows to the lanes' global addresses (null:
// not stored), one whole row per lane group and instruction. The caller
// orders the buffer's writes before it (__syncwarp); the buffer may be
// rewritten after a __syncwarp that follows it.
// Pieces are read eight rows' worth at a time before any of them is stored,
// so the shared loads are not held behind the global stores.
template <int P>
__device__ __forceinline__ void scatter_rows_p(const uint8_t *wbuf, uint8_t *row) {
  constexpr int RPI = 32 / P, N = 32 / RPI, B = 8;
  const int lane = threadIdx.x & 31, c = lane % P, rs = lane / P;
  const uint64_t me = reinterpret_cast<uint64_t>(row);
#pragma unroll
  for (int i0 = 0; i0 < N; i0 += B) {
    uint4 v[B];
    uint64_t d[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int r = (i0 + i) * RPI + rs;
      d[i] = __shfl_sync(0xFFFFFFFFu, me, r);
      v[i] = *reinterpret_cast<const uint4 *>(wbuf + swz_offset(r, c));
    }
#pragma unroll
    for (int i = 0; i < B; ++i)
      if (d[i]) *reinterpret_cast<uint4 *>(d[i] + 16u * c) = v[i];
  }
}

// The same two moves with each lane's row given as a 32-bit offset from
// `base` in 16-byte units (layouts whose rows all lie in [base, base + 64 GB)
// at non-negative offsets, flagged `narrow` by the host): one shuffle per row
// instead of two, and the swizzled shared-memory positions of a lane's pieces
// computed once per call. Piece c = lane % P of row r = i * RPI + lane / P is
// at swz_offset(r, c), whose bank term ((c ^ r) & 7) depends on i only
// through (i * RPI) & 7, so its K = 8 / RPI (at least 1) distinct addresses
// serve every i with a constant added.
__device__ __forceinline__ void cp_async16_s(uint32_t sdst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sdst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(saddr));
  return v;
}
template <int P, int HALF = 4096>
struct RowPieces {
  static constexpr int RPI = 32 / P;              // rows per copy instruction
  static constexpr int NI = 32 / RPI;             // instructions per 32 rows
  static constexpr int K = RPI >= 8 ? 1 : 8 / RPI;
  uint32_t s[K];
  int c, rs;
  __device__ __forceinline__ explicit RowPieces(const uint8_t *wbuf) {
    const int lane = threadIdx.x & 31;
    c = lane % P;
    rs = lane / P;
    const uint32_t sb = smem_u32(wbuf) + uint32_t((c >> 3) * HALF + rs * 128);
    const uint32_t k = uint32_t((c & 7) ^ (rs & 7));
#pragma unroll
    for (int j = 0; j < K; ++j) s[j] = sb + ((k ^ uint32_t((j * RPI) & 7)) << 4);
  }
  __device__ __forceinline__ uint32_t at(int i) const { return s[i % K] + uint32_t(i * RPI * 128); }
};
// Lanes without a row pass offset 0 (their row reads base's first row,
// which is not used).
template <int P, int HALF = 4096>
__device__ __forceinline__ void gather_rows_narrow(uint8_t *wbuf, const uint8_t *base,
                                                   uint32_t off16) {
  const RowPieces<P, HALF> rp(wbuf);
  const uint8_t *g = base + 16 * rp.c;
#pragma unroll
  for (int i = 0; i < RowPieces<P, HALF>::NI; ++i) {
    const uint32_t o = __shfl_sync(0xFFFFFFFFu, off16, i * RowPieces<P, HALF>::RPI + rp.rs);
    cp_async16_s(rp.at(i), g + uint64_t(o) * 16);
  }
  cp_async_commit();
}
// Lanes without a row pass ~0u (nothing is stored for them).
template <int P>
__device__ __forceinline__ void scatter_rows_narrow(const uint8_t *wbuf, uint8_t *base,
                                                    uint32_t off16) {
  constexpr int N = RowPieces<P>::NI, B = 8;
  const RowPieces<P> rp(wbuf);
  uint8_t *g = base + 16 * rp.c;
#pragma unroll
  for (int i0 = 0; i0 < N; i0 += B) {
    uint4 v[B];
    uint32_t d[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      d[i] = __shfl_sync(0xFFFFFFFFu, off16, (i0 + i) * RowPieces<P>::RPI + rp.rs);
      v[i] = lds128(rp.at(i0 + i));
    }
#pragma unroll
    for (int i = 0; i < B; ++i)
      if (d[i] != ~0u) *reinterpret_cast<uint4 *>(g + uint64_t(d[i]) * 16) = v[i];
  }
}

// Rows of D bf16 (2*D bytes, D/8 pieces).
template <int D, int HALF = 4096>
__device__ __forceinline__ void gather_rows(uint8_t *wbuf, const uint8_t *row, const void *dummy) {
  gather_rows_p<D / 8, HALF>(wbuf, row, dummy);
}
template <int D>
__device__ __forceinline__ void scatter_rows(const uint8_t *wbuf, uint8_t *row) {
  scatter_rows_p<D / 8>(wbuf, row);
}

// --------------------------------------------------------- addressing --
// Dense: v = ((l*2 + kv)*H + h)*T + t.
__device__ __forceinline__ uint8_t *vec_addr(const DenseLayout &L, const uint32_t *,
                                             uint32_t v, bool &ok) {
  const uint32_t lkh = fdiv(L.T, v), t = v - lkh * L.T.d;
  const uint32_t lk = fdiv(L.H, lkh), h = lkh - lk * L.H.d;
  ok = true;
  return L.base + int64_t(lk >> 1) * L.s_l + int64_t(lk & 1u) * L.s_kv + int64_t(h) * L.s_h +
         int64_t(t) * L.s_t;
}
// Paged: v = ((l*2 + kv)*H + h)*Ttot + cum[r] + t; page from the page table.
__device__ __forceinline__ uint8_t *vec_addr(const PagedLayout &L, const uint32_t *cum,
                                             uint32_t v, bool &ok) {
  const uint32_t lkh = fdiv(L.T, v), u = v - lkh * L.T.d;
  const uint32_t lk = fdiv(L.H, lkh), h = lkh - lk * L.H.d;
  uint32_t lo = 0, hi = L.n_req - 1;  // largest r with cum[r] <= u
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  const uint32_t t = u - cum[lo];
  const uint32_t pi = fdiv(L.PT, t), slot = t - pi * L.PT.d;
  const int32_t page = __ldg(L.page_table + int64_t(lo) * L.pt_stride + pi);
  ok = page >= 0 && int64_t(page) < L.num_pages;
  return L.base + int64_t(lk >> 1) * L.s_l + int64_t(page) * L.s_p + int64_t(lk & 1u) * L.s_kv +
         int64_t(h) * L.s_h + int64_t(slot) * L.s_slot;
}

}  // namespace kvc
