// Main encode kernel: load/gather -> signs -> fp32 Walsh-Hadamard -> group
// min/max -> fp16 meta -> quantize -> pack -> lossless decision for the code
// chunk (bit-plane shuffle + zero-byte elimination when it pays) -> the code
// chunk goes straight to its raw-layout position in the stream, the meta
// slice to the workspace. The transformed tensor and the raw payload never
// reach HBM (the fusion of "Beyond Compression Ratio: High-Throughput KV
// Compression for Disaggregated LLM Serving", Abstract: transform and
// quantization in one kernel with no intermediate tensor; an LC-style
// lossless backend of composable primitives).
//
// The stream holds every code chunk before every meta chunk, so a code
// chunk's final offset is c * 16 KB whenever no earlier code chunk shrank;
// the finishing kernel (kvc_finish.cuh) writes the table, the meta chunks and
// the header, and moves code chunks only in the case that one shrank. This
// kernel therefore has no dependency between CTAs: each CTA takes tiles
// (one tile = one 16 KB code chunk) blockIdx.x, + gridDim.x, ...
//
// CTA = 8 warps, one head_dim vector per thread held in registers. Each
// thread issues the bulk-async copy of its own vector row (dense, or paged
// through the page table) into a padded shared-memory stage, two units of
// 256 rows in flight ahead of the computation.
#pragma once

#include <type_traits>

#include "kvc_device.cuh"

namespace kvc {

constexpr int kEncThreads = 256;  // one vector per thread
constexpr int kEncStages = 2;

template <int D, int BITS, int G, int NT = kEncThreads>
struct Cfg {
  static constexpr int ROW = D * 2;              // bytes of one bf16 vector
  static constexpr int ROWP = ROW + 16;          // padded smem row (no bank conflicts)
  static constexpr int CB = D * BITS / 8;        // code bytes per vector
  static constexpr int CW = CB / 4;              // code words per vector
  static constexpr int NG = D / G;               // groups per vector
  static constexpr int MB = NG * 4;              // meta bytes per vector
  static constexpr int VC = kChunk / CB;         // vectors per code chunk
  static constexpr int R = G * BITS / 32;        // code chunks per meta chunk
  static constexpr int VM = VC * R;              // vectors per meta chunk
  static constexpr int NSUB = VC / NT;           // units of NT vectors per tile
  static constexpr int SLICE = VC * MB;          // meta bytes per tile
  static constexpr int LOG2D = D == 64 ? 6 : D == 128 ? 7 : 8;
  static constexpr int K = LOG2D / 2;            // meta stored x 2^-K
  static constexpr int QMAX = (1 << BITS) - 1;
  static_assert(NSUB >= 1 && VC % NT == 0, "unit size");
  static_assert(R >= 2 && R <= 16, "segment size");
  static_assert(SLICE % 32 == 0, "meta slices hold whole 8-word groups");
};

struct EncCtl {
  uint64_t full[kEncStages];  // stage filled (kEncThreads arrivals + bytes)
  uint32_t red[kEncThreads / 32];
};

template <int D, int BITS, int G>
constexpr size_t enc_smem_bytes(bool paged) {
  using C = Cfg<D, BITS, G>;
  return size_t(kEncStages) * kEncThreads * C::ROWP + 3 * size_t(kChunk) + 2 * size_t(C::SLICE) +
         sizeof(EncCtl) + (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
}

template <class L>
constexpr bool kIsPaged = std::is_same<L, PagedLayout>::value;

// ------------------------------------------------------------------------
// One vector: shared-memory row in, codes + meta out. Scalar fp32 (on
// sm_100a the paired f32x2 ops have lower element throughput than scalar
// FADD, and a paired multiply followed by a paired add may be fused).
// ------------------------------------------------------------------------
template <int D, int BITS, int G>
struct Enc : Cfg<D, BITS, G> {
  using C = Cfg<D, BITS, G>;

  // E1/E2: widen bf16 exactly and flip the sign bit of negative channels.
  static __device__ __forceinline__ void unpack(const uint8_t *row, const uint32_t *__restrict__ mask,
                                                float (&y)[D]) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
      const uint4 v = r4[q];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * q + e;
        const uint32_t a = w[e] ^ mask[j];
        y[2 * j] = __uint_as_float(a << 16);
        y[2 * j + 1] = __uint_as_float(a & 0xFFFF0000u);
      }
    }
  }

  // Group minimum / maximum by pairwise trees (exact, order-free), NaN
  // propagating so a non-finite group is always seen.
  static __device__ __forceinline__ void minmax(const float (&y)[D], int g, float &mn, float &mx) {
    float lo[G / 4], hi[G / 4];
#pragma unroll
    for (int i = 0; i < G / 4; ++i) {
      const int c = g * G + 4 * i;
      lo[i] = min3n(y[c], y[c + 1], min2n(y[c + 2], y[c + 3]));
      hi[i] = max3n(y[c], y[c + 1], max2n(y[c + 2], y[c + 3]));
    }
#pragma unroll
    for (int n = G / 8; n >= 1; n /= 2) {  // G/4 is a power of two
#pragma unroll
      for (int i = 0; i < n; ++i) {
        lo[i] = min2n(lo[2 * i], lo[2 * i + 1]);
        hi[i] = max2n(hi[2 * i], hi[2 * i + 1]);
      }
    }
    mn = lo[0];
    mx = hi[0];
  }

  // E3..E7 on y (transformed in place). Reading R5: asymmetric min/max group
  // quantization, fp16 zero (round down) and scale (round up), both x 2^-K.
  static __device__ __forceinline__ uint32_t vector(float (&y)[D], uint32_t (&code)[C::CW],
                                                    uint32_t (&meta)[C::NG]) {
    fwht<D>(y);
    uint32_t err = 0;
    float zf[C::NG], rr[C::NG];
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      float mn, mx;
      minmax(y, g, mn, mx);
      mn = __fadd_rn(mn, 0.0f);  // -0 -> +0
      mx = __fadd_rn(mx, 0.0f);
      if (!(isfinite(mn) && isfinite(mx))) err |= 1u;
      const float down = 1.0f / float(1 << C::K), up = float(1 << C::K);
      const __half zh = __float2half_rd(__fmul_rn(mn, down));
      zf[g] = __fmul_rn(__half2float(zh), up);
      const float s32 = __fdiv_rn(__fsub_rn(mx, zf[g]), float(C::QMAX));
      const __half sh = __float2half_ru(__fmul_rn(s32, down));
      const float sf = __fmul_rn(__half2float(sh), up);
      const uint16_t zb = __half_as_ushort(zh), sb = __half_as_ushort(sh);
      if ((zb & 0x7FFFu) == 0x7C00u || (sb & 0x7FFFu) == 0x7C00u) err |= 2u;
      rr[g] = ((sb & 0x7FFFu) == 0) ? 0.0f : __frcp_rn(sf);
      meta[g] = uint32_t(sb) | (uint32_t(zb) << 16);
    }
    // E6/E7, one code word at a time: q = RNE(fl(fl(y - zf) * r)); adding
    // 1.5*2^23 (a separate rounding: __fmul_rn is never fused into a
    // multiply-add) leaves q in the low bits. The clamp to [0, 2^b - 1] never
    // acts for a finite group: y - zf >= 0 since zf <= min, and sf >=
    // (max - zf)/(2^b - 1) keeps the product below 2^b - 1 + 2^-20. Codes
    // pack LSB first in channel order (reading R6).
    constexpr float kMagic = 12582912.0f;
    constexpr int per = 8 / BITS;  // codes per byte
#pragma unroll
    for (int W = 0; W < C::CW; ++W) {
      uint32_t b[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < per; ++e) {
          const int c = (W * 4 + k) * per + e, g = c / G;
          const float t = __fmul_rn(__fsub_rn(y[c], zf[g]), rr[g]);
          acc += __float_as_uint(__fadd_rn(t, kMagic)) << (e * BITS);
        }
        b[k] = acc;
      }
      code[W] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    }
    return err;
  }
};

// ------------------------------------------------------------------------
// Once per tile (all threads): raw / zero-byte decision for the code chunk,
// the meta slice's shuffled-byte count, then thread 0 stores both.
// ------------------------------------------------------------------------
template <int D, int BITS, int G>
__device__ __forceinline__ void finalize_tile(const EncArgs &a, EncCtl *ctl, uint32_t tile,
                                              uint32_t nvec, uint32_t nnz, uint8_t *cslot,
                                              uint8_t *mslot, uint8_t *s_scr) {
  using C = Cfg<D, BITS, G>;
  constexpr int NT = kEncThreads;
  const int tid = threadIdx.x;
  const uint32_t total_nnz = block_sum<NT>(nnz, ctl->red);
  const uint32_t code_len = nvec * C::CB;
  uint32_t code_size = code_len;
  if (code_len == kChunk && kBitmap + total_nnz < kChunk) {
    ze_encode<NT>(cslot, s_scr, ctl->red);
    code_size = kBitmap + total_nnz;
    for (uint32_t b = code_size + tid; b < round16(code_size); b += NT) cslot[b] = 0;
  }
  // The meta chunk's shuffled-byte count is the sum over its slices (each
  // slice holds whole 8-word groups); it decides the meta chunk's storage.
  const uint32_t slice_bytes = nvec * C::MB;
  uint32_t part = 0;
  for (uint32_t gi = tid; gi < slice_bytes / 32; gi += NT) {
    const uint4 *s = reinterpret_cast<const uint4 *>(mslot + gi * 32);
    const uint4 x = s[0], y = s[1];
    part += __popc(x.x | x.y | x.z | x.w | y.x | y.y | y.z | y.w);
  }
  const uint32_t meta_nnz = block_sum<NT>(part, ctl->red);
  fence_proxy_async_smem();
  named_bar_sync(1, NT);
  if (tid == 0) {
    bulk_s2g(a.out + a.data_base + uint64_t(tile) * kChunk, cslot, uint32_t(round16(code_size)));
    bulk_s2g(a.ws_meta + uint64_t(tile) * C::SLICE, mslot, uint32_t(round16(slice_bytes)));
    bulk_commit();
    a.code_size[tile] = code_size;
    atomicAdd(a.meta_nnz + tile / C::R, meta_nnz);
    if (code_size != code_len) atomicOr(a.flags, 1u);
  }
}

// ------------------------------------------------------------------------
// The kernel.
// ------------------------------------------------------------------------
template <int D, int BITS, int G, class Layout>
__global__ void __launch_bounds__(kEncThreads, 1)
    encode_kernel(const __grid_constant__ EncArgs a, const __grid_constant__ Layout lay) {
  using C = Cfg<D, BITS, G>;
  using E = Enc<D, BITS, G>;
  constexpr int NT = kEncThreads;
  constexpr bool kPaged = kIsPaged<Layout>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *s_in = smem;
  uint8_t *s_code = s_in + kEncStages * NT * C::ROWP;
  uint8_t *s_scr = s_code + 2 * kChunk;
  uint8_t *s_meta = s_scr + kChunk;
  EncCtl *ctl = reinterpret_cast<EncCtl *>(s_meta + 2 * C::SLICE);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(ctl + 1);
  const int tid = threadIdx.x;

  if (tid == 0) {
    for (int i = 0; i < kEncStages; ++i) mbar_init(&ctl->full[i], NT);
    mbar_fence_init();
  }
  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
  }
  __syncthreads();

  const uint32_t grid = gridDim.x, n_tiles = a.n_tiles;
  const uint32_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + grid - 1) / grid : 0;
  const uint32_t n_units = my_tiles * C::NSUB;

  // Each thread copies its own row of unit u (tile blockIdx.x + k*grid).
  auto issue = [&](uint32_t u) {
    const int stage = u % kEncStages;
    uint64_t *bar = &ctl->full[stage];
    const uint32_t tile = blockIdx.x + (u / C::NSUB) * grid;
    const uint32_t j = (u % C::NSUB) * NT + tid;
    const uint32_t nvec = min(uint32_t(C::VC), a.V - tile * C::VC);
    if (j < nvec) {
      bool ok;
      const uint8_t *src = vec_addr(lay, s_cum, tile * C::VC + j, ok);
      if (ok) {
        mbar_arrive_expect_tx(bar, C::ROW);
        bulk_g2s(s_in + (stage * NT + tid) * C::ROWP, src, C::ROW, bar);
        return;
      }
      set_status(a.status, KVC_ERR_CORRUPT);
    }
    mbar_arrive(bar);
  };
  for (uint32_t u = 0; u < kEncStages && u < n_units; ++u) issue(u);

  uint32_t nnz = 0, err = 0;
#pragma unroll 1
  for (uint32_t u = 0; u < n_units; ++u) {
    const int stage = u % kEncStages;
    const uint32_t k = u / C::NSUB, sub = u % C::NSUB;
    const uint32_t tile = blockIdx.x + k * grid, slot = k & 1;
    // The stores of tile k-2 (same slot) must have read the slot (thread 0
    // owns the bulk groups; the barrier below publishes the wait).
    if (sub == 0 && k >= 2 && tid == 0) bulk_wait_read<1>();
    if (!mbar_wait(&ctl->full[stage], (u / kEncStages) & 1, a.status))
      set_status(a.status, KVC_ERR_TIMEOUT);
    const uint32_t nvec = min(uint32_t(C::VC), a.V - tile * C::VC);
    const uint32_t j = sub * NT + tid;
    const bool valid = j < nvec;
    float yv[D];
    if (valid) E::unpack(s_in + (stage * NT + tid) * C::ROWP, a.sign_mask, yv);
    named_bar_sync(1, NT);  // stage read by every thread; slot free
    if (u + kEncStages < n_units) issue(u + kEncStages);

    uint8_t *cslot = s_code + slot * kChunk;
    uint8_t *mslot = s_meta + slot * C::SLICE;
    uint32_t code[C::CW] = {};
    if (valid) {
      uint32_t meta[C::NG];
      err |= E::vector(yv, code, meta);
      uint4 *cd = reinterpret_cast<uint4 *>(cslot + j * C::CB);
#pragma unroll
      for (int q = 0; q < C::CW / 4; ++q)
        cd[q] = make_uint4(code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
      uint32_t *md = reinterpret_cast<uint32_t *>(mslot + j * C::MB);
      if constexpr (C::NG == 1) {
        md[0] = meta[0];
      } else if constexpr (C::NG == 2) {
        *reinterpret_cast<uint2 *>(md) = make_uint2(meta[0], meta[1]);
      } else {
        *reinterpret_cast<uint4 *>(md) = make_uint4(meta[0], meta[1], meta[2], meta[3]);
      }
    }
    {  // shuffled-byte count of this vector's 8-word groups (see chunk_nnz_part)
      uint32_t orv[(C::CW + 7) / 8] = {};
#pragma unroll
      for (int W = 0; W < C::CW; ++W) orv[W / 8] |= code[W];
      if constexpr (C::CW >= 8) {
#pragma unroll
        for (int q = 0; q < C::CW / 8; ++q) nnz += __popc(orv[q]);
      } else {
        const uint32_t o = orv[0] | __shfl_xor_sync(0xFFFFFFFFu, orv[0], 1);
        if ((tid & 1) == 0) nnz += __popc(o);
      }
    }
    if (sub == C::NSUB - 1) {
      finalize_tile<D, BITS, G>(a, ctl, tile, nvec, nnz, cslot, mslot, s_scr);
      nnz = 0;
    }
  }
  if (err & 1u) set_status(a.status, KVC_ERR_NONFINITE);
  if (err & 2u) set_status(a.status, KVC_ERR_RANGE);
  if (tid == 0) bulk_wait_all<0>();
}

}  // namespace kvc
