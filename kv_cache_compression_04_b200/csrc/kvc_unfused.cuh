// Unfused baseline of the encode step, kept for measurement: the same
// arithmetic as encode_kernel split into two kernels with the transformed
// tensor in HBM between them (fp32, 4*d bytes per vector) -- the separate
// transform and quantization kernels whose intermediate tensor the fused
// kernel avoids ("Beyond Compression Ratio: High-Throughput KV Compression for
// Disaggregated LLM Serving", Abstract: fusing the randomized Hadamard
// transform with quantization removes the full-size intermediate). The stream
// it produces is the fused path's, byte for byte.
#pragma once

#include "kvc_encode.cuh"

namespace kvc {

// Shared memory: per-warp buffers of 32 fp32 rows (16 KB at d = 128; the
// first (d/64) * 4 KB also take the bf16 input rows) | per-warp mbarriers |
// request prefix (paged).
template <int D>
struct UnfSmem {
  static constexpr size_t WBUF = size_t(D) * 4 * 32;
  static constexpr size_t wbars = kEncWarps * WBUF;
  static constexpr size_t cum = wbars + kEncWarps * 8;
  static_assert(WBUF % 1024 == 0, "swizzled buffers stay 1024-byte aligned");
};
template <int D>
constexpr size_t unf_smem_bytes(bool paged) {
  return UnfSmem<D>::cum + (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
}

// Kernel 1: E1..E3. Vector v's transformed values go to ymid + v * d (fp32,
// channel order), staged per warp and stored with 16-byte stores, one
// 4*d-byte row per warp instruction (d = 128).
template <int D, class Layout>
__global__ void __launch_bounds__(kEncThreads, 1)
    transform_kernel(const __grid_constant__ EncArgs a, const __grid_constant__ Layout lay) {
  using E = Enc<D, 4, D>;  // unpack only (bits and group do not enter it)
  constexpr bool kPaged = kIsPaged<Layout>;
  using S = UnfSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t *wbuf = smem + warp * S::WBUF;
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem + S::wbars) + warp;
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(smem + S::cum);
  if (lane == 0) {
    mbar_init(wbar, 1);
    mbar_fence_init();
  }
  __syncwarp();
  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
    __syncthreads();
  }
  const uint32_t V = a.V;
  const uint32_t n_blocks = (V + 31) / 32;
  const uint32_t stride = gridDim.x * kEncWarps;
  bool use_tma = false;
  if constexpr (!kPaged) use_tma = lay.tma != 0;
  uint32_t phase = 0;
#pragma unroll 1
  for (uint32_t blk = blockIdx.x * kEncWarps + warp; blk < n_blocks; blk += stride) {
    const uint32_t v = blk * 32 + lane;
    // rows of the block into the buffer (the previous block's stores have
    // read it: the warp synchronized after them)
    if (use_tma) {
      if constexpr (!kPaged) {
        if (lane == 0) {
          const uint32_t v0 = blk * 32, lkh = fdiv(lay.T, v0), t0 = v0 - lkh * lay.T.d;
          const uint32_t lk = fdiv(lay.H, lkh), h = lkh - lk * lay.H.d;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(wbar, uint32_t(D / 64) * 4096);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(wbuf + hh * 4096, &lay.tmap, hh * 64, int(t0), int(h), int(lk & 1u),
                        int(lk >> 1), wbar);
        }
        if (!mbar_wait(wbar, phase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
        phase ^= 1;
      }
    } else {
      const uint8_t *src = nullptr;
      if (v < V) {
        bool ok;
        src = vec_addr(lay, s_cum, v, ok);
        if (!ok) {
          set_status(a.status, KVC_ERR_CORRUPT);
          src = nullptr;
        }
      }
      gather_rows<D>(wbuf, src, a.out);
      cp_async_wait_all();
      __syncwarp();
    }
    Pairs<D> y;
    E::unpack_swz(wbuf, lane, GlobalSigns{a.sign_mask, a.sign_lo}, y);
    fwht_pairs<D>(y);
    __syncwarp();  // every lane has read its input row
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {  // piece c: channels 4c .. 4c + 3
      const int j = 4 * (c % (D / 8));
      const bool hi = c >= D / 8;
      *reinterpret_cast<float4 *>(wbuf + swz_offset(lane, c)) =
          hi ? make_float4(y.p[j].y, y.p[j + 1].y, y.p[j + 2].y, y.p[j + 3].y)
             : make_float4(y.p[j].x, y.p[j + 1].x, y.p[j + 2].x, y.p[j + 3].x);
    }
    __syncwarp();
    scatter_rows_p<D / 4>(wbuf, v < V ? reinterpret_cast<uint8_t *>(a.ymid + uint64_t(v) * D)
                                      : nullptr);
    __syncwarp();  // the stores have read the buffer
  }
}

// Kernel 2: E4..E7 from the transformed tensor, then the fused kernel's
// stores and counts (encode_finish_block). Rows are gathered one block ahead.
template <int D, int BITS, int G>
__global__ void __launch_bounds__(kEncThreads, 1) quantize_kernel(const __grid_constant__ EncArgs a) {
  using S = UnfSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t *wbuf = smem + warp * S::WBUF;
  const uint32_t V = a.V;
  const uint32_t n_blocks = (V + 31) / 32;
  const uint32_t stride = gridDim.x * kEncWarps;
  uint32_t blk = blockIdx.x * kEncWarps + warp, err = 0;
  auto row = [&](uint32_t v) -> const uint8_t * {
    return v < V ? reinterpret_cast<const uint8_t *>(a.ymid + uint64_t(v) * D) : nullptr;
  };
  if (blk < n_blocks) gather_rows_p<D / 4>(wbuf, row(blk * 32 + lane), a.out);
#pragma unroll 1
  for (; blk < n_blocks; blk += stride) {
    const uint32_t v = blk * 32 + lane;
    cp_async_wait_all();
    __syncwarp();
    Pairs<D> y;
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
      const float4 lo = *reinterpret_cast<const float4 *>(wbuf + swz_offset(lane, q));
      const float4 hi = *reinterpret_cast<const float4 *>(wbuf + swz_offset(lane, q + D / 8));
      y.p[4 * q] = make_float2(lo.x, hi.x);
      y.p[4 * q + 1] = make_float2(lo.y, hi.y);
      y.p[4 * q + 2] = make_float2(lo.z, hi.z);
      y.p[4 * q + 3] = make_float2(lo.w, hi.w);
    }
    __syncwarp();
    if (blk + stride < n_blocks) gather_rows_p<D / 4>(wbuf, row((blk + stride) * 32 + lane), a.out);
    encode_finish_block<D, BITS, G, false, false>(a, blk, v, v < V, y, err);
  }
  err = __reduce_or_sync(0xFFFFFFFFu, err);
  if (lane == 0) {
    if (err & 1u) set_status(a.status, KVC_ERR_NONFINITE);
    if (err & 2u) set_status(a.status, KVC_ERR_RANGE);
  }
}

}  // namespace kvc
