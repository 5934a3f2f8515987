// Launch helpers shared by the per-head_dim translation units.
#pragma once

#include <atomic>
#include <utility>

#include "kvc_decode.cuh"

namespace kvc {

// Launches kernel k so that it may begin while the previous kernel on the
// stream finishes (programmatic dependent launch); k must start with
// grid_dependency_wait().
template <class... KArgs, class... Args>
inline cudaError_t launch_after(void (*k)(KArgs...), int grid, int threads, size_t smem,
                                cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(unsigned(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kernel_timing().events ? 0 : 1;  // timed calls: plain stream order
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
  timing_mark(st);
  return e;
}

// launch_after without the timing mark: the kernel's time is counted in the
// interval of the launch that follows it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_after_unmarked(void (*k)(KArgs...), int grid, int threads, size_t smem,
                                         cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(unsigned(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kernel_timing().events ? 0 : 1;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// Opt each instantiation into large dynamic shared memory once per device.
// `Tag` makes the flag per kernel instantiation (kernels share a pointer type).
template <class Tag, class Kernel>
inline cudaError_t prepare(Kernel k, size_t smem) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int D, int BITS, int G, class Layout, bool kNarrow, bool kSearch, int kVar>
cudaError_t launch_enc_k(const EncArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  auto k = encode_kernel<D, BITS, G, Layout, kNarrow, kSearch, kVar>;
  const size_t smem = enc_smem_bytes<D>(kIsPaged<Layout>);
  struct Tag {};
  cudaError_t e = prepare<Tag>(k, smem);
  if (e != cudaSuccess) return e;
  // one CTA per SM; warps take blocks of 32 vectors round-robin
  const uint32_t n_blocks = (a.V + 31) / 32;
  const uint32_t want = (n_blocks + kEncWarps - 1) / kEncWarps;
  const int grid = int(want < uint32_t(sms) ? want : uint32_t(sms));
  if constexpr (kIsPaged<Layout>) {
    // the blocks' load plans, a dependent launch after the workspace clear
    // whose time counts in the encode interval
    if (lay.tma && n_blocks > 1) {
      const uint32_t pw = (n_blocks - 1 + 255) / 256, pcap = uint32_t(sms) * 16;
      e = launch_after_unmarked(paged_plan_kernel<D>, int(pw < pcap ? pw : pcap), 256, 0, st, a,
                                lay, uint32_t(32 * Cfg<D, BITS, G>::MB));
      if (e != cudaSuccess) return e;
    }
  }
  // a dependent launch after the workspace clear (or the plans): see
  // encode_kernel
  return launch_after(k, grid, kEncThreads, smem, st, a, lay);
}
// Paged rows named by 32-bit offsets when the pool allows (narrow row
// copies). Dense inputs keep the 64-bit gather next to their tensor-map
// loads: both paths in one kernel would not fit its registers.
// The search mode counts more per block (encode_finish_block's kSearch).
template <int D, int BITS, int G, class Layout, bool kSearch, int kVar>
cudaError_t launch_enc_s(const EncArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  if constexpr (kIsPaged<Layout>) {
    if (lay.narrow) return launch_enc_k<D, BITS, G, Layout, true, kSearch, kVar>(a, lay, sms, st);
  }
  return launch_enc_k<D, BITS, G, Layout, false, kSearch, kVar>(a, lay, sms, st);
}
template <int D, int BITS, int G, class Layout, int kVar>
cudaError_t launch_enc(const EncArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  return a.mode == KVC_LOSSLESS_SEARCH
             ? launch_enc_s<D, BITS, G, Layout, true, kVar>(a, lay, sms, st)
             : launch_enc_s<D, BITS, G, Layout, false, kVar>(a, lay, sms, st);
}

template <int D, class Layout, bool kNarrow>
cudaError_t prepare_dec(const size_t smem) {
  struct Tag {};
  return prepare<Tag>(decode_kernel<D, Layout, kNarrow>, smem);
}

template <int D, class Layout>
cudaError_t launch_dec(const DecArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  // rows named by 32-bit offsets when the layout allows (narrow row copies)
  auto k = lay.narrow ? decode_kernel<D, Layout, true> : decode_kernel<D, Layout, false>;
  const size_t smem = DecSmem<D>::bytes(kIsPaged<Layout>);
  cudaError_t e = lay.narrow ? prepare_dec<D, Layout, true>(smem)
                             : prepare_dec<D, Layout, false>(smem);
  if (e != cudaSuccess) return e;
  // one CTA per SM; tiles are the code chunks (at least 128 vectors each)
  const uint64_t min_vc = uint64_t(kChunk) / (uint64_t(D) * 4 / 8);
  const uint64_t tiles = (uint64_t(a.V) + min_vc - 1) / min_vc;
  const int grid = tiles == 0 ? 1 : int(tiles < uint64_t(sms) ? tiles : uint64_t(sms));
  // pre-pass: expand zero-byte-eliminated meta chunks into the workspace
  auto mk = meta_expand_kernel<D>;
  struct MetaTag {};
  e = prepare<MetaTag>(mk, meta_smem_bytes());
  if (e != cudaSuccess) return e;
  const uint32_t mcap = uint32_t(kMetaCtas) * uint32_t(sms);
  const int mgrid = int(a.ws_meta_chunks == 0 ? 1u : (a.ws_meta_chunks < mcap ? a.ws_meta_chunks : mcap));
  e = launch_after(mk, mgrid, kMetaThreads, meta_smem_bytes(), st, a);  // after the status clear
  if (e != cudaSuccess) return e;
  // code chunks that used zero-byte elimination (returns at once if none);
  // 256 chunks per CTA and scan step, for the largest code region (4-bit)
  auto ek = elim_decode_kernel<D, Layout>;
  const size_t esmem = ElimSmem<D>::bytes(kIsPaged<Layout>);
  struct ElimTag {};
  e = prepare<ElimTag>(ek, esmem);
  if (e != cudaSuccess) return e;
  const uint64_t egrid_want = (tiles + kElimThreads - 1) / kElimThreads;
  const int egrid = egrid_want == 0 ? 1 : int(egrid_want < uint64_t(sms) ? egrid_want : uint64_t(sms));
  // The elimination kernel (which usually returns at once) is a dependent
  // launch; the decode kernel is not (as a dependent launch it measured
  // slower when compress and decompress calls alternate on a stream).
  e = launch_after(ek, egrid, kElimThreads, esmem, st, a, lay);
  if (e != cudaSuccess) return e;
  k<<<grid, kDecThreads, smem, st>>>(a, lay);
  timing_mark(st);
  return cudaGetLastError();
}

// The encode kernel for `group` at fixed head_dim and bits.
template <int D, int BITS, int kVar, class Layout>
cudaError_t launch_enc_g(int group, const EncArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  if constexpr (D == 128) {
    if (group == 128) return launch_enc<D, BITS, 128, Layout, kVar>(a, lay, sms, st);
  }
  if (group == 64) return launch_enc<D, BITS, 64, Layout, kVar>(a, lay, sms, st);
  if (group == 32) return launch_enc<D, BITS, 32, Layout, kVar>(a, lay, sms, st);
  return cudaErrorInvalidValue;
}

// 2- and 4-bit codes of the min/max and absmax quantizers with the global
// sign diagonal here; 8-bit codes, per-vector diagonals and the FP4
// quantizer in the `_var` launchers (their own translation units).
template <int D, class Layout, class Var>
cudaError_t launch_enc_dispatch(int bits, int group, const EncArgs &a, const Layout &lay, int sms,
                                cudaStream_t st, Var var) {
  if (a.vec_signs || a.fp4 || bits == 8) return var(bits, group, a, lay, sms, st);
  if (bits == 4) return launch_enc_g<D, 4, 0>(group, a, lay, sms, st);
  if (bits == 2) return launch_enc_g<D, 2, 0>(group, a, lay, sms, st);
  return cudaErrorInvalidValue;
}
template <int D, class Layout>
cudaError_t launch_enc_dispatch_var(int bits, int group, const EncArgs &a, const Layout &lay,
                                    int sms, cudaStream_t st) {
  if (a.fp4) {
    if (bits != 4) return cudaErrorInvalidValue;
    return a.vec_signs ? launch_enc_g<D, 4, 3>(group, a, lay, sms, st)
                       : launch_enc_g<D, 4, 2>(group, a, lay, sms, st);
  }
  if (!a.vec_signs)
    return bits == 8 ? launch_enc_g<D, 8, 0>(group, a, lay, sms, st) : cudaErrorInvalidValue;
  if (bits == 8) return launch_enc_g<D, 8, 1>(group, a, lay, sms, st);
  if (bits == 4) return launch_enc_g<D, 4, 1>(group, a, lay, sms, st);
  if (bits == 2) return launch_enc_g<D, 2, 1>(group, a, lay, sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace kvc
