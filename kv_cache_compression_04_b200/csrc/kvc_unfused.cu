// Launches of the unfused baseline (transform kernel, quantize kernel).
#include "kvc_launch.cuh"
#include "kvc_unfused.cuh"

namespace kvc {

namespace {

int enc_grid(const EncArgs &a, int sms) {
  const uint32_t n_blocks = (a.V + 31) / 32;
  const uint32_t want = (n_blocks + kEncWarps - 1) / kEncWarps;
  return int(want < uint32_t(sms) ? (want ? want : 1u) : uint32_t(sms));
}

template <int D, class Layout>
cudaError_t launch_tf(const EncArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  auto k = transform_kernel<D, Layout>;
  const size_t smem = unf_smem_bytes<D>(kIsPaged<Layout>);
  struct Tag {};
  cudaError_t e = prepare<Tag>(k, smem);
  if (e != cudaSuccess) return e;
  k<<<enc_grid(a, sms), kEncThreads, smem, st>>>(a, lay);
  return cudaGetLastError();
}

template <int D, int BITS, int G>
cudaError_t launch_q(const EncArgs &a, int sms, cudaStream_t st) {
  auto k = quantize_kernel<D, BITS, G>;
  const size_t smem = unf_smem_bytes<D>(false);
  struct Tag {};
  cudaError_t e = prepare<Tag>(k, smem);
  if (e != cudaSuccess) return e;
  k<<<enc_grid(a, sms), kEncThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_transform_dense(int d, const EncArgs &a, const DenseLayout &lay, int sms,
                                   cudaStream_t st) {
  return d == 128 ? launch_tf<128>(a, lay, sms, st) : launch_tf<64>(a, lay, sms, st);
}
cudaError_t launch_transform_paged(int d, const EncArgs &a, const PagedLayout &lay, int sms,
                                   cudaStream_t st) {
  return d == 128 ? launch_tf<128>(a, lay, sms, st) : launch_tf<64>(a, lay, sms, st);
}
cudaError_t launch_quantize(int d, int bits, int group, const EncArgs &a, int sms, cudaStream_t st) {
  if (d == 128) {
    if (bits == 8 && group == 128) return launch_q<128, 8, 128>(a, sms, st);
    if (bits == 8 && group == 64) return launch_q<128, 8, 64>(a, sms, st);
    if (bits == 8 && group == 32) return launch_q<128, 8, 32>(a, sms, st);
    if (bits == 4 && group == 128) return launch_q<128, 4, 128>(a, sms, st);
    if (bits == 4 && group == 64) return launch_q<128, 4, 64>(a, sms, st);
    if (bits == 4 && group == 32) return launch_q<128, 4, 32>(a, sms, st);
    if (bits == 2 && group == 128) return launch_q<128, 2, 128>(a, sms, st);
    if (bits == 2 && group == 64) return launch_q<128, 2, 64>(a, sms, st);
    if (bits == 2 && group == 32) return launch_q<128, 2, 32>(a, sms, st);
  } else {
    if (bits == 8 && group == 64) return launch_q<64, 8, 64>(a, sms, st);
    if (bits == 8 && group == 32) return launch_q<64, 8, 32>(a, sms, st);
    if (bits == 4 && group == 64) return launch_q<64, 4, 64>(a, sms, st);
    if (bits == 4 && group == 32) return launch_q<64, 4, 32>(a, sms, st);
    if (bits == 2 && group == 64) return launch_q<64, 2, 64>(a, sms, st);
    if (bits == 2 && group == 32) return launch_q<64, 2, 32>(a, sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvc
