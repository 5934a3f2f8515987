// Finishing and compaction launches of kvc_compress (dense and paged input).
#include "kvc_finish.cuh"
#include "kvc_launch.cuh"

namespace kvc {

namespace {

template <class Layout>
cudaError_t launch_fin(const FinArgs &a, const Layout &lay, int sms, cudaStream_t st) {
  auto fk = finish_kernel<Layout>;
  const size_t fsmem = fin_smem_bytes(kIsPaged<Layout>);
  struct FinTag {};
  cudaError_t e = prepare<FinTag>(fk, fsmem);
  if (e != cudaSuccess) return e;
  // one meta chunk per CTA where possible (several CTAs share an SM)
  const uint32_t want = a.n_meta > 1 ? a.n_meta : 1u, cap = 4u * uint32_t(sms);
  const int grid = int(want < cap ? want : cap);
  e = launch_after(fk, grid, kFinThreads, fsmem, st, a, lay);
  if (e != cudaSuccess) return e;
  if (a.n_code == 0) {
    timing_mark(st);  // no compaction kernel: its interval is empty
    return e;
  }
  // Returns at once unless a code chunk shrank (flag set by the encode kernel).
  auto ck = compact_kernel;
  const size_t csmem = fin_smem_bytes(false);
  struct CompactTag {};
  e = prepare<CompactTag>(ck, csmem);
  if (e != cudaSuccess) return e;
  const int cgrid = int(a.n_code < cap ? a.n_code : cap);
  return launch_after(ck, cgrid, kFinThreads, csmem, st, a);
}

}  // namespace

cudaError_t launch_finish_dense(const FinArgs &a, const DenseLayout &lay, int sms, cudaStream_t st) {
  return launch_fin(a, lay, sms, st);
}
cudaError_t launch_finish_paged(const FinArgs &a, const PagedLayout &lay, int sms, cudaStream_t st) {
  return launch_fin(a, lay, sms, st);
}

}  // namespace kvc
