// Launches of kvc_attend: meta chunk expansion (shared with the decoder),
// the split-K attention kernel, the combining kernel.
#include "kvc_attend.cuh"
#include "kvc_attend_mma.cuh"
#include "kvc_launch.cuh"

namespace kvc {

namespace {

template <int BITS, int G, int QPK>
cudaError_t launch_att_k(const AttnArgs &a, int units, cudaStream_t st) {
  // 2- and 4-bit codes of the affine quantizers: tensor cores (query heads
  // in tiles of 4); 8-bit and FP4 codes: CUDA cores
  if constexpr (BITS != 8 && QPK >= 2) {
    if (!a.fp4 && !a.cuda_cores) {
      // the per-call and per-unit preparation, then the attention (dependent
      // launches; the preparation's time counts in the attention's interval)
      cudaError_t e = launch_after_unmarked(attend_prep_kernel<BITS, G, (QPK <= 4)>, units + 1,
                                            kAttThreads, 0, st, a);
      if (e != cudaSuccess) return e;
      return launch_after(attend_mma_kernel<BITS, G, QPK < 4 ? 4 : QPK>, units * int(a.splits),
                          kAttThreads, 0, st, a);
    }
  }
  if constexpr (BITS == 4) {
    if (a.fp4)
      attend_kernel<128, 4, G, QPK, true><<<units * a.splits, kAttThreads, 0, st>>>(a);
    else
      attend_kernel<128, 4, G, QPK><<<units * a.splits, kAttThreads, 0, st>>>(a);
  } else {
    attend_kernel<128, BITS, G, QPK><<<units * a.splits, kAttThreads, 0, st>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  timing_mark(st);
  return e;
}

template <int BITS, int G>
cudaError_t launch_att_q(const AttnArgs &a, int units, cudaStream_t st) {
  // query heads per kv head, rounded up to a compiled count
  if (a.qpk == 1) return launch_att_k<BITS, G, 1>(a, units, st);
  if (a.qpk == 2) return launch_att_k<BITS, G, 2>(a, units, st);
  if (a.qpk <= 4) return launch_att_k<BITS, G, 4>(a, units, st);
  if (a.qpk <= 8) return launch_att_k<BITS, G, 8>(a, units, st);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attend(const AttnArgs &a, const DecArgs &d, int sms, cudaStream_t st) {
  // eliminated meta chunks into the workspace (a dependent launch of the status clear)
  auto mk = meta_expand_kernel<128>;
  struct MetaTag {};
  cudaError_t e = prepare<MetaTag>(mk, meta_smem_bytes());
  if (e != cudaSuccess) return e;
  const uint32_t mcap = uint32_t(kMetaCtas) * uint32_t(sms);
  const int mgrid = int(d.ws_meta_chunks == 0 ? 1u : (d.ws_meta_chunks < mcap ? d.ws_meta_chunks : mcap));
  e = launch_after(mk, mgrid, kMetaThreads, meta_smem_bytes(), st, d);
  if (e != cudaSuccess) return e;
  const int units = int(a.layers * a.n_req * a.kv_heads);
  if (a.bits == 8 && a.group == 128) e = launch_att_q<8, 128>(a, units, st);
  else if (a.bits == 8 && a.group == 64) e = launch_att_q<8, 64>(a, units, st);
  else if (a.bits == 8 && a.group == 32) e = launch_att_q<8, 32>(a, units, st);
  else if (a.bits == 4 && a.group == 128) e = launch_att_q<4, 128>(a, units, st);
  else if (a.bits == 4 && a.group == 64) e = launch_att_q<4, 64>(a, units, st);
  else if (a.bits == 4 && a.group == 32) e = launch_att_q<4, 32>(a, units, st);
  else if (a.bits == 2 && a.group == 128) e = launch_att_q<2, 128>(a, units, st);
  else if (a.bits == 2 && a.group == 64) e = launch_att_q<2, 64>(a, units, st);
  else if (a.bits == 2 && a.group == 32) e = launch_att_q<2, 32>(a, units, st);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  const uint32_t n_out = a.layers * a.n_req * a.kv_heads * a.qpk;
  return launch_after(attend_combine_kernel<128>, int((n_out + kCombWarps - 1) / kCombWarps),
                      kCombWarps * 32, 0, st, a);
}

}  // namespace kvc
