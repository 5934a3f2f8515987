// Decode instantiation: head_dim 64, paged receiver.
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_decode_paged_d64(const DecArgs &a, const PagedLayout &lay, int sms,
                                  cudaStream_t st) {
  return launch_dec<64>(a, lay, sms, st);
}
}  // namespace kvc
