// Decode instantiation: head_dim 64, dense receiver.
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_decode_dense_d64(const DecArgs &a, const DenseLayout &lay, int sms,
                                  cudaStream_t st) {
  return launch_dec<64>(a, lay, sms, st);
}
}  // namespace kvc
