// Decode instantiation: head_dim 128, dense receiver.
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_decode_dense_d128(const DecArgs &a, const DenseLayout &lay, int sms,
                                  cudaStream_t st) {
  return launch_dec<128>(a, lay, sms, st);
}
}  // namespace kvc
