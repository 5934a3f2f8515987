// Encode instantiations: head_dim 128, dense input, 8-bit codes and
// per-(layer, kv, head) sign diagonals.
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_encode_dense_d128_var(int bits, int group, const EncArgs &a,
                                      const DenseLayout &lay, int sms, cudaStream_t st) {
  return launch_enc_dispatch_var<128>(bits, group, a, lay, sms, st);
}
}  // namespace kvc
