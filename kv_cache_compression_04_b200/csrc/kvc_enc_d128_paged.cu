// Encode instantiations: head_dim 128, paged input, 2- and 4-bit codes with
// the global sign diagonal (8-bit codes and per-vector diagonals:
// kvc_enc_d128_paged_var.cu).
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_encode_paged_d128(int bits, int group, const EncArgs &a, const PagedLayout &lay,
                                  int sms, cudaStream_t st) {
  return launch_enc_dispatch<128>(bits, group, a, lay, sms, st, launch_encode_paged_d128_var);
}
}  // namespace kvc
