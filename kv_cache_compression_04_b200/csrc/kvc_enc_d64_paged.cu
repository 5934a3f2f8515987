// Encode instantiations: head_dim 64, paged input, 2- and 4-bit codes with
// the global sign diagonal (8-bit codes and per-vector diagonals:
// kvc_enc_d64_paged_var.cu).
#include "kvc_launch.cuh"

namespace kvc {
cudaError_t launch_encode_paged_d64(int bits, int group, const EncArgs &a, const PagedLayout &lay,
                                  int sms, cudaStream_t st) {
  return launch_enc_dispatch<64>(bits, group, a, lay, sms, st, launch_encode_paged_d64_var);
}
}  // namespace kvc
