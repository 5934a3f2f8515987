// kvc_compress_noalloc: kvc_compress with its workspace in this file's static
// device block instead of caller memory. Nothing here allocates: the block is
// part of the module image, its address is looked up once per device with
// cudaGetSymbolAddress, and kvc_compress clears the part of it that must
// start at zero on the caller's stream.
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/kvc.h"

namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[KVC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of the block on the current device (looked up once).
kvc_status scratch_ptr(void **p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || !q) return KVC_ERR_CUDA;
    g_scratch_ptr[dev] = q;
  }
  *p = g_scratch_ptr[dev];
  return KVC_OK;
}

}  // namespace

extern "C" kvc_status kvc_compress_noalloc(const kvc_kv_desc *kv, const kvc_params *params,
                                           void *out, size_t out_capacity,
                                           uint64_t *out_bytes_dev, uint32_t *status_dev,
                                           kvc_stream_t stream) {
  if (!params) return KVC_ERR_INVALID_ARG;
  // 0 for an invalid description: kvc_compress below returns the precise error
  if (kvc_workspace_bytes(kv, params) > KVC_NOALLOC_SCRATCH_BYTES) return KVC_ERR_CAPACITY;
  if (status_dev && (reinterpret_cast<uintptr_t>(status_dev) & 3u)) return KVC_ERR_INVALID_ARG;
  void *ws = nullptr;
  kvc_status st = scratch_ptr(&ws);
  if (st != KVC_OK) return st;
  st = kvc_compress(kv, params, out, out_capacity, out_bytes_dev, ws, KVC_NOALLOC_SCRATCH_BYTES,
                    stream);
  if (st != KVC_OK || !status_dev) return st;
  // the status word is the first 4 bytes of the workspace
  if (cudaMemcpyAsync(status_dev, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVC_ERR_CUDA;
  return KVC_OK;
}
