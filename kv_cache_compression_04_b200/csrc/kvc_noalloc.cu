// kvc_compress_noalloc: kvc_compress with its workspace in this file's static
// device block instead of caller memory. Nothing here allocates: the block is
// part of the module image, its address is looked up with
// cudaGetSymbolAddress once per CUDA context (a context's address stays valid
// for its lifetime), and kvc_compress clears the part of it that must start
// at zero on the caller's stream.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/kvc.h"

namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[KVC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the context the address was looked up in (by its process-unique
// ID, so a context created after a device reset never matches an old entry,
// even if it reuses the old handle value) and the address.
unsigned long long g_ctx_id[kMaxDevices];
void *g_scratch_ptr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <class Fn>
Fn driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Device address of the block in the current context (looked up again
// whenever the current context is not the one of the cached address).
kvc_status scratch_ptr(void **p) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return KVC_ERR_CUDA;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVC_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return KVC_ERR_CUDA;
  if (!ctx) {  // no context current in this thread yet: cudaSetDevice makes the primary one so
    if (cudaSetDevice(dev) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || !ctx)
      return KVC_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return KVC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev] || g_ctx_id[dev] != id) {
    void *q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || !q) return KVC_ERR_CUDA;
    g_scratch_ptr[dev] = q;
    g_ctx_id[dev] = id;
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
