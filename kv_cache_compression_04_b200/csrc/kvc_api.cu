// Host side of the C ABI in include/kvc.h: argument validation, stream layout
// arithmetic, workspace layout, kernel parameters and launches. Allocates
// nothing and keeps no state beyond per-kernel launch attributes.
#include <string.h>

#include <initializer_list>
#include <utility>

#include <cuda_runtime.h>

#include "kvc_internal.h"
#include "../../include/kvc_test.h"

using namespace kvc;

namespace kvc {
KernelTiming &kernel_timing() {
  static thread_local KernelTiming t;
  return t;
}
}  // namespace kvc

namespace {

struct Shape {
  int D = 0, bits = 0, G = 0;
  uint64_t T = 0;      // tokens per (layer, kv, head), summed over requests
  uint64_t V = 0;      // vectors
  uint32_t n_req = 0;
  uint64_t CB = 0, MB = 0, VC = 0, R = 0;
  uint64_t n_code = 0, n_seg = 0, n_chunks = 0;
  uint64_t data_base = 0, max_bytes = 0, ws_bytes = 0;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Clears n 16-byte words (the per-call part of a workspace), so that the
// next kernel can be a dependent launch of it.
__global__ void __launch_bounds__(256) clear_words_kernel(uint4 *p, uint64_t n) {
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += uint64_t(gridDim.x) * blockDim.x)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
}
inline cudaError_t clear_words(void *p, uint64_t bytes, int sms, cudaStream_t st) {
  const uint64_t n = bytes / 16, want = (n + 255) / 256, cap = uint64_t(sms) * 4;
  const int grid = int(want == 0 ? 1 : (want < cap ? want : cap));
  timing_mark(st);  // before a call's first kernel
  clear_words_kernel<<<grid, 256, 0, st>>>(static_cast<uint4 *>(p), n);
  timing_mark(st);
  return cudaGetLastError();
}

// Sets this thread's kernel timing for the duration of one timed call.
struct TimedCall {
  explicit TimedCall(const cudaEvent_t *ev) { kernel_timing() = KernelTiming{ev, 0}; }
  ~TimedCall() { kernel_timing() = KernelTiming{}; }
};

bool stride_ok(int64_t s) { return s % 8 == 0; }  // 16-byte vector starts

// Shape and layout checks shared by both directions (bits/group optional).
kvc_status describe(const kvc_kv_desc *kv, const kvc_params *p, Shape &s) {
  if (!kv) return KVC_ERR_INVALID_ARG;
  if (kv->kind != KVC_DENSE && kv->kind != KVC_PAGED) return KVC_ERR_INVALID_ARG;
  if (kv->layers < 0 || kv->kv_heads < 0) return KVC_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return KVC_ERR_UNSUPPORTED;
  s.D = kv->head_dim;
  if (!stride_ok(kv->stride_layer) || !stride_ok(kv->stride_kv) || !stride_ok(kv->stride_head))
    return KVC_ERR_INVALID_ARG;
  if (kv->kind == KVC_DENSE) {
    if (kv->tokens < 0 || kv->tokens >= (int64_t(1) << 31)) return KVC_ERR_INVALID_ARG;
    if (!stride_ok(kv->stride_token)) return KVC_ERR_INVALID_ARG;
    s.T = uint64_t(kv->tokens);
    s.n_req = 1;
  } else {
    if (kv->n_requests < 0 || kv->n_requests > KVC_MAX_REQUESTS) return KVC_ERR_INVALID_ARG;
    if (kv->n_requests > 0 && !kv->seq_lens) return KVC_ERR_INVALID_ARG;
    if (kv->page_tokens < 1 || !stride_ok(kv->stride_page) || !stride_ok(kv->stride_slot))
      return KVC_ERR_INVALID_ARG;
    int64_t maxlen = 0;
    for (int r = 0; r < kv->n_requests; ++r) {
      if (kv->seq_lens[r] < 0) return KVC_ERR_INVALID_ARG;
      s.T += uint64_t(kv->seq_lens[r]);
      maxlen = kv->seq_lens[r] > maxlen ? kv->seq_lens[r] : maxlen;
    }
    if (s.T >= (uint64_t(1) << 31)) return KVC_ERR_INVALID_ARG;
    if (s.T > 0) {
      if (!kv->page_table || kv->num_pages < 1) return KVC_ERR_INVALID_ARG;
      if (kv->page_table_stride < (maxlen + kv->page_tokens - 1) / kv->page_tokens)
        return KVC_ERR_INVALID_ARG;
    }
    s.n_req = uint32_t(kv->n_requests);
  }
  s.V = uint64_t(kv->layers) * 2u * uint64_t(kv->kv_heads) * s.T;
  if (s.V >= (uint64_t(1) << 31)) return KVC_ERR_UNSUPPORTED;
  if (s.V > 0 && (!kv->data || !aligned16(kv->data))) return KVC_ERR_INVALID_ARG;
  if (!p) return KVC_OK;
  if (p->bits != 2 && p->bits != 4 && p->bits != 8) return KVC_ERR_UNSUPPORTED;
  if ((p->quant != KVC_QUANT_ASYM && p->quant != KVC_QUANT_SYM && p->quant != KVC_QUANT_FP4) ||
      (p->signs != KVC_SIGNS_GLOBAL && p->signs != KVC_SIGNS_PER_VECTOR))
    return KVC_ERR_UNSUPPORTED;
  if (p->quant == KVC_QUANT_FP4 && p->bits != 4) return KVC_ERR_UNSUPPORTED;
  if (p->group_size != 32 && p->group_size != 64 && p->group_size != 128)
    return KVC_ERR_UNSUPPORTED;
  if (p->group_size > s.D) return KVC_ERR_UNSUPPORTED;
  if (p->lossless < KVC_LOSSLESS_FIXED || p->lossless > KVC_LOSSLESS_NONE || p->reserved != 0)
    return KVC_ERR_UNSUPPORTED;
  s.bits = p->bits;
  s.G = p->group_size;
  // Stream layout (readings R12/R13): codes and meta chunked separately into
  // 16 KB chunks; one meta chunk covers R = G*bits/32 code chunks.
  s.CB = uint64_t(s.D) * s.bits / 8;
  s.MB = uint64_t(s.D / s.G) * 4;
  s.VC = kChunk / s.CB;
  s.R = uint64_t(s.G) * s.bits / 32;
  s.n_code = (s.V + s.VC - 1) / s.VC;
  s.n_seg = (s.n_code + s.R - 1) / s.R;
  s.n_chunks = s.n_code + s.n_seg;
  s.data_base = round16(kHeader + 8 * s.n_chunks + 4 * uint64_t(s.n_req));
  s.max_bytes = s.data_base;
  if (s.n_code) {
    const uint64_t VM = s.VC * s.R;
    s.max_bytes += (s.n_code - 1) * kChunk + round16((s.V - (s.n_code - 1) * s.VC) * s.CB);
    s.max_bytes += (s.n_seg - 1) * kChunk + round16((s.V - (s.n_seg - 1) * VM) * s.MB);
  }
  s.ws_bytes = ws_layout(s.n_code, s.n_seg).total;
  return KVC_OK;
}

// Meta chunks of the largest meta region any supported group size gives for
// this shape (group 32: head_dim / 8 bytes per vector).
uint64_t max_meta_chunks(const Shape &s) {
  const uint64_t mb = uint64_t(s.D / 32) * 4;
  return (s.V * mb + kChunk - 1) / kChunk;
}
uint64_t decompress_ws_bytes(const Shape &s) { return kWsCtl + max_meta_chunks(s) * kChunk; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Rows at non-negative offsets below 64 GB from the base can be named by a
// 32-bit count of 16-byte units (the kernels' narrow row copies).
bool narrow_extent(std::initializer_list<std::pair<int64_t, int64_t>> dims, int64_t row_bytes) {
  int64_t hi = row_bytes;
  for (const auto &d : dims) {  // (stride in bytes, index count)
    if (d.first < 0) return false;
    if (d.second > 1) hi += d.first * (d.second - 1);
  }
  return hi <= (int64_t(1) << 36);
}

DenseLayout dense_layout(const kvc_kv_desc *kv, const Shape &s) {
  DenseLayout L{};
  L.base = static_cast<uint8_t *>(kv->data);
  L.s_l = kv->stride_layer * 2;
  L.s_kv = kv->stride_kv * 2;
  L.s_h = kv->stride_head * 2;
  L.s_t = kv->stride_token * 2;
  L.T = make_fastdiv(s.T ? uint32_t(s.T) : 1u);
  L.H = make_fastdiv(kv->kv_heads ? uint32_t(kv->kv_heads) : 1u);
  L.tokens = uint32_t(s.T);
  L.narrow = narrow_extent({{L.s_l, kv->layers}, {L.s_kv, 2}, {L.s_h, kv->kv_heads},
                            {L.s_t, int64_t(s.T)}},
                           2 * int64_t(s.D));
  return L;
}

// Tensor map of a dense input for the encoder's per-warp tensor loads:
// 5-D [layers][2][kv_heads][tokens][head_dim], boxes of 32 tokens x 64
// channels with 128-byte swizzle. Only when every 32-vector block lies in one
// head row (tokens % 32 == 0); the encoder copies rows one by one otherwise.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return EncodeTiledFn(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

void add_tensor_map(const kvc_kv_desc *kv, const Shape &s, DenseLayout &L) {
  L.tma = 0;
  if (s.V == 0 || s.T % 32 != 0) return;
  const EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return;
  const cuuint64_t dims[5] = {cuuint64_t(s.D), cuuint64_t(s.T), cuuint64_t(kv->kv_heads), 2,
                              cuuint64_t(kv->layers)};
  const cuuint64_t strides[4] = {cuuint64_t(L.s_t), cuuint64_t(L.s_h), cuuint64_t(L.s_kv),
                                 cuuint64_t(L.s_l)};
  const cuuint32_t box[5] = {64, 32, 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  if (fn(&L.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, kv->data, dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
    L.tma = 1;
}

// Tensor map of a paged pool for the encoder's run loads: 5-D [layers]
// [pages][2 * kv_heads][page_tokens][head_dim] with kv and head merged into
// one dimension (needs stride_kv == kv_heads * stride_head), boxes of one run
// of slots x 64 channels with 128-byte swizzle. A run is 16 slots, 8 for
// pages of 8; page_tokens must be a power of two from 8 to 512, and the
// pool fit the load plans' fields (paged_plan_kernel): 2 * kv_heads <= 2048,
// layers <= 4096, num_pages < 2^27.
void add_tensor_map_paged(const kvc_kv_desc *kv, const Shape &s, PagedLayout &L) {
  L.tma = 0;
  const int64_t pt = kv->page_tokens;
  if (s.V == 0 || pt < 8 || pt > 512 || (pt & (pt - 1)) != 0 ||
      kv->stride_kv != kv->kv_heads * kv->stride_head || 2 * int64_t(kv->kv_heads) > 2048 ||
      kv->layers > 4096 || kv->num_pages >= (int64_t(1) << 27))
    return;
  if (kv->stride_slot <= 0 || kv->stride_head <= 0 || kv->stride_page <= 0 || kv->stride_layer <= 0)
    return;
  const EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return;
  const cuuint64_t dims[5] = {cuuint64_t(s.D), cuuint64_t(kv->page_tokens),
                              cuuint64_t(2 * kv->kv_heads), cuuint64_t(kv->num_pages),
                              cuuint64_t(kv->layers)};
  const cuuint64_t strides[4] = {cuuint64_t(L.s_slot), cuuint64_t(L.s_h), cuuint64_t(L.s_p),
                                 cuuint64_t(L.s_l)};
  uint32_t page_lg = 3;
  while ((int64_t(1) << page_lg) < pt) ++page_lg;
  const uint32_t run_lg = page_lg < 4 ? page_lg : 4;
  const cuuint32_t box[5] = {64, cuuint32_t(1u << run_lg), 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  if (fn(&L.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, kv->data, dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS) {
    L.tma = 1;
    L.run_lg = run_lg;
    L.page_lg = page_lg;
  }
}

void paged_layout(const kvc_kv_desc *kv, const Shape &s, PagedLayout &L) {
  L.tma = 0;  // add_tensor_map_paged sets it for the encoder
  L.run_lg = L.page_lg = 0;
  L.base = static_cast<uint8_t *>(kv->data);
  L.s_l = kv->stride_layer * 2;
  L.s_p = kv->stride_page * 2;
  L.s_kv = kv->stride_kv * 2;
  L.s_h = kv->stride_head * 2;
  L.s_slot = kv->stride_slot * 2;
  L.page_table = kv->page_table;
  L.pt_stride = kv->page_table_stride;
  L.num_pages = kv->num_pages;
  L.T = make_fastdiv(s.T ? uint32_t(s.T) : 1u);
  L.H = make_fastdiv(kv->kv_heads ? uint32_t(kv->kv_heads) : 1u);
  L.PT = make_fastdiv(uint32_t(kv->page_tokens));
  L.n_req = s.n_req;
  L.narrow = narrow_extent({{L.s_l, kv->layers}, {L.s_p, kv->num_pages}, {L.s_kv, 2},
                            {L.s_h, kv->kv_heads}, {L.s_slot, kv->page_tokens}},
                           2 * int64_t(s.D));
  L.cum[0] = 0;
  for (uint32_t r = 0; r < s.n_req; ++r) L.cum[r + 1] = L.cum[r] + uint32_t(kv->seq_lens[r]);
}

}  // namespace

extern "C" {

size_t kvc_max_compressed_bytes(const kvc_kv_desc *kv, const kvc_params *params) {
  Shape s;
  if (!params || describe(kv, params, s) != KVC_OK) return 0;
  return size_t(s.max_bytes);
}

size_t kvc_decompress_workspace_bytes(const kvc_kv_desc *out) {
  Shape s;
  if (describe(out, nullptr, s) != KVC_OK) return 0;
  return size_t(decompress_ws_bytes(s));
}

size_t kvc_workspace_bytes(const kvc_kv_desc *kv, const kvc_params *params) {
  Shape s;
  if (!params || describe(kv, params, s) != KVC_OK) return 0;
  return size_t(s.ws_bytes);
}

size_t kvc_unfused_workspace_bytes(const kvc_kv_desc *kv, const kvc_params *params) {
  Shape s;
  if (!params || describe(kv, params, s) != KVC_OK) return 0;
  return size_t(round256(s.ws_bytes) + s.V * uint64_t(s.D) * 4);
}

namespace {

// kvc_compress, or (unfused) the two-kernel baseline that keeps the
// transformed vectors in the workspace after the compress workspace.
kvc_status compress_impl(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                         size_t out_capacity, uint64_t *out_bytes_dev, void *workspace,
                         size_t workspace_bytes, kvc_stream_t stream, bool unfused,
                         uint32_t ticket_skip = 0, uint64_t wait_ns = kWaitNs) {
  Shape s;
  if (!params) return KVC_ERR_INVALID_ARG;
  kvc_status st = describe(kv, params, s);
  if (st != KVC_OK) return st;
  // the unfused baseline: the global diagonal and the affine quantizers only
  if (unfused && (params->signs != KVC_SIGNS_GLOBAL || params->quant == KVC_QUANT_FP4))
    return KVC_ERR_UNSUPPORTED;
  if (!out || !aligned16(out) || !workspace || !aligned16(workspace)) return KVC_ERR_INVALID_ARG;
  const uint64_t need = unfused ? round256(s.ws_bytes) + s.V * uint64_t(s.D) * 4 : s.ws_bytes;
  if (out_capacity < s.max_bytes || workspace_bytes < need) return KVC_ERR_CAPACITY;
  const int sms = sm_count();
  if (sms <= 0) return KVC_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const WsLayout w = ws_layout(s.n_code, s.n_seg);
  uint32_t *ctl = reinterpret_cast<uint32_t *>(ws);  // status, flags, ticket, reads, first, -, saved
  EncArgs a{};
  a.V = uint32_t(s.V);
  a.out = static_cast<uint8_t *>(out);
  a.data_base = s.data_base;
  a.status = ctl;
  a.flags = ctl + 1;
  a.first_inv = ctl + 4;
  a.saved = reinterpret_cast<unsigned long long *>(ctl + 6);
  a.code_nnz = reinterpret_cast<unsigned long long *>(ws + w.code_nnz);
  a.meta_nnz = reinterpret_cast<unsigned long long *>(ws + w.meta_nnz);
  a.ws_meta = ws + w.meta;
  a.ymid = unfused ? reinterpret_cast<float *>(ws + round256(s.ws_bytes)) : nullptr;
  a.one = 1.0f;
  a.mode = uint32_t(params->lossless);
  a.sym = params->quant == KVC_QUANT_SYM ? 1u : 0u;
  a.vec_signs = params->signs == KVC_SIGNS_PER_VECTOR ? 1u : 0u;
  a.fp4 = params->quant == KVC_QUANT_FP4 ? 1u : 0u;
  a.seed = params->sign_seed;
  a.tdiv = make_fastdiv(uint32_t(s.T ? s.T : 1));
  sign_masks(params->sign_seed, s.D, a.sign_mask);
  for (int k = 0; k < s.D / 2; ++k) a.sign_lo[k] = a.sign_mask[k] << 16;

  FinArgs f{};
  f.V = uint32_t(s.V);
  f.n_code = uint32_t(s.n_code);
  f.n_meta = uint32_t(s.n_seg);
  f.n_chunks = uint32_t(s.n_chunks);
  f.cb = uint32_t(s.CB);
  f.mb = uint32_t(s.MB);
  f.vc = uint32_t(s.VC);
  f.vm = uint32_t(s.VC * s.R);
  f.out = a.out;
  f.out_capacity = out_capacity;
  f.data_base = s.data_base;
  f.out_bytes_dev = out_bytes_dev;
  f.status = ctl;
  f.flags = ctl + 1;
  f.first_inv = ctl + 4;
  f.saved = a.saved;
  f.ticket = ctl + 2;  // ticket[0]: next code chunk to move, ticket[1]: chunks read
  f.code_nnz = a.code_nnz;
  f.meta_nnz = a.meta_nnz;
  f.code_size = reinterpret_cast<uint32_t *>(ws + w.code_size);
  f.done = reinterpret_cast<uint32_t *>(ws + w.done);
  f.meta_size = reinterpret_cast<uint32_t *>(ws + w.meta_size);
  f.code_off = reinterpret_cast<uint64_t *>(ws + w.code_off);
  f.ws_meta = a.ws_meta;
  f.layers = uint32_t(kv->layers);
  f.kv_heads = uint32_t(kv->kv_heads);
  f.head_dim = uint32_t(s.D);
  f.group = uint32_t(s.G);
  f.bits = uint32_t(s.bits);
  f.k = (s.D == 64 ? 6u : s.D == 128 ? 7u : 8u) / 2;
  f.origin = kv->kind == KVC_PAGED ? 1u : 0u;
  f.n_req = s.n_req;
  f.tokens = s.T;
  f.seed = params->sign_seed;
  f.mode = uint32_t(params->lossless);
  f.quant = uint32_t(params->quant);
  f.signs = uint32_t(params->signs);
  f.wait_ns = wait_ns;
  f.ticket_skip = ticket_skip;

  if (clear_words(ws, w.zero_bytes, sms, cs) != cudaSuccess) return KVC_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  if (kv->kind == KVC_DENSE) {
    DenseLayout L = dense_layout(kv, s);
    add_tensor_map(kv, s, L);
    if (s.n_code && unfused) {
      e = launch_transform_dense(s.D, a, L, sms, cs);
      if (e == cudaSuccess) e = launch_quantize(s.D, s.bits, s.G, a, sms, cs);
    } else if (s.n_code) {
      e = s.D == 128 ? launch_encode_dense_d128(s.bits, s.G, a, L, sms, cs)
                     : launch_encode_dense_d64(s.bits, s.G, a, L, sms, cs);
    } else {
      timing_mark(cs);  // no encode kernel: its interval is empty
    }
    if (e == cudaSuccess) e = launch_finish_dense(f, L, sms, cs);
  } else {
    static thread_local PagedLayout L;  // large (4 KB) parameter block
    paged_layout(kv, s, L);
    add_tensor_map_paged(kv, s, L);
    if (s.n_code && unfused) {
      e = launch_transform_paged(s.D, a, L, sms, cs);
      if (e == cudaSuccess) e = launch_quantize(s.D, s.bits, s.G, a, sms, cs);
    } else if (s.n_code) {
      e = s.D == 128 ? launch_encode_paged_d128(s.bits, s.G, a, L, sms, cs)
                     : launch_encode_paged_d64(s.bits, s.G, a, L, sms, cs);
    } else {
      timing_mark(cs);  // no encode kernel: its interval is empty
    }
    if (e == cudaSuccess) e = launch_finish_paged(f, L, sms, cs);
  }
  return e == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

}  // namespace

kvc_status kvc_compress(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                        size_t out_capacity, uint64_t *out_bytes_dev, void *workspace,
                        size_t workspace_bytes, kvc_stream_t stream) {
  return compress_impl(kv, params, out, out_capacity, out_bytes_dev, workspace, workspace_bytes,
                       stream, false);
}

kvc_status kvc_compress_unfused(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                                size_t out_capacity, uint64_t *out_bytes_dev, void *workspace,
                                size_t workspace_bytes, kvc_stream_t stream) {
  return compress_impl(kv, params, out, out_capacity, out_bytes_dev, workspace, workspace_bytes,
                       stream, true);
}

kvc_status kvc_test_compress_stalled(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                                     size_t out_capacity, uint64_t *out_bytes_dev,
                                     void *workspace, size_t workspace_bytes,
                                     uint32_t skip_chunks, uint64_t wait_ns,
                                     kvc_stream_t stream) {
  if (skip_chunks == 0 || wait_ns == 0 || wait_ns > kWaitNs) return KVC_ERR_INVALID_ARG;
  return compress_impl(kv, params, out, out_capacity, out_bytes_dev, workspace, workspace_bytes,
                       stream, false, skip_chunks, wait_ns);
}

kvc_status kvc_compress_timed(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                              size_t out_capacity, uint64_t *out_bytes_dev, void *workspace,
                              size_t workspace_bytes, void *const *events, int n_events,
                              kvc_stream_t stream) {
  if (!events || n_events != 5) return KVC_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return KVC_ERR_INVALID_ARG;
  TimedCall timed(reinterpret_cast<const cudaEvent_t *>(events));
  return compress_impl(kv, params, out, out_capacity, out_bytes_dev, workspace, workspace_bytes,
                       stream, false);
}

kvc_status kvc_decompress_timed(const void *in, size_t in_bytes, const kvc_kv_desc *out,
                                void *workspace, size_t workspace_bytes, void *const *events,
                                int n_events, kvc_stream_t stream) {
  if (!events || n_events != 5) return KVC_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return KVC_ERR_INVALID_ARG;
  TimedCall timed(reinterpret_cast<const cudaEvent_t *>(events));
  return kvc_decompress(in, in_bytes, out, workspace, workspace_bytes, stream);
}

extern "C++" {  // (the test kernels, inside the C-linkage block)
namespace kvc {
__global__ void e2m1_test_kernel(const float *in, uint8_t *out, uint32_t n) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = uint8_t(e2m1_rne(in[i]));
}
template <int Q>
__global__ void div_const_test_kernel(const float *in, float *out, uint32_t n) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = div_const<Q>(in[i]);
}
__global__ void rcp_scale_test_kernel(const float *in, float *out, uint32_t n) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = rcp_scale(in[i]);
}
}  // namespace kvc
}

kvc_status kvc_test_rcp_scale(const float *in, float *out, uint64_t n, kvc_stream_t stream) {
  if (!in || !out || n >= (uint64_t(1) << 31)) return KVC_ERR_INVALID_ARG;
  if (n == 0) return KVC_OK;
  kvc::rcp_scale_test_kernel<<<unsigned((n + 255) / 256), 256, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(in, out, uint32_t(n));
  return cudaGetLastError() == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

kvc_status kvc_test_div_const(const float *in, float *out, uint64_t n, int q,
                              kvc_stream_t stream) {
  if (!in || !out || n >= (uint64_t(1) << 31)) return KVC_ERR_INVALID_ARG;
  void (*k)(const float *, float *, uint32_t) = nullptr;
  switch (q) {
    case 1: k = kvc::div_const_test_kernel<1>; break;
    case 3: k = kvc::div_const_test_kernel<3>; break;
    case 7: k = kvc::div_const_test_kernel<7>; break;
    case 15: k = kvc::div_const_test_kernel<15>; break;
    case 127: k = kvc::div_const_test_kernel<127>; break;
    case 255: k = kvc::div_const_test_kernel<255>; break;
    default: return KVC_ERR_INVALID_ARG;
  }
  if (n == 0) return KVC_OK;
  k<<<unsigned((n + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, out,
                                                                                 uint32_t(n));
  return cudaGetLastError() == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

kvc_status kvc_test_e2m1(const float *in, uint8_t *out, uint64_t n, kvc_stream_t stream) {
  if (!in || !out || n >= (uint64_t(1) << 31)) return KVC_ERR_INVALID_ARG;
  if (n == 0) return KVC_OK;
  kvc::e2m1_test_kernel<<<unsigned((n + 255) / 256), 256, 0,
                          reinterpret_cast<cudaStream_t>(stream)>>>(in, out, uint32_t(n));
  return cudaGetLastError() == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

kvc_status kvc_attend_timed(const void *in, size_t in_bytes, const kvc_attn_desc *attn,
                            void *workspace, size_t workspace_bytes, void *const *events,
                            int n_events, kvc_stream_t stream) {
  if (!events || n_events != 5) return KVC_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return KVC_ERR_INVALID_ARG;
  TimedCall timed(reinterpret_cast<const cudaEvent_t *>(events));
  return kvc_attend(in, in_bytes, attn, workspace, workspace_bytes, stream);
}

kvc_status kvc_decompress(const void *in, size_t in_bytes, const kvc_kv_desc *out,
                          void *workspace, size_t workspace_bytes, kvc_stream_t stream) {
  Shape s;
  kvc_status st = describe(out, nullptr, s);
  if (st != KVC_OK) return st;
  if (!in || !aligned16(in) || !workspace || !aligned16(workspace)) return KVC_ERR_INVALID_ARG;
  if (workspace_bytes < decompress_ws_bytes(s)) return KVC_ERR_CAPACITY;
  const int sms = sm_count();
  if (sms <= 0) return KVC_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  DecArgs a{};
  a.in = static_cast<const uint8_t *>(in);
  a.in_bytes = in_bytes;
  a.status = static_cast<uint32_t *>(workspace);
  a.layers = uint32_t(out->layers);
  a.kv_heads = uint32_t(out->kv_heads);
  a.head_dim = uint32_t(s.D);
  a.n_req = s.n_req;
  a.tokens = s.T;
  a.V = uint32_t(s.V);
  a.paged_receiver = out->kind == KVC_PAGED ? 1u : 0u;
  a.tdiv = make_fastdiv(uint32_t(s.T ? s.T : 1));
  a.ws_meta = static_cast<uint8_t *>(workspace) + kWsCtl;
  a.ws_meta_chunks = uint32_t(max_meta_chunks(s));
  if (clear_words(workspace, kWsCtl, sms, cs) != cudaSuccess) return KVC_ERR_CUDA;
  cudaError_t e;
  if (out->kind == KVC_DENSE) {
    DenseLayout L = dense_layout(out, s);
    add_tensor_map(out, s, L);
    e = s.D == 128 ? launch_decode_dense_d128(a, L, sms, cs) : launch_decode_dense_d64(a, L, sms, cs);
  } else {
    static thread_local PagedLayout L;
    paged_layout(out, s, L);
    e = s.D == 128 ? launch_decode_paged_d128(a, L, sms, cs) : launch_decode_paged_d64(a, L, sms, cs);
  }
  return e == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

namespace {
constexpr int kAttTokHost = 256;  // tokens per attention CTA (kvc_attend.cuh: kAttTok)

// Shape checks of kvc_attend and its workspace layout: status | expanded
// meta chunks | split partials.
struct AttnShape {
  Shape s;
  uint64_t meta_off, meta_chunks, part_off, prep_off, total;
  uint32_t splits, units;
};
kvc_status attn_shape(const kvc_attn_desc *at, AttnShape &r) {
  if (!at) return KVC_ERR_INVALID_ARG;
  if (at->head_dim != 128) return KVC_ERR_UNSUPPORTED;
  if (at->q_per_kv < 1 || at->q_per_kv > 8) return KVC_ERR_UNSUPPORTED;
  if (at->kernel != 0 && at->kernel != 1) return KVC_ERR_INVALID_ARG;
  if (at->n_requests < 1 || at->n_requests > KVC_MAX_REQUESTS || !at->seq_lens)
    return KVC_ERR_INVALID_ARG;
  // the stream's logical shape as a paged description without pages: the
  // shape checks and layout arithmetic of the codec
  kvc_kv_desc kv{};
  kv.kind = KVC_DENSE;
  kv.layers = at->layers;
  kv.kv_heads = at->kv_heads;
  kv.head_dim = at->head_dim;
  int64_t T = 0, maxlen = 0;
  for (int i = 0; i < at->n_requests; ++i) {
    if (at->seq_lens[i] < 0) return KVC_ERR_INVALID_ARG;
    T += at->seq_lens[i];
    maxlen = at->seq_lens[i] > maxlen ? at->seq_lens[i] : maxlen;
  }
  kv.tokens = T;
  kv.data = reinterpret_cast<void *>(uintptr_t(16));  // shape only: never read
  kv.stride_token = at->head_dim;
  kv.stride_head = T * at->head_dim;
  kv.stride_kv = kv.stride_head * at->kv_heads;
  kv.stride_layer = kv.stride_kv * 2;
  kvc_params p{at->bits, at->group_size, 0, KVC_LOSSLESS_FIXED, at->quant, KVC_SIGNS_GLOBAL, 0};
  const kvc_status st = describe(&kv, &p, r.s);
  if (st != KVC_OK) return st;
  r.s.n_req = uint32_t(at->n_requests);
  r.splits = uint32_t(maxlen == 0 ? 1 : (maxlen + kAttTokHost - 1) / kAttTokHost);
  r.units = uint32_t(at->layers) * uint32_t(at->n_requests) * uint32_t(at->kv_heads);
  r.meta_off = kWsCtl;
  // the stated group fixes the meta chunk count (a stream with another
  // group fails the header check; meta expansion never exceeds the slots)
  r.meta_chunks = (r.s.V * uint64_t(at->head_dim / at->group_size) * 4 + kChunk - 1) / kChunk;
  r.part_off = round256(r.meta_off + r.meta_chunks * kChunk);
  r.prep_off = round256(r.part_off + uint64_t(r.units) * r.splits * uint64_t(at->q_per_kv) *
                                         (uint64_t(at->head_dim) + 4) * sizeof(float));
  r.total = r.prep_off + prep_bytes(uint32_t(r.meta_chunks), r.units);
  return KVC_OK;
}
}  // namespace

size_t kvc_attend_workspace_bytes(const kvc_attn_desc *at) {
  AttnShape r;
  return attn_shape(at, r) == KVC_OK ? size_t(r.total) : 0;
}

kvc_status kvc_attend(const void *in, size_t in_bytes, const kvc_attn_desc *at, void *workspace,
                      size_t workspace_bytes, kvc_stream_t stream) {
  AttnShape r;
  kvc_status st = attn_shape(at, r);
  if (st != KVC_OK) return st;
  if (!in || !aligned16(in) || !workspace || !aligned16(workspace) || !at->q || !at->out ||
      (reinterpret_cast<uintptr_t>(at->q) & 1u) || (reinterpret_cast<uintptr_t>(at->out) & 3u))
    return KVC_ERR_INVALID_ARG;
  if (workspace_bytes < r.total) return KVC_ERR_CAPACITY;
  const int sms = sm_count();
  if (sms <= 0) return KVC_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecArgs d{};
  d.in = static_cast<const uint8_t *>(in);
  d.in_bytes = in_bytes;
  d.status = reinterpret_cast<uint32_t *>(ws);
  d.layers = uint32_t(at->layers);
  d.kv_heads = uint32_t(at->kv_heads);
  d.head_dim = uint32_t(at->head_dim);
  d.n_req = r.s.n_req;
  d.tokens = r.s.T;
  d.V = uint32_t(r.s.V);
  d.paged_receiver = 0;
  d.ws_meta = ws + r.meta_off;
  d.ws_meta_chunks = uint32_t(r.meta_chunks);
  static thread_local AttnArgs a;  // large (4 KB) parameter block
  a.in = d.in;
  a.in_bytes = in_bytes;
  a.status = d.status;
  a.layers = d.layers;
  a.kv_heads = d.kv_heads;
  a.n_req = d.n_req;
  a.qpk = uint32_t(at->q_per_kv);
  a.bits = uint32_t(at->bits);
  a.group = uint32_t(at->group_size);
  a.fp4 = at->quant == KVC_QUANT_FP4 ? 1u : 0u;
  a.cuda_cores = at->kernel == 1 ? 1u : 0u;
  a.tokens = r.s.T;
  a.V = d.V;
  a.splits = r.splits;
  a.q = static_cast<const uint16_t *>(at->q);
  a.scale = at->scale;
  a.out = at->out;
  a.part = reinterpret_cast<float *>(ws + r.part_off);
  a.ws_meta = d.ws_meta;
  a.prep = ws + r.prep_off;
  a.n_meta = uint32_t(r.meta_chunks);
  a.cum[0] = 0;
  for (int i = 0; i < at->n_requests; ++i) a.cum[i + 1] = a.cum[i] + uint32_t(at->seq_lens[i]);
  if (clear_words(workspace, kWsCtl, sms, cs) != cudaSuccess) return KVC_ERR_CUDA;
  return launch_attend(a, d, sms, cs) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

kvc_status kvc_stream_status(const void *workspace, kvc_stream_t stream) {
  if (!workspace) return KVC_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return KVC_ERR_CUDA;
  return v <= KVC_ERR_CUDA ? static_cast<kvc_status>(v) : KVC_ERR_CUDA;
}

const char *kvc_status_string(kvc_status status) {
  switch (status) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_INVALID_ARG: return "KVC_ERR_INVALID_ARG";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED";
    case KVC_ERR_CAPACITY: return "KVC_ERR_CAPACITY";
    case KVC_ERR_NONFINITE: return "KVC_ERR_NONFINITE";
    case KVC_ERR_RANGE: return "KVC_ERR_RANGE";
    case KVC_ERR_CORRUPT: return "KVC_ERR_CORRUPT";
    case KVC_ERR_TIMEOUT: return "KVC_ERR_TIMEOUT";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA";
  }
  return "KVC_ERR_UNKNOWN";
}

}  // extern "C"
