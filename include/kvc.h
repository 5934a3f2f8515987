/*
 * kvc.h — C ABI of libkvc.so, a B200 (sm_100a) KV-cache codec in the manner of
 * FastKVComp ("Beyond Compression Ratio: High-Throughput KV Compression for
 * Disaggregated LLM Serving", Abstract and Methodology; podcast page
 * "FastKVComp: checking whether high-throughput KV compression pays off",
 * episode notes).
 *
 * Encode: random +-1 signs and an fp32 Walsh-Hadamard transform over head_dim,
 * 2- or 4-bit asymmetric group quantization with fp16 scale/zero, code packing,
 * then a lossless stage over 16 KB chunks (bit-plane shuffle, zero-byte
 * elimination with a bitmap, device-wide prefix sum of chunk sizes and
 * compaction) into one self-describing byte stream. Decode inverts every step.
 * Only the quantization loses information.
 *
 * Conventions shared by every entry point:
 *  - Memory. The caller owns every buffer (input, output, page table,
 *    workspace, stream). The library allocates nothing; its only global state
 *    is the static workspace block of kvc_compress_noalloc (end of this
 *    file). Calls are re-entrant, but concurrent calls need distinct
 *    workspaces.
 *  - Asynchrony. All device work is enqueued on `stream` (a cudaStream_t; 0 is
 *    the legacy default stream). Pointers marked DEVICE must stay valid until
 *    that work completes.
 *  - Synchronous errors. Argument, shape and capacity errors are returned
 *    before anything is enqueued: KVC_ERR_INVALID_ARG, KVC_ERR_UNSUPPORTED,
 *    KVC_ERR_CAPACITY. A failed CUDA launch returns KVC_ERR_CUDA.
 *  - Data-dependent errors (non-finite input, fp16 meta overflow, a corrupt
 *    stream, an invalid page index, a device wait that ran out) are written to
 *    a status word in the workspace; kvc_stream_status() reads it. The first
 *    error of a call wins; each call clears the word when it starts.
 *  - Bounds. Encode never writes outside [out, out + out_capacity) or the
 *    workspace; decode never writes outside the output slots its descriptor
 *    names. On an error the output content is unspecified.
 *  - Alignment. `data`, `out`, the stream passed to decode and `workspace`
 *    must be 16-byte aligned; every vector start (all strides times 2 bytes)
 *    must be 16-byte aligned, i.e. strides are multiples of 8 elements.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that this header
 * needs no CUDA include. */
typedef struct CUstream_st *kvc_stream_t;

typedef enum {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1, /* null pointer, bad shape, stride or alignment     */
  KVC_ERR_UNSUPPORTED = 2, /* bits / group / head_dim outside the built set    */
  KVC_ERR_CAPACITY = 3,    /* out_capacity or workspace too small              */
  KVC_ERR_NONFINITE = 4,   /* an input vector transforms to inf or NaN         */
  KVC_ERR_RANGE = 5,       /* a group's zero or scale overflows fp16           */
  KVC_ERR_CORRUPT = 6,     /* stream header, table or chunk inconsistent, or a
                              page index outside the pool                     */
  KVC_ERR_TIMEOUT = 7,     /* a bounded device wait gave up                   */
  KVC_ERR_CUDA = 8         /* CUDA runtime error (launch, copy, device)       */
} kvc_status;

/* Lossless-stage modes of the encoder ("Beyond Compression Ratio: High-
 * Throughput KV Compression for Disaggregated LLM Serving", Abstract and
 * Methodology: a searchable backend that composes primitives into
 * pipelines). A stored chunk's pipeline id (bits 60..63 of its table entry)
 * says which primitives were applied:
 *   0  bit-plane shuffle of 32-bit words, zero-byte elimination with a
 *      2048-byte bitmap
 *   1  each 32-bit word XOR the previous word, restarting every 32 vectors
 *      (meta chunks only), then as 0
 *   2  bit-plane shuffle, two-level zero-byte elimination: the 2048-byte
 *      bitmap itself eliminated under a 256-byte bitmap
 *   3  the XOR of 1, then as 2
 * KVC_LOSSLESS_FIXED uses pipeline 0 only. KVC_LOSSLESS_SEARCH gives every
 * full chunk the shortest of its candidates (code chunks: 0 and 2; meta
 * chunks: 0..3, or 0 and 1 when a vector has one group), ties to the lower
 * id. KVC_LOSSLESS_NONE stores every chunk raw (no lossless stage). In every
 * mode a chunk is stored transformed only if that makes it strictly shorter,
 * and the code region follows the elimination rule documented at
 * kvc_compress. A decoder handles every mode. */
enum { KVC_LOSSLESS_FIXED = 0, KVC_LOSSLESS_SEARCH = 1, KVC_LOSSLESS_NONE = 2 };

/* Quantizer variants and sign diagonals (the FP4Quant abstract on the first
 * page lists quantizer variants of the transform + low-bit step; these are
 * the ones with an exact oracle):
 *   KVC_QUANT_ASYM  asymmetric min/max per group: zero = RD16(min), scale =
 *                   RU16((max - zero) / (2^b - 1)), code = RNE((y - zero) / scale)
 *   KVC_QUANT_SYM   symmetric absmax per group: scale = RU16(max|y| /
 *                   (2^(b-1) - 1)), code = RNE(y / scale) + 2^(b-1) in
 *                   [1, 2^b - 1]; the stored zero is -2^(b-1) * scale, so
 *                   every decoder reads both alike (zero + code * scale)
 *   KVC_QUANT_FP4   4-bit e2m1 codes (0, +-0.5, +-1, +-1.5, +-2, +-3, +-4,
 *                   +-6) with two scales (the FP4Quant abstract's
 *                   micro-grouped dual-scale FP4): per group an fp16 scale
 *                   s2 = RU16(max|y| / 2688), per half-group an e4m3
 *                   micro-scale s1 = RU(max_half|y| / (6 s2)) (at most 448);
 *                   code = e2m1 nearest to y / (s1 s2), ties to even; meta
 *                   bytes s2 (LE), s1 of each half. bits must be 4.
 *   KVC_SIGNS_GLOBAL      one +-1 diagonal for every vector
 *   KVC_SIGNS_PER_VECTOR  one per (layer, kv, head): vector index i (its
 *                   position in the order [layer][kv][head]) takes the
 *                   SplitMix64 outputs i*W .. i*W + W - 1 (W = head_dim / 64)
 * The stream's header flags record both (bits 1..2 and 3); a decoder needs
 * no parameter for them. Decoded values: zero + code * scale (ASYM, SYM),
 * e2m1(code) * s1 * s2 (FP4), each exact in fp32 before the inverse
 * transform. */
enum { KVC_QUANT_ASYM = 0, KVC_QUANT_SYM = 1, KVC_QUANT_FP4 = 2 };
enum { KVC_SIGNS_GLOBAL = 0, KVC_SIGNS_PER_VECTOR = 1 };

/* Quantization and lossless parameters.
 *  bits       2, 4 or 8 bits per code.
 *  group_size 32, 64 or 128 consecutive channels of the transformed vector
 *             share one fp16 zero and scale; must divide head_dim.
 *  sign_seed  seeds the +-1 diagonal: channel c is negated iff bit (c mod 64)
 *             of SplitMix64 output number floor(c/64), counted from state =
 *             sign_seed, is 1 (per-vector diagonals: see above).
 *  lossless   KVC_LOSSLESS_* (encoder only).
 *  quant      KVC_QUANT_*.
 *  signs      KVC_SIGNS_* (kvc_compress_unfused: KVC_SIGNS_GLOBAL and the
 *             min/max or absmax quantizer only).
 *  reserved   must be 0.
 * Other values are refused with KVC_ERR_UNSUPPORTED. */
typedef struct {
  int32_t bits;
  int32_t group_size;
  uint64_t sign_seed;
  int32_t lossless;
  int32_t quant;
  int32_t signs;
  int32_t reserved;
} kvc_params;

enum { KVC_DENSE = 0, KVC_PAGED = 1 };

/* Largest request count of a paged descriptor. */
#define KVC_MAX_REQUESTS 1024

/* A KV cache: logical shape [layers, 2 (K, V), kv_heads, tokens, head_dim],
 * bf16, head_dim contiguous. Vectors are coded in the logical order
 * [layer][kv][head][request][token]; a dense tensor is one request.
 *
 * kind = KVC_DENSE:
 *   element (l, kv, h, t, c) at data + l*stride_layer + kv*stride_kv +
 *   h*stride_head + t*stride_token + c (strides in elements).
 * kind = KVC_PAGED (a pool of pages of page_tokens token slots):
 *   token t of request r sits in page p = page_table[r*page_table_stride +
 *   t/page_tokens], slot t % page_tokens; element (l, kv, h, r, t, c) at
 *   data + l*stride_layer + p*stride_page + kv*stride_kv + h*stride_head +
 *   (t % page_tokens)*stride_slot + c. Pages are checked against
 *   [0, num_pages); a page outside it sets KVC_ERR_CORRUPT and its vectors
 *   are neither read nor written.
 *
 * head_dim is 64 or 128 in this build (256 returns KVC_ERR_UNSUPPORTED). */
typedef struct {
  int32_t kind;
  int32_t layers;
  int32_t kv_heads;
  int32_t head_dim;
  void *data;                 /* DEVICE bf16 tensor or page pool             */
  int64_t stride_layer;       /* elements, both kinds                        */
  int64_t stride_kv;          /* elements, both kinds                        */
  int64_t stride_head;        /* elements, both kinds                        */
  /* dense */
  int64_t tokens;             /* T >= 0                                      */
  int64_t stride_token;       /* elements                                    */
  /* paged */
  int32_t page_tokens;        /* token slots per page, >= 1                  */
  int32_t n_requests;         /* 0 .. KVC_MAX_REQUESTS                       */
  int64_t stride_page;        /* elements                                    */
  int64_t stride_slot;        /* elements                                    */
  int64_t num_pages;          /* pages in the pool                           */
  const int32_t *seq_lens;    /* HOST [n_requests], tokens per request >= 0  */
  const int32_t *page_table;  /* DEVICE int32 [n_requests][page_table_stride] */
  int64_t page_table_stride;  /* entries per request row                     */
} kvc_kv_desc;

/* Exact worst-case stream length for this shape and these parameters: the
 * header and tables plus every chunk at its raw length, each rounded up to
 * 16 bytes. Host only, pure; returns 0 for an invalid description.
 * Source: no page defines a size bound; it follows from the lossless stage
 * keeping a chunk raw whenever coding would not shorten it ("Beyond
 * Compression Ratio: High-Throughput KV Compression for Disaggregated LLM
 * Serving", Methodology: the LC-based backend of composed primitives), so the
 * stream never exceeds the quantized payload plus its tables. */
size_t kvc_max_compressed_bytes(const kvc_kv_desc *kv, const kvc_params *params);

/* (No page defines the workspace calls and the status read below: they
 * exist because this library allocates nothing and reports data-dependent
 * errors from the device.)
 *
 * Workspace bytes kvc_compress needs for this shape (DEVICE memory, 16-byte
 * aligned, caller-owned, contents need not be initialized). Returns 0 for an
 * invalid description. */
size_t kvc_workspace_bytes(const kvc_kv_desc *kv, const kvc_params *params);

/* Workspace bytes kvc_decompress needs to decode into `out` (DEVICE memory,
 * 16-byte aligned, caller-owned, contents need not be initialized): a status
 * word plus room to expand the meta chunks that used zero-byte elimination,
 * sized for the largest meta region any group size gives this shape
 * (head_dim / 8 bytes per vector, about 6% of the raw bf16 size). Returns 0
 * for an invalid description. */
size_t kvc_decompress_workspace_bytes(const kvc_kv_desc *out);

/* Source of the operation: "Beyond Compression Ratio: High-Throughput KV
 * Compression for Disaggregated LLM Serving", Abstract and Methodology (the
 * distribution transformation and the low-bit quantization fused in one
 * kernel with no intermediate tensor, then the LC-based lossless backend);
 * podcast page "FastKVComp: checking whether high-throughput KV compression
 * pays off", episode notes (the stages are a randomized Hadamard transform,
 * low-bit quantization and a lossless codec; the prefill side compresses the
 * cache before it crosses the link to the decode GPU).
 *
 * Compresses `kv` into `out` (DEVICE, out_capacity bytes, which must be at
 * least kvc_max_compressed_bytes). The stream length is written to the
 * header's stream_bytes field and, if out_bytes_dev (DEVICE) is not null, to
 * *out_bytes_dev. Stream layout (little-endian): 64-byte header; u64 chunk
 * table (bits 0..15 unpadded chunk size, bits 16..59 offset from the data base
 * in 16-byte units, bits 60..63 the chunk's lossless pipeline id, 0 for a
 * raw chunk); u32 token count per request; zero padding to 16 bytes;
 * the chunks, each zero-padded to 16 bytes. The code and meta regions are cut
 * into 16 KB chunks; a meta chunk covers group_size*bits/32 code chunks. Chunk
 * order (table and data): every code chunk, then every meta chunk. A chunk is
 * stored through a lossless pipeline (params->lossless) only if that makes it
 * shorter; in the code
 * region, only if moreover the padded bytes saved there are at least 1/64 of
 * the padded bytes from the first shrinking code chunk to the region's end
 * (the bytes that shift), else every code chunk is stored raw. The call
 * launches four kernels on `stream` (workspace clear; encode; table, meta
 * chunks and header; compaction, which returns at once unless code chunks
 * are stored eliminated), five for a paged pool whose page size is a power
 * of two from 8 to 512 (the blocks' load plans, written into the
 * workspace's meta region, before the encode). */
kvc_status kvc_compress(const kvc_kv_desc *kv, const kvc_params *params,
                        void *out, size_t out_capacity, uint64_t *out_bytes_dev,
                        void *workspace, size_t workspace_bytes,
                        kvc_stream_t stream);

/* Source of the operation: podcast page "FastKVComp: checking whether
 * high-throughput KV compression pays off", episode notes (the decode GPU
 * receives the compressed cache; encode plus decode time is what the wire
 * time saved must exceed; only the quantization loses information, so the
 * decoder inverts the lossless codec exactly and the transform up to the
 * quantization error).
 *
 * Decompresses the stream at `in` (DEVICE, in_bytes readable bytes) into the
 * slots described by `out`; workspace_bytes must be at least
 * kvc_decompress_workspace_bytes(out). Bits, group size and sign seed come from the
 * stream. The logical shape must match the stream's: layers, kv_heads,
 * head_dim and total tokens; a paged receiver must also match the stream's
 * request count and per-request token counts. The receiver's layout (dense or
 * paged, page table, strides) may differ from the sender's. A mismatch or any
 * inconsistency in the stream sets KVC_ERR_CORRUPT; reads stay inside
 * [in, in + in_bytes). Slots outside the described tokens are not written.
 * The call launches three kernels on `stream` (meta chunk expansion; decode
 * of the code chunks that used zero-byte elimination, which returns at once
 * unless the header flags some; decode of the raw code chunks). */
kvc_status kvc_decompress(const void *in, size_t in_bytes, const kvc_kv_desc *out,
                          void *workspace, size_t workspace_bytes,
                          kvc_stream_t stream);

/* Waits for `stream`, then returns the status word of the last call that used
 * this workspace (KVC_OK if it found no data-dependent error), or
 * KVC_ERR_CUDA if the stream reports a CUDA error. */
kvc_status kvc_stream_status(const void *workspace, kvc_stream_t stream);

/* Static, human-readable name of a status. */
const char *kvc_status_string(kvc_status status);

/* ---- Compression without a caller-provided workspace (the pages have no
 * counterpart; this is a deployment convenience).
 *
 * Some callers cannot hand out device memory at transfer time: a serving
 * engine typically gives nearly all of HBM to its paged KV pool when it
 * starts, and its transfer path must not ask any allocator for more (a
 * request may block, synchronize the device or fail under memory pressure at
 * exactly the moment a KV cache is leaving). kvc_compress_noalloc does the
 * same work as kvc_compress, with the same arguments and results, but its
 * workspace is a fixed block of the library's own static device memory
 * (KVC_NOALLOC_SCRATCH_BYTES per device, reserved when the library's module
 * is loaded on that device) instead of caller memory. It allocates nothing.
 *
 *  - Limit. Shapes whose kvc_workspace_bytes exceeds KVC_NOALLOC_SCRATCH_BYTES
 *    return KVC_ERR_CAPACITY before anything is enqueued. The workspace is
 *    about 16 KB per 16 KB of meta (fp16 scale and zero per group), so 16 MiB
 *    holds e.g. 32 layers x 8 kv_heads x 4096 tokens x head_dim 128 at group
 *    128 (8.1 MiB), not at group 64 (16.1 MiB).
 *  - Set-up. The first call in each CUDA context (per device, with that
 *    device current) looks up the block's device address and keeps it for
 *    that context; later calls in the same context only compare the current
 *    context's ID with the kept one. After a device reset (a new primary
 *    context) the next call looks the address up again. Make the first call
 *    in a context before any stream capture on the device. A failed look-up
 *    returns KVC_ERR_CUDA.
 *  - Status. If status_dev (DEVICE, 4 bytes, 4-byte aligned) is not null, the
 *    call's status word is copied there on `stream` after the encode; pass
 *    status_dev to kvc_stream_status() to read it.
 *  - Concurrency. There is one block per device, so calls on the same device
 *    must not overlap: a call enqueued on one stream while another is still
 *    running on a different stream (or from another thread) races on the
 *    block and corrupts both streams. Serialize them, e.g. on one stream. */
#define KVC_NOALLOC_SCRATCH_BYTES (16u << 20)
kvc_status kvc_compress_noalloc(const kvc_kv_desc *kv, const kvc_params *params,
                                void *out, size_t out_capacity,
                                uint64_t *out_bytes_dev, uint32_t *status_dev,
                                kvc_stream_t stream);

/* Unfused baseline, for measurement only ("Beyond Compression Ratio:
 * High-Throughput KV Compression for Disaggregated LLM Serving", Abstract:
 * the fused transform + quantization kernel is compared against separate
 * kernels). kvc_compress_unfused writes exactly the stream kvc_compress
 * writes, with the same arguments and errors, but runs the transform (signs
 * and Walsh-Hadamard) and the quantization as two kernels with the
 * transformed vectors in HBM between them (fp32, 4 * head_dim bytes per
 * vector, at the end of the workspace). workspace_bytes must be at least
 * kvc_unfused_workspace_bytes(kv, params) (0 for an invalid description). */
size_t kvc_unfused_workspace_bytes(const kvc_kv_desc *kv, const kvc_params *params);
kvc_status kvc_compress_unfused(const kvc_kv_desc *kv, const kvc_params *params,
                                void *out, size_t out_capacity,
                                uint64_t *out_bytes_dev, void *workspace,
                                size_t workspace_bytes, kvc_stream_t stream);

/* ---- Attention over the compressed cache (the first page's ZipFusion
 * abstract: decode attention that consumes the compressed KV cache in
 * registers, without decompressing it to memory first).
 *
 * One decode step of grouped-query attention for every layer and request of
 * a compressed cache: query head j of layer l and request r attends to kv
 * head j / q_per_kv over the request's tokens,
 *   out = sum_t softmax_t(scale * q . k_t) v_t,
 * with k_t, v_t the stream's decoded vectors without the decoder's final
 * bf16 rounding (its fp32 transformed values mapped back by the inverse
 * transform). The kernels score and accumulate in the transformed domain
 * (q . k = (H D q) . y / d) and invert the transform once per query head, so
 * no decoded key or value is written to memory.
 *
 * The stream must describe a cache of this shape with these bits, group and
 * quantizer (ASYM and SYM decode alike, either matches the other), head_dim
 * 128, either sign mode, and store every code chunk raw (the header flag clear, the
 * usual case; KVC_ERR_CORRUPT in the status word otherwise); its meta chunks
 * may use any lossless pipeline. q: DEVICE bf16 [layers][n_requests]
 * [kv_heads * q_per_kv][128], contiguous; out: DEVICE fp32 of the same shape
 * (zeros for a request without tokens). seq_lens: HOST, the stream's
 * per-request token counts. q_per_kv 1 to 8. The workspace holds the
 * status word, the expanded meta chunks, the split partials and (tensor-core
 * path) each (layer, request, kv head)'s prepared query fragments. */
typedef struct {
  int32_t layers;
  int32_t kv_heads;
  int32_t head_dim;           /* 128 */
  int32_t q_per_kv;           /* 1 .. 8 (e.g. 4 for 32 query / 8 kv heads) */
  int32_t bits;               /* as compressed */
  int32_t group_size;         /* as compressed */
  int32_t quant;              /* as compressed (KVC_QUANT_*; ASYM and SYM alike) */
  int32_t kernel;             /* 0: tensor cores (2- and 4-bit ASYM / SYM codes, 2..8
                                 query heads per kv head), CUDA cores otherwise;
                                 1: CUDA cores always (for comparison) */
  int32_t n_requests;         /* 1 .. KVC_MAX_REQUESTS */
  float scale;                /* e.g. 1 / sqrt(head_dim) */
  const int32_t *seq_lens;    /* HOST [n_requests] */
  const void *q;              /* DEVICE bf16 */
  float *out;                 /* DEVICE fp32 */
} kvc_attn_desc;
size_t kvc_attend_workspace_bytes(const kvc_attn_desc *attn);
kvc_status kvc_attend(const void *in, size_t in_bytes, const kvc_attn_desc *attn,
                      void *workspace, size_t workspace_bytes, kvc_stream_t stream);

/* Measurement only (no page defines these; they let a benchmark time each
 * kernel of a call with CUDA events on the call's own stream). The same work
 * and results as kvc_compress / kvc_decompress, with n_events == 5 caller-
 * created CUDA events (cudaEvent_t, passed as void *) recorded on `stream`:
 * events[0] before the call's first kernel and events[i] after its i-th
 * kernel. Compress: workspace clear, encode, finishing (table, meta chunks,
 * header), compaction. Decompress: status clear, meta chunk expansion,
 * decode of eliminated code chunks, decode. Attend: status clear, meta chunk
 * expansion, attention (split-K), combination. A kernel that a call does not
 * need gets an empty interval. The kernels of a timed call start in plain
 * stream order, without overlapping the previous kernel's tail, so a timed
 * call can take a few microseconds longer than an ordinary one. Other
 * n_events or a null event: KVC_ERR_INVALID_ARG. */
kvc_status kvc_compress_timed(const kvc_kv_desc *kv, const kvc_params *params, void *out,
                              size_t out_capacity, uint64_t *out_bytes_dev, void *workspace,
                              size_t workspace_bytes, void *const *events, int n_events,
                              kvc_stream_t stream);
kvc_status kvc_decompress_timed(const void *in, size_t in_bytes, const kvc_kv_desc *out,
                                void *workspace, size_t workspace_bytes, void *const *events,
                                int n_events, kvc_stream_t stream);
kvc_status kvc_attend_timed(const void *in, size_t in_bytes, const kvc_attn_desc *attn,
                            void *workspace, size_t workspace_bytes, void *const *events,
                            int n_events, kvc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KVC_H */
