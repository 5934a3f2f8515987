/*
 * kvc_oracle.h — plain, slow CPU oracle of the FastKVComp-style KV-cache codec.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package entry's smoke check and
 * the benchmark's CPU-baseline leg may call, link or execute this code. The
 * product path (the CUDA library) never uses it, and the two share no code:
 * every definition below is written independently of the CUDA sources.
 *
 * What it computes (sources: "Beyond Compression Ratio: High-Throughput KV
 * Compression for Disaggregated LLM Serving", Abstract and Methodology; the
 * podcast page "FastKVComp: checking whether high-throughput KV compression
 * pays off", episode notes):
 *   encode = random +-1 signs, Hadamard transform over head_dim, low-bit group
 *            quantization, then a lossless codec over the quantized payload;
 *   decode = the exact inverse of the lossless codec, then dequantization,
 *            inverse Hadamard and unsigning.
 * The pages name the stages only. Every exact rule here (butterfly order, sign
 * generator, meta rounding, stream format) is a stated reading, listed in the
 * design notes with its justification.
 *
 * Floating point: the method's arithmetic is fp32 with one IEEE rounding per
 * operation (no fused multiply-add). Build with -ffp-contract=off
 * -fno-fast-math. Status codes use the same numbering as the library ABI.
 */
#ifndef KVC_ORACLE_H
#define KVC_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ORC_OK = 0,
  ORC_ERR_INVALID_ARG = 1,
  ORC_ERR_UNSUPPORTED = 2,
  ORC_ERR_CAPACITY = 3,
  ORC_ERR_NONFINITE = 4,
  ORC_ERR_RANGE = 5,
  ORC_ERR_CORRUPT = 6
};

#define ORC_CHUNK 16384      /* lossless chunk length in bytes            */
#define ORC_BITMAP 2048      /* zero-byte-elimination bitmap bytes        */
#define ORC_BITMAP2 256      /* second-level bitmap bytes (pipelines 2, 3) */
#define ORC_HEADER 64        /* stream header bytes                       */
#define ORC_MAGIC 0x3143564Bu /* "KVC1" little-endian                    */
#define ORC_MAX_D 256
#define ORC_MAX_SEG 32       /* code chunks per segment: g * b / 32 <= 128 * 8 / 32 */
#define ORC_QUANT_ASYM 0      /* reading R5: min/max, zero and scale        */
#define ORC_QUANT_SYM 1       /* reading R19: symmetric absmax              */
#define ORC_QUANT_FP4 2       /* reading R22: e2m1 codes, dual scales (4 bit) */
#define ORC_SIGNS_GLOBAL 0    /* reading R3: one diagonal for the tensor    */
#define ORC_SIGNS_PER_VECTOR 1 /* reading R20: one per (layer, kv, head)   */

/* ---- scalar building blocks (each pinned by its own test) ---------------- */
uint64_t orc_splitmix64_next(uint64_t *state);
void orc_sign_words(uint64_t seed, int d, uint64_t *words);
void orc_sign_words_at(uint64_t seed, int d, uint64_t index, uint64_t *words);
void orc_fwht(float *y, int d);
int orc_meta_shift(int d);
float orc_bf16_to_f32(uint16_t b);
uint16_t orc_f32_to_bf16_rne(float x);
float orc_f16_to_f32(uint16_t h);
uint16_t orc_f32_to_f16_rd(float x);
uint16_t orc_f32_to_f16_ru(float x);

/* ---- one vector ----------------------------------------------------------- */
int orc_quantize_scalar(float y, float zf, float r, int qmax);
int orc_quantize_scalar_sym(float y, float r, int bits);
int orc_quantize_vector_q(const uint16_t *x, int d, int bits, int g, int quant,
                          const uint64_t *sign_words, uint8_t *codes,
                          uint8_t *meta);
int orc_quantize_vector(const uint16_t *x, int d, int bits, int g,
                        const uint64_t *sign_words, uint8_t *codes,
                        uint8_t *meta);
void orc_dequantize_vector(const uint8_t *codes, const uint8_t *meta, int d,
                           int bits, int g, const uint64_t *sign_words,
                           uint16_t *xhat);
void orc_dequantize_vector_f64(const uint8_t *codes, const uint8_t *meta, int d,
                               int bits, int g, const uint64_t *sign_words,
                               double *xhat);
void orc_dequantize_vector_q(const uint8_t *codes, const uint8_t *meta, int d, int bits, int g,
                             int quant, const uint64_t *sign_words, uint16_t *xhat);
void orc_dequantize_vector_f64_q(const uint8_t *codes, const uint8_t *meta, int d, int bits,
                                 int g, int quant, const uint64_t *sign_words, double *xhat);
float orc_e2m1_to_f32(int code);
int orc_f32_to_e2m1_rne(float p);
float orc_e4m3_to_f32(int b);
int orc_f32_to_e4m3_ru(float x);
void orc_pack_codes(const uint8_t *q, int d, int bits, uint8_t *packed);
void orc_unpack_codes(const uint8_t *packed, int d, int bits, uint8_t *q);

/* ---- lossless stage on one chunk ------------------------------------------ */
void orc_bitplane_shuffle(const uint8_t *in, uint8_t *out);
void orc_bitplane_unshuffle(const uint8_t *in, uint8_t *out);
uint32_t orc_lossless_encode_chunk(const uint8_t *in, uint32_t len,
                                   uint8_t *out);
int orc_lossless_decode_chunk(const uint8_t *in, uint32_t size, uint32_t len,
                              uint8_t *out);

/* ---- composable lossless pipelines (LC-style search, reading R17) --------- */
/* Pipeline ids of a stored chunk (bits 60..63 of its table entry):
 *   0  bit-plane shuffle, zero-byte elimination with a 2048-byte bitmap
 *   1  XOR of each word with the previous word, restarting at every run of
 *      32 vectors (meta chunks), then as 0
 *   2  bit-plane shuffle, two-level zero-byte elimination (the 2048-byte
 *      bitmap itself zero-byte eliminated under a 256-byte bitmap)
 *   3  the XOR of 1, then as 2
 * A raw chunk (size == length) has id 0. */
#define ORC_PIPE_ZE 0
#define ORC_PIPE_XOR_ZE 1
#define ORC_PIPE_ZE2 2
#define ORC_PIPE_XOR_ZE2 3
/* Encoder modes (orc_desc.lossless): FIXED uses pipeline 0 only; SEARCH picks,
 * per full chunk, the shortest candidate (code chunks: 0, 2; meta chunks with
 * at least two groups per vector: 0..3; other meta chunks: 0, 1), ties to the
 * lower id; NONE stores every chunk raw. */
#define ORC_LOSSLESS_FIXED 0
#define ORC_LOSSLESS_SEARCH 1
#define ORC_LOSSLESS_NONE 2
void orc_xor_words(uint8_t *chunk, uint32_t n_words, int run_words);
void orc_unxor_words(uint8_t *chunk, uint32_t n_words, int run_words);
uint32_t orc_ze2_encode(const uint8_t *shuffled, uint8_t *out);
int orc_ze2_decode(const uint8_t *in, uint32_t size, uint8_t *shuffled);
uint32_t orc_chunk_encode_pipe(const uint8_t *in, int pipe, int words_per_vector,
                               uint8_t *out);
int orc_chunk_decode_pipe(const uint8_t *in, uint32_t size, uint32_t len, int pipe,
                          int words_per_vector, uint8_t *out);
uint32_t orc_chunk_encode_select(const uint8_t *in, uint32_t len, int is_meta,
                                 int words_per_vector, int mode, uint8_t *out,
                                 int *pipe);

/* ---- stream --------------------------------------------------------------- */
typedef struct {
  int32_t bits, group, head_dim, layers, kv_heads, origin, n_requests;
  uint64_t sign_seed;
  const uint32_t *token_lens; /* [n_requests] tokens per request          */
  int32_t lossless;           /* ORC_LOSSLESS_* (encoder only)            */
  int32_t quant;              /* ORC_QUANT_* (header flags bits 1..2)     */
  int32_t signs;              /* ORC_SIGNS_* (header flags bit 3)         */
} orc_desc;

typedef struct {
  uint64_t V;             /* vectors                                       */
  uint32_t code_bytes;    /* packed code bytes per vector                  */
  uint32_t meta_bytes;    /* meta bytes per vector                         */
  uint32_t vec_per_code;  /* vectors per code chunk                        */
  uint32_t code_per_seg;  /* code chunks per meta chunk (segment)          */
  uint64_t n_code, n_meta, n_chunks, n_seg;
  uint64_t data_base;     /* byte offset of the first chunk                */
  uint64_t max_bytes;     /* worst-case stream length                      */
} orc_layout;

int orc_check_desc(const orc_desc *d);
int orc_layout_of(const orc_desc *d, orc_layout *lay);
uint64_t orc_max_compressed_bytes(const orc_desc *d);

/* Stream chunk index of code chunk c and of meta chunk s. */
uint64_t orc_code_chunk_index(const orc_layout *lay, uint64_t c);
uint64_t orc_meta_chunk_index(const orc_layout *lay, uint64_t s);

/* Encodes segment s from its vectors (vectors [s*VM, min((s+1)*VM, V)) in
 * logical order, d bf16 each). Writes the segment's chunks, unpadded, back to
 * back into chunks (capacity (code_per_seg+1)*ORC_CHUNK), their sizes into
 * sizes[] and their pipeline ids into pipes[] (code chunks first, then the
 * meta chunk), per chunk as chosen by d->lossless (the code-region rule R16
 * is applied by orc_compress over the whole stream, not here). Returns the
 * status and the number of chunks through n_out. */
int orc_encode_segment(const orc_desc *d, uint64_t s, const uint16_t *vectors,
                       uint8_t *chunks, uint32_t *sizes, uint8_t *pipes, uint32_t *n_out);
int orc_decode_segment(const orc_desc *d, uint64_t s, const uint8_t *chunks,
                       const uint32_t *sizes, const uint8_t *pipes, uint16_t *vectors);

/* Reading R16: 1 iff some code chunk shrinks and the padded bytes saved are
 * at least 1/64 of the padded bytes from the first shrinking code chunk on. */
int orc_code_elim_pays(const uint32_t *sizes, const uint32_t *lens, uint64_t n_code);
int orc_compress(const orc_desc *d, const uint16_t *vectors, uint8_t *out,
                 uint64_t capacity, uint64_t *out_bytes);
int orc_decompress(const uint8_t *stream, uint64_t stream_bytes,
                   const orc_desc *expect, uint16_t *vectors);

/* The same two calls with their per-segment loop spread over n_threads
 * POSIX threads (segment s on thread s mod n_threads). Segments are
 * independent and every result is placed by its segment index, so the
 * output and status equal the single-thread calls'. */
#define ORC_MAX_THREADS 256
int orc_compress_mt(const orc_desc *d, const uint16_t *vectors, uint8_t *out,
                    uint64_t capacity, uint64_t *out_bytes, int n_threads);
int orc_decompress_mt(const uint8_t *stream, uint64_t stream_bytes,
                      const orc_desc *expect, uint16_t *vectors, int n_threads);

/* The stream's decoded vectors without the final bf16 rounding, in double
 * ([V][d], orc_dequantize_vector_f64). */
int orc_decode_values_mt(const uint8_t *stream, uint64_t stream_bytes,
                         const orc_desc *expect, double *vals, int n_threads);

/* Reading R18: one decode step of grouped-query attention over the stream's
 * keys and values (all layers and requests), in double; see kvc_oracle.c. */
int orc_attend(const uint8_t *stream, uint64_t stream_bytes, const orc_desc *expect,
               const uint16_t *q, int q_per_kv, double scale, double *out, int n_threads);

/* ---- layouts: logical vector order [layer][kv][head][request][token] ------ */
void orc_gather_dense(const uint16_t *base, int layers, int kv_heads,
                      int64_t tokens, int d, int64_t s_layer, int64_t s_kv,
                      int64_t s_head, int64_t s_token, uint64_t v_begin,
                      uint64_t v_end, uint16_t *out);
void orc_gather_paged(const uint16_t *pool, int layers, int kv_heads, int d,
                      int64_t s_layer, int64_t s_page, int64_t s_kv,
                      int64_t s_head, int64_t s_slot, int page_tokens,
                      int n_requests, const uint32_t *seq_lens,
                      const int32_t *page_table, int64_t pt_stride,
                      uint64_t v_begin, uint64_t v_end, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif
