// Decode kernels (D1..D9): parse and validate the stream -> undo zero-byte
// elimination and the bit-plane shuffle of the chunks that used them ->
// unpack -> dequantize -> fp32 Walsh-Hadamard (the encoder's butterfly) ->
// scale by 2^-log2(d) -> unsign -> bf16 -> store (tensor copies for a dense
// receiver with a tensor map, else 16-byte stores through the receiver's
// layout or page table). The decoder is the inverse path the podcast page
// "FastKVComp: checking whether high-throughput KV compression pays off"
// (episode notes) places on the decode GPU.
//
// Three kernels per call:
//  meta_expand_kernel   expands the meta chunks that used elimination into
//                       the workspace;
//  elim_decode_kernel   decodes the (rare) code chunks that used elimination,
//                       spread over the CTAs; returns at once unless the
//                       header says there are some;
//  decode_kernel        decodes every raw code chunk. The chunk table stores
//                       every chunk's offset, so each CTA takes a contiguous
//                       range of code chunks (tiles) and reads its chunks
//                       directly: no scan, no inter-CTA waits. Every table
//                       entry is checked against its predecessor (offset =
//                       previous offset + padded previous size) by the CTA
//                       whose range holds it, so a consistent table is a
//                       prefix sum. Warps decode blocks of 32 vectors
//                       independently.
#pragma once

#include "kvc_encode.cuh"

namespace kvc {

constexpr int kDecWarps = 12;
constexpr int kDecThreads = kDecWarps * 32;

struct DecCtl {
  uint64_t cbar[kDecWarps][2];  // per-warp code + meta blocks loaded (two buffers)
  uint32_t red[kDecThreads / 32];
  uint32_t hdr_ok;
  uint32_t bits, group, n_req_stream, n_chunks, code_elim, vec_signs, quant;
  uint64_t data_base, stream_bytes, seed;
  alignas(16) uint32_t mask[128];  // read as uint4
};

// Shared memory: per-warp output staging | per-warp code blocks | per-warp
// meta blocks | control | request prefix (paged).
template <int D>
struct DecSmem {
  static constexpr size_t WBUF = size_t(D / 64) * 4096;    // 32 rows, 128-byte swizzled halves
  // code block of 32 vectors at up to 4 bits (an 8-bit block fills both of a
  // warp's buffers and is loaded single-buffered)
  static constexpr size_t BLK = 32 * size_t(D) / 2;
  static constexpr size_t MBLK = 32 * (size_t(D) / 32) * 4;  // widest meta block (group 32)
  static constexpr size_t rows = 0;
  static constexpr size_t code = rows + kDecWarps * WBUF;
  static constexpr size_t meta = code + 2 * kDecWarps * BLK;
  static constexpr size_t ctl = meta + 2 * kDecWarps * MBLK;
  static constexpr size_t cum = ctl + ((sizeof(DecCtl) + 15) & ~size_t(15));
  static constexpr size_t bytes(bool paged) {
    return cum + (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
  }
};

__device__ __forceinline__ uint32_t ld_u32(const uint8_t *p) {
  return *reinterpret_cast<const uint32_t *>(p);
}
__device__ __forceinline__ uint64_t ld_u64(const uint8_t *p) {
  return *reinterpret_cast<const uint64_t *>(p);
}

// D1: the header (reading R12) against the receiver's description.
struct StreamHdr {
  uint32_t ok, bits, group, n_req, n_chunks, code_elim, vec_signs, quant;
  uint64_t data_base, stream_bytes, seed;
};
template <int D>
__device__ __forceinline__ StreamHdr parse_header(const DecArgs &a) {
  constexpr uint32_t kLog2D = D == 64 ? 6 : D == 128 ? 7 : 8;
  StreamHdr r{};
  const uint8_t *h = a.in;
  if (a.in_bytes < kHeader) return r;
  const uint32_t bits = h[8], k = h[9], group = ld_u32(h + 12);
  // flags: bit 0 code chunks eliminated, bits 1..2 the quantizer (0 or 1;
  // both decode alike), bit 3 per-vector sign diagonals, the rest zero
  const uint32_t flags = h[11], quant = (flags >> 1) & 3u;
  bool ok = ld_u32(h) == kMagic && (ld_u32(h + 4) & 0xFFFFu) == 1 && (flags & 0xF0u) == 0 &&
            quant <= 2 && (quant != 2 || bits == 4) &&
            (ld_u32(h + 4) >> 16) == kHeader && (bits == 2 || bits == 4 || bits == 8) &&
            k == kLog2D / 2 &&
            (group == 32 || group == 64 || group == 128) && group <= D &&
            ld_u32(h + 16) == a.layers && ld_u32(h + 20) == 2 && ld_u32(h + 24) == a.kv_heads &&
            ld_u32(h + 28) == a.head_dim && ld_u64(h + 32) == a.tokens;
  if (!ok) return r;
  const uint32_t n_req = ld_u32(h + 48), n_chunks = ld_u32(h + 52);
  const uint64_t stream_bytes = ld_u64(h + 56);
  const uint64_t cb = uint64_t(D) * bits / 8, mbv = uint64_t(D / group) * 4;
  const uint64_t n_code = (uint64_t(a.V) * cb + kChunk - 1) / kChunk;
  const uint64_t n_meta = (uint64_t(a.V) * mbv + kChunk - 1) / kChunk;
  const uint64_t base = round16(kHeader + 8ull * n_chunks + 4ull * n_req);
  ok = n_chunks == n_code + n_meta && base <= stream_bytes && stream_bytes <= a.in_bytes &&
       (!a.paged_receiver || n_req == a.n_req);
  r.ok = ok;
  r.bits = bits;
  r.group = group;
  r.n_req = n_req;
  r.n_chunks = n_chunks;
  r.data_base = base;
  r.stream_bytes = stream_bytes;
  r.seed = ld_u64(h + 40);
  r.code_elim = flags & 1u;
  r.vec_signs = (flags >> 3) & 1u;
  r.quant = quant;
  return r;
}

template <int D, int BITS, int G, bool kFp4 = false>
struct Dec : Cfg<D, BITS, G> {
  using C = Cfg<D, BITS, G>;

  // Reading R9: y^ = fl(zf + fl(q*sf)), the encoder's butterfly, then
  // x^ = bf16_RNE(sign * (u * 2^-log2 d)). Computed here in an exactly
  // equivalent order: zf and sf are pre-scaled by 2^-log2 d (exact), so every
  // value of the butterfly is the reference value times 2^-log2 d; no value
  // can become subnormal (all are 0 or at least 2^-28 in magnitude: fp16
  // meta values are multiples of 2^-24), so scaling commutes with every
  // rounding. q*sf is exact (q < 16 times an fp16 value needs at most 15
  // significant bits), so one fused multiply-add equals fl(zf + fl(q*sf)).
  // The vector is held as pairs (c, c + d/2) like the encoder's.
  // FP4: the hardware's e2m1 -> f16 conversion turns each code byte (two
  // adjacent channels) into their values, exact in f16 and in fp32.
  template <class SG>
  static __device__ __forceinline__ void vector(const uint8_t *codes, const uint8_t *meta,
                                                const SG &sg, uint32_t (&out)[D / 2]) {
    float zf[kFp4 ? 1 : C::NG], sf[kFp4 ? 1 : C::NG];
    float S[kFp4 ? 2 * C::NG : 1];  // FP4 (reading R22): s1 * s2 per half-group, x 2^-log2 d
    const float up = float(1 << C::K) / float(D);
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      const uint32_t m = reinterpret_cast<const uint32_t *>(meta)[g];
      const float s = __fmul_rn(__half2float(__ushort_as_half(uint16_t(m & 0xFFFFu))), up);
      if constexpr (kFp4) {
        S[2 * g] = __fmul_rn(e4m3_value((m >> 16) & 0xFFu), s);
        S[2 * g + 1] = __fmul_rn(e4m3_value(m >> 24), s);
      } else {
        sf[g] = s;
        zf[g] = __fmul_rn(__half2float(__ushort_as_half(uint16_t(m >> 16))), up);
      }
    }
    Pairs<D> y;
    if constexpr (kFp4) {  // e2m1(code) * S, exact
      static_assert(BITS == 4, "FP4 codes are 4-bit");
#pragma unroll
      for (int q4 = 0; q4 < C::CW / 4; ++q4) {
        const uint4 v = reinterpret_cast<const uint4 *>(codes)[q4];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // byte k of word 4 q4 + e: channels c, c + 1
            const int c = 8 * (4 * q4 + e) + 2 * k;
            const float2 f = e2m1x2_to_float2(w[e] >> (8 * k));
            y.at(c) = f.x;
            y.at(c + 1) = f.y;
          }
      }
#pragma unroll
      for (int j = 0; j < D / 2; ++j) {
        const int ha = j / (G / 2), hb = (j + D / 2) / (G / 2);
        y.p[j] = mul2(y.p[j], make_float2(S[ha], S[hb]));
      }
    } else {
      // Code -> float: a byte permute puts the code in the low byte of the bit
      // pattern 0x4B4000qq = 1.5*2^23 + q; subtracting 1.5*2^23 gives q exactly.
      // Pair j takes channel j from the first half of the code words and
      // channel j + d/2 from the second; each 16-byte piece of either half is
      // loaded when the pairs reach it.
      constexpr int per_word = 32 / BITS;          // codes per word
      constexpr int per_byte = 8 / BITS;
      constexpr int HW = C::CW / 2;                // words per half
      constexpr int PW = HW < 4 ? HW : 4;          // words per piece
      constexpr int NP = HW / PW;                  // pieces per half
      constexpr int JP = PW * per_word;            // pairs per piece
      constexpr uint32_t kMagicBits = 0x4B400000u;
      constexpr float kMagic = 12582912.0f;
      const float2 mag = make_float2(kMagic, kMagic);
#pragma unroll
      for (int piece = 0; piece < NP; ++piece) {
        uint32_t lo[PW], hi[PW];
        if constexpr (PW == 4) {
          const uint4 a = reinterpret_cast<const uint4 *>(codes)[piece];
          const uint4 b = reinterpret_cast<const uint4 *>(codes)[NP + piece];
          lo[0] = a.x, lo[1] = a.y, lo[2] = a.z, lo[3] = a.w;
          hi[0] = b.x, hi[1] = b.y, hi[2] = b.z, hi[3] = b.w;
        } else {
          const uint4 a = reinterpret_cast<const uint4 *>(codes)[0];
          lo[0] = a.x, lo[1] = a.y, hi[0] = a.z, hi[1] = a.w;
        }
        auto code_float = [&](const uint32_t (&w)[PW], int c) -> float {
          const int W = c / per_word, r = c % per_word, k = r / per_byte, e = r % per_byte;
          const uint32_t part =
              (w[W] >> (e * BITS)) & (BITS == 8 ? 0xFFFFFFFFu : BITS == 4 ? 0x0F0F0F0Fu : 0x03030303u);
          return __uint_as_float(__byte_perm(part, kMagicBits, 0x7640 | k));
        };
#pragma unroll
        for (int i = 0; i < JP; ++i) {
          const int j = piece * JP + i;
          const int ga = j / G, gb = (j + D / 2) / G;
          const float2 q = sub2(make_float2(code_float(lo, i), code_float(hi, i)), mag);
          y.p[j] = fma2(q, make_float2(sf[ga], sf[gb]), make_float2(zf[ga], zf[gb]));
        }
      }
    }
    fwht_pairs<D>(y);
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
      const uint4 m4 = sg.quad(q);
      const uint32_t m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = 4 * q + e;
        const __nv_bfloat162 b = __floats2bfloat162_rn(y.at(2 * k), y.at(2 * k + 1));
        out[k] = *reinterpret_cast<const uint32_t *>(&b) ^ m[e];
      }
    }
  }
};

// D5..D8 of vector v with the global sign diagonal (masks in shared
// memory). A stream with per-vector diagonals (reading R20) is corrected in
// the staging buffer by fix_row_signs.
template <int D, int BITS, int G, bool kFp4>
__device__ __forceinline__ void decode_vector(const uint32_t *mask,
                                              const uint8_t *codes, const uint8_t *meta,
                                              uint32_t (&out)[D / 2]) {
  Dec<D, BITS, G, kFp4>::vector(codes, meta, GlobalSigns{mask}, out);
}

// This lane's staged row XOR the global masks XOR the masks of its vector's
// own diagonal ((layer, kv, head) index `index`). Not inlined: inlined, the
// untaken branch alone measured 7% on the default decode (register and
// schedule changes of the surrounding loop).
template <int D>
__device__ __noinline__ void fix_row_signs(uint8_t *stage, const uint32_t *mask, uint64_t seed,
                                           uint32_t index) {
  const int lane = threadIdx.x & 31;
  VectorSigns<D> sg;
  vec_sign_words<D>(seed, index, sg.S);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    uint4 *p = reinterpret_cast<uint4 *>(stage + swz_offset(lane, c));
    uint4 w = *p;
    w.x ^= mask[4 * c] ^ sg.word(4 * c);
    w.y ^= mask[4 * c + 1] ^ sg.word(4 * c + 1);
    w.z ^= mask[4 * c + 2] ^ sg.word(4 * c + 2);
    w.w ^= mask[4 * c + 3] ^ sg.word(4 * c + 3);
    *p = w;
  }
}

// Writes this lane's decoded row (bf16 words `out`) into the warp's staging
// buffer as row `lane` of the 128-byte swizzle (conflict-free).
template <int D>
__device__ __forceinline__ void stage_row(const uint32_t (&out)[D / 2], uint8_t *stage) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < D / 8; ++c)
    *reinterpret_cast<uint4 *>(stage + swz_offset(lane, c)) =
        make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
}

// Dense receiver with a tensor map (tokens % 32 == 0, so the block is 32
// vectors of one head row): lane 0 stores the staged block with one tensor
// copy per 64-channel half.
template <int D>
__device__ __forceinline__ void store_block_tma(const DenseLayout &lay, const uint32_t (&out)[D / 2],
                                                uint32_t v0, uint8_t *stage, bool &stage_busy,
                                                const DecArgs &a, uint32_t vec_signs,
                                                const uint32_t *mask, uint64_t seed) {
  const int lane = threadIdx.x & 31;
  if (stage_busy && lane == 0) bulk_wait_read<0>();  // the previous block's stores have read it
  __syncwarp();
  stage_row<D>(out, stage);
  if (vec_signs) fix_row_signs<D>(stage, mask, seed, fdiv(a.tdiv, v0 + lane));
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    const uint32_t lkh = fdiv(lay.T, v0), t0 = v0 - lkh * lay.T.d;
    const uint32_t lk = fdiv(lay.H, lkh), h = lkh - lk * lay.H.d;
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh)
      tma_store_5d(&lay.tmap, hh * 64, int(t0), int(h), int(lk & 1u), int(lk >> 1), stage + hh * 4096);
    bulk_commit();
  }
  stage_busy = true;
}

template <int D, int BITS, int G, class Layout, bool kNarrow, bool kFp4 = false>
__device__ void decode_body(const DecArgs &a, const Layout &lay, DecCtl *ctl, uint8_t *smem,
                            const uint32_t *cum) {
  using C = Cfg<D, BITS, G>;
  using S = DecSmem<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t V = a.V;
  const uint32_t n_tiles = (V + C::VC - 1) / C::VC;
  const uint32_t t0 = uint32_t(uint64_t(blockIdx.x) * n_tiles / gridDim.x);
  const uint32_t t1 = uint32_t(uint64_t(blockIdx.x + 1) * n_tiles / gridDim.x);
  if (t0 >= t1) return;
  const uint8_t *in = a.in;
  const uint64_t base = ctl->data_base;
  const uint64_t limit = min(a.in_bytes, ctl->stream_bytes);
  const uint8_t *table = in + kHeader;
  uint8_t *cbuf = smem + S::code + 2 * warp * S::BLK;
  uint8_t *mbuf = smem + S::meta + 2 * warp * S::MBLK;
  const uint32_t seg0 = t0 / C::R, seg1 = (t1 - 1) / C::R;

  // D2: table entries of this range (code chunks t0..t1-1, meta chunks
  // seg0..seg1): each offset continues its predecessor, stays inside the
  // stream, and each size is the chunk's raw length or a valid eliminated
  // size (full chunks only); the last chunk ends the stream.
  // Pipeline ids (reading R17): 0 on a raw chunk; 0 or 2 on a code chunk;
  // 0..3 on a meta chunk. Sizes: at least the bitmap of the chosen form.
  auto entry_ok = [&](uint64_t i, uint32_t len, bool is_meta) {
    const uint64_t e = ld_u64(table + 8 * i);
    const uint64_t off = entry_offset(e);
    const uint32_t size = entry_size(e), pipe = entry_pipe(e);
    uint64_t expect = 0;
    if (i > 0) {
      const uint64_t p = ld_u64(table + 8 * (i - 1));
      expect = entry_offset(p) + round16(entry_size(p));
    }
    const bool pipe_ok = size == len ? pipe == 0 : (pipe <= 3 && (is_meta || !(pipe & 1u)));
    const uint32_t min_size = (pipe & 2u) ? uint32_t(kBitmap2) : uint32_t(kBitmap);
    bool ok = off == expect && base + off + round16(size) <= limit && pipe_ok &&
              (size == len || (len == uint32_t(kChunk) && size >= min_size && size < len));
    if (i + 1 == ctl->n_chunks) ok = ok && base + off + round16(size) == ctl->stream_bytes;
    return ok;
  };
  // Also counts the range's code chunks that used zero-byte elimination
  // (usually none: then phase 1 and the per-block raw test are skipped).
  bool any_elim;
  {
    uint32_t bad = 0, elim = 0;
    for (uint32_t t = t0 + tid; t < t1; t += kDecThreads) {
      const uint32_t len = min(uint32_t(C::VC), V - t * C::VC) * C::CB;
      bad |= !entry_ok(t, len, false);
      elim |= entry_size(ld_u64(table + 8 * uint64_t(t))) != len;
    }
    for (uint32_t s = seg0 + tid; s <= seg1; s += kDecThreads)
      bad |= !entry_ok(uint64_t(n_tiles) + s, min(uint32_t(C::VM), V - s * C::VM) * C::MB, true);
    const uint32_t sum = block_sum<kDecThreads>(bad | (elim << 16), ctl->red);
    any_elim = sum != 0;
    // such chunks must be announced by the header (elim_decode_kernel
    // decodes them only then)
    if ((sum & 0xFFFFu) || (any_elim && !ctl->code_elim)) {
      if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
      return;
    }
  }

  // D3 for meta: a raw meta chunk is read in place; an eliminated one was
  // expanded into the workspace by meta_expand_kernel.
  auto meta_src = [&](uint32_t v0) -> const uint8_t * {
    const uint32_t s = v0 / C::VM;
    const uint64_t me = ld_u64(table + 8 * (uint64_t(n_tiles) + s));
    const uint32_t mlen = min(uint32_t(C::VM), V - s * C::VM) * C::MB;
    const uint8_t *chunk = entry_size(me) == mlen ? in + base + entry_offset(me)
                                                  : a.ws_meta + uint64_t(s) * kChunk;
    return chunk + uint64_t(v0 - s * C::VM) * C::MB;
  };
  // Lane 0 starts the loads of a block's meta bytes and, unless they are
  // already in shared memory (csrc null), its code bytes, into buffer k.
  auto issue = [&](uint32_t v0, uint32_t nvec, const uint8_t *csrc, uint32_t k) {
    if (lane == 0) {
      const uint32_t cbytes = csrc ? nvec * C::CB : 0u;
      const uint32_t mbytes = uint32_t(round16(nvec * C::MB));
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&ctl->cbar[warp][k], cbytes + mbytes);
      if (csrc) bulk_g2s(cbuf + k * S::BLK, csrc, cbytes, &ctl->cbar[warp][k]);
      bulk_g2s(mbuf + k * S::MBLK, meta_src(v0), mbytes, &ctl->cbar[warp][k]);
    }
  };
  uint32_t cphase = 0;  // bit k: phase of buffer k
  auto wait = [&](uint32_t k) {
    if (!mbar_wait(&ctl->cbar[warp][k], (cphase >> k) & 1, a.status))
      set_status(a.status, KVC_ERR_TIMEOUT);
    cphase ^= 1u << k;
  };
  bool stage_busy = false;
  // Decoded blocks go through a per-warp staging buffer: dense receivers with
  // a tensor map store them with tensor copies, other receivers with 16-byte
  // stores, half a warp per row (scatter_rows).
  bool use_tma = false;
  if constexpr (!kIsPaged<Layout>) use_tma = lay.tma != 0;
  uint8_t *stage = smem + S::rows + warp * S::WBUF;
  // Decodes vectors v0 .. v0 + nv - 1 (one per lane) whose codes start at
  // `codes` (CB bytes each, lane order) and meta at `meta` (MB bytes each).
  // One copy of the unrolled vector code serves both store paths.
  auto emit = [&](const uint8_t *codes, const uint8_t *meta, uint32_t v0, uint32_t nv) {
    uint32_t out[D / 2];
    const bool act = uint32_t(lane) < nv;
    if (act) decode_vector<D, BITS, G, kFp4>(ctl->mask, codes + lane * C::CB, meta + lane * C::MB, out);
    if constexpr (!kIsPaged<Layout>) {
      if (use_tma) {
        store_block_tma<D>(lay, out, v0, stage, stage_busy, a, ctl->vec_signs, ctl->mask,
                           ctl->seed);
        return;
      }
    }
    uint8_t *dst = nullptr;
    if (act) {
      bool ok;
      dst = vec_addr(lay, cum, v0 + lane, ok);
      if (!ok) {
        set_status(a.status, KVC_ERR_CORRUPT);
        dst = nullptr;
      }
    }
    __syncwarp();  // the previous block's scatter has read the buffer
    stage_row<D>(out, stage);
    if (ctl->vec_signs) fix_row_signs<D>(stage, ctl->mask, ctl->seed, fdiv(a.tdiv, v0 + lane));
    __syncwarp();
    if constexpr (kNarrow)
      scatter_rows_narrow<D / 8>(stage, lay.base, dst ? uint32_t((dst - lay.base) >> 4) : ~0u);
    else
      scatter_rows<D>(stage, dst);
  };

  // Raw code chunks, blocks of 32 vectors round-robin over the warps (chunks
  // that used zero-byte elimination are decoded by elim_decode_kernel); each
  // warp loads a block's code and meta bytes with bulk copies into one of its
  // two buffers while it decodes the previous block.
  const uint32_t vs0 = t0 * C::VC, vs1 = min(t1 * C::VC, V);
  const uint32_t nblk = (vs1 - vs0 + 31) / 32;
  auto raw_block = [&](uint32_t b) {  // block b lies in a raw code chunk
    const uint32_t t = (vs0 + b * 32) / C::VC;
    const uint64_t ce = ld_u64(table + 8 * uint64_t(t));
    return entry_size(ce) == min(uint32_t(C::VC), V - t * C::VC) * C::CB;
  };
  auto next_raw = [&](uint32_t b) {
    while (any_elim && b < nblk && !raw_block(b)) b += kDecWarps;
    return b;
  };
  auto issue_raw = [&](uint32_t b, uint32_t k) {
    const uint32_t v0 = vs0 + b * 32, t = v0 / C::VC;
    const uint64_t ce = ld_u64(table + 8 * uint64_t(t));
    issue(v0, min(32u, vs1 - v0),
          in + base + entry_offset(ce) + uint64_t(v0 - t * C::VC) * C::CB, k);
  };
  uint32_t b = next_raw(warp), k = 0;
  __syncwarp();
  if constexpr (32 * C::CB > S::BLK) {  // 8-bit: one block in both buffers
#pragma unroll 1
    while (b < nblk) {
      issue_raw(b, 0);
      wait(0);
      const uint32_t v0 = vs0 + b * 32;
      emit(cbuf, mbuf, v0, min(32u, vs1 - v0));
      b = next_raw(b + kDecWarps);
      __syncwarp();  // every lane is done with the buffers
    }
    bulk_wait_all<0>();
    return;
  }
  if (b < nblk) issue_raw(b, 0);
#pragma unroll 1
  while (b < nblk) {
    const uint32_t nb = next_raw(b + kDecWarps);
    __syncwarp();  // every lane is done with buffer k ^ 1 (the block before b)
    if (nb < nblk) issue_raw(nb, k ^ 1);
    wait(k);
    const uint32_t v0 = vs0 + b * 32;
    emit(cbuf + k * S::BLK, mbuf + k * S::MBLK, v0, min(32u, vs1 - v0));
    b = nb;
    k ^= 1;
  }
  bulk_wait_all<0>();
}

template <int D, class Layout, bool kNarrow>
__global__ void __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ DecArgs a, const __grid_constant__ Layout lay) {
  constexpr bool kPaged = kIsPaged<Layout>;
  using S = DecSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  DecCtl *ctl = reinterpret_cast<DecCtl *>(smem + S::ctl);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(smem + S::cum);
  const int tid = threadIdx.x;

  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
  }
  if (tid < kDecWarps) {
    mbar_init(&ctl->cbar[tid][0], 1);
    mbar_init(&ctl->cbar[tid][1], 1);
    mbar_fence_init();
  }
  if (tid == 0) {
    const StreamHdr h = parse_header<D>(a);
    ctl->hdr_ok = h.ok;
    ctl->bits = h.bits;
    ctl->group = h.group;
    ctl->n_req_stream = h.n_req;
    ctl->n_chunks = h.n_chunks;
    ctl->code_elim = h.code_elim;
    ctl->vec_signs = h.vec_signs;
    ctl->quant = h.quant;
    ctl->data_base = h.data_base;
    ctl->stream_bytes = h.stream_bytes;
    ctl->seed = h.seed;
    if (h.ok) sign_masks(h.seed, D, ctl->mask);
  }
  __syncthreads();
  bool ok = ctl->hdr_ok;
  if (ok) {  // token table: per request for a paged receiver, total otherwise
    const uint8_t *tt = a.in + kHeader + 8ull * ctl->n_chunks;
    uint32_t bad = 0;
    uint64_t sum = 0;
    for (uint32_t r = tid; r < ctl->n_req_stream; r += blockDim.x) {
      const uint32_t n = ld_u32(tt + 4ull * r);
      sum += n;
      if constexpr (kPaged) bad |= n != s_cum[r + 1] - s_cum[r];
    }
    const uint32_t hi = block_sum<kDecThreads>(uint32_t(sum >> 32), ctl->red);
    const uint32_t any_bad = block_sum<kDecThreads>(bad, ctl->red);
    const uint32_t lo32 = uint32_t(sum);
    const uint32_t lo_lo = block_sum<kDecThreads>(lo32 & 0xFFFFu, ctl->red);
    const uint32_t lo_hi = block_sum<kDecThreads>(lo32 >> 16, ctl->red);
    const uint64_t total = (uint64_t(hi) << 32) + (uint64_t(lo_hi) << 16) + lo_lo;
    ok = !any_bad && total == a.tokens;
  }
  if (!ok) {
    if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
    return;
  }
  const uint32_t bits = ctl->bits, group = ctl->group;
  if (ctl->quant == 2) {  // FP4 (4-bit; the header check guarantees it)
    if constexpr (D == 128) {
      if (group == 128)
        decode_body<128, 4, 128, Layout, kNarrow, true>(a, lay, ctl, smem, s_cum);
      else if (group == 64)
        decode_body<128, 4, 64, Layout, kNarrow, true>(a, lay, ctl, smem, s_cum);
      else
        decode_body<128, 4, 32, Layout, kNarrow, true>(a, lay, ctl, smem, s_cum);
    } else {
      if (group == 64)
        decode_body<64, 4, 64, Layout, kNarrow, true>(a, lay, ctl, smem, s_cum);
      else
        decode_body<64, 4, 32, Layout, kNarrow, true>(a, lay, ctl, smem, s_cum);
    }
    return;
  }
  if constexpr (D == 128) {
    if (bits == 8 && group == 128)
      decode_body<128, 8, 128, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 64)
      decode_body<128, 8, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 32)
      decode_body<128, 8, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 128)
      decode_body<128, 4, 128, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 64)
      decode_body<128, 4, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 32)
      decode_body<128, 4, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 128)
      decode_body<128, 2, 128, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 64)
      decode_body<128, 2, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else
      decode_body<128, 2, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
  } else {
    if (bits == 8 && group == 64)
      decode_body<64, 8, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 32)
      decode_body<64, 8, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 64)
      decode_body<64, 4, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 32)
      decode_body<64, 4, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 64)
      decode_body<64, 2, 64, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
    else
      decode_body<64, 2, 32, Layout, kNarrow>(a, lay, ctl, smem, s_cum);
  }
}


// Pre-pass of kvc_decompress: expands every meta chunk that used zero-byte
// elimination (D3, D4) into the workspace, slot s at ws_meta + s * 16 KB, so
// that the decode kernel reads each block's meta with one bulk copy and never
// stops for a meta chunk. A raw meta chunk is left where it is. Every table
// entry used here is bounds-checked on its own (the decode kernel checks the
// whole table); a bad one only records KVC_ERR_CORRUPT.
constexpr int kMetaThreads = 256;
struct MetaCtl {
  uint64_t full[1];
  uint32_t red[kMetaThreads / 32];
  uint32_t ok, bits, group, n_chunks;
  uint64_t base, limit;
};
constexpr int kMetaCtas = 6;  // per SM: one chunk buffer each, so latency hides across CTAs
// Shared memory: chunk buffer | plane-word scratch | 2 KB bitmap of the
// two-level form | MetaCtl.
constexpr size_t meta_smem_bytes() { return 2 * size_t(kChunk) + kBitmap + sizeof(MetaCtl); }

template <int D>
__global__ void __launch_bounds__(kMetaThreads, kMetaCtas)
    meta_expand_kernel(const __grid_constant__ DecArgs a) {
  grid_dependency_wait();  // the status clear
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *buf = smem, *scr = smem + kChunk, *bm = smem + 2 * kChunk;
  MetaCtl *ctl = reinterpret_cast<MetaCtl *>(smem + 2 * kChunk + kBitmap);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&ctl->full[0], 1);
    mbar_fence_init();
    const StreamHdr h = parse_header<D>(a);
    ctl->ok = h.ok;
    ctl->bits = h.bits;
    ctl->group = h.group;
    ctl->n_chunks = h.n_chunks;
    ctl->base = h.data_base;
    ctl->limit = min(a.in_bytes, h.stream_bytes);
  }
  __syncthreads();
  if (!ctl->ok) return;  // the decode kernel reports the header
  const uint32_t cb = D * ctl->bits / 8, mb = (D / ctl->group) * 4;
  const uint32_t vc = kChunk / cb, vm = vc * (ctl->group * ctl->bits / 32);
  const uint32_t n_code = (a.V + vc - 1) / vc, n_meta = (a.V + vm - 1) / vm;
  if (n_meta > a.ws_meta_chunks) return;  // cannot happen for a consistent header
  const uint8_t *table = a.in + kHeader;
  const uint64_t base = ctl->base, limit = ctl->limit;
  uint32_t phase = 0;
  // this CTA's chunks s = blockIdx.x + i * gridDim.x that used elimination
#pragma unroll 1
  for (uint32_t s = blockIdx.x; s < n_meta; s += gridDim.x) {
    const uint64_t e = ld_u64(table + 8 * (uint64_t(n_code) + s)), off = entry_offset(e);
    const uint32_t size = entry_size(e), pipe = entry_pipe(e), len = min(vm, a.V - s * vm) * mb;
    if (size == len) continue;  // raw: read in place by the decode kernel (which checks it)
    const bool ok = len == uint32_t(kChunk) && pipe <= 3 &&
                    size >= ((pipe & 2u) ? uint32_t(kBitmap2) : uint32_t(kBitmap)) &&
                    size < len && base + off + round16(size) <= limit;
    if (!ok) {
      if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
      continue;
    }
    if (tid == 0) {
      bulk_wait_read<0>();  // the previous chunk's store has read the buffer
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&ctl->full[0], uint32_t(round16(size)));
      bulk_g2s(buf, a.in + base + off, uint32_t(round16(size)), &ctl->full[0]);
    }
    if (!mbar_wait(&ctl->full[0], phase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
    phase ^= 1;
    if (lossless_decode<kMetaThreads>(buf, scr, bm, ctl->red, size, pipe, 8 * mb)) {
      fence_proxy_async_smem();
      named_bar_sync(1, kMetaThreads);
      if (tid == 0) {
        bulk_s2g(a.ws_meta + uint64_t(s) * kChunk, buf, kChunk);
        bulk_commit();
      }
    } else if (tid == 0) {
      set_status(a.status, KVC_ERR_CORRUPT);
    }
  }
  if (tid == 0) bulk_wait_all<0>();
}

// ------------------------------------------------------------------------
// Code chunks that used zero-byte elimination (rare: e.g. the heads whose
// keys have the largest outlier channels, where many codes sit at one end of
// the grid). The header's flag says whether there are any; without it this
// kernel returns at once. CTA b tests code chunks b, b + grid, ... 256 at a
// time (such chunks come in runs, which this spreads over the CTAs), expands
// each eliminated one in shared memory (D3, D4) and decodes its vectors like
// decode_kernel, which skips them. Table entries used here are bounds-checked
// on their own (decode_kernel checks the whole table).
// ------------------------------------------------------------------------
constexpr int kElimWarps = 8;
constexpr int kElimThreads = kElimWarps * 32;
struct ElimCtl {
  uint64_t zbar;
  uint64_t mbar[kElimWarps];
  uint32_t red[kElimThreads / 32];
  uint32_t ok, bits, group, nlist, vec_signs, quant;
  uint64_t base, limit, seed;
  alignas(16) uint32_t mask[128];
  uint32_t list[kElimThreads];
};
// Shared memory: per-warp staging | per-warp meta blocks | chunk | scratch |
// control | request prefix (paged).
template <int D>
struct ElimSmem {
  static constexpr size_t WBUF = size_t(D / 64) * 4096;
  static constexpr size_t MBLK = 32 * (size_t(D) / 32) * 4;
  static constexpr size_t meta = kElimWarps * WBUF;
  static constexpr size_t chunk = meta + kElimWarps * MBLK;
  static constexpr size_t scr = chunk + kChunk;
  static constexpr size_t bm = scr + kChunk;  // bitmap of the two-level form
  static constexpr size_t ctl = bm + kBitmap;
  static constexpr size_t cum = ctl + ((sizeof(ElimCtl) + 15) & ~size_t(15));
  static constexpr size_t bytes(bool paged) {
    return cum + (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
  }
};

template <int D, int BITS, int G, class Layout, bool kFp4 = false>
__device__ void elim_body(const DecArgs &a, const Layout &lay, ElimCtl *ctl, uint8_t *smem,
                          const uint32_t *cum) {
  using C = Cfg<D, BITS, G>;
  using S = ElimSmem<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t V = a.V;
  const uint32_t n_code = (V + C::VC - 1) / C::VC;
  const uint8_t *table = a.in + kHeader;
  const uint64_t base = ctl->base, limit = ctl->limit;
  uint8_t *stage = smem + warp * S::WBUF;
  uint8_t *mbuf = smem + S::meta + warp * S::MBLK;
  uint8_t *chunk = smem + S::chunk;
  uint8_t *scr = smem + S::scr;
  uint8_t *bmp = smem + S::bm;
  bool use_tma = false;
  if constexpr (!kIsPaged<Layout>) use_tma = lay.tma != 0;
  bool stage_busy = false;
  uint32_t zphase = 0, mphase = 0;
  auto len_of = [&](uint32_t c) { return min(uint32_t(C::VC), V - c * C::VC) * C::CB; };
  // meta of vectors v0 .. v0 + nv - 1 (one meta chunk): raw in the stream or
  // expanded by meta_expand_kernel; null for an entry out of bounds
  auto meta_src = [&](uint32_t v0, uint32_t nv) -> const uint8_t * {
    const uint32_t s = v0 / C::VM;
    const uint64_t e = ld_u64(table + 8 * (uint64_t(n_code) + s));
    const uint32_t mlen = min(uint32_t(C::VM), V - s * C::VM) * C::MB;
    const uint64_t off = entry_offset(e);
    if (entry_size(e) != mlen) return a.ws_meta + uint64_t(s) * kChunk + (v0 - s * C::VM) * C::MB;
    const uint64_t at = off + uint64_t(v0 - s * C::VM) * C::MB;
    return base + at + round16(nv * C::MB) <= limit ? a.in + base + at : nullptr;
  };
#pragma unroll 1
  for (uint64_t j0 = 0; uint64_t(blockIdx.x) + j0 * gridDim.x < n_code; j0 += kElimThreads) {
    if (tid == 0) ctl->nlist = 0;
    __syncthreads();
    const uint64_t cc = uint64_t(blockIdx.x) + (j0 + tid) * gridDim.x;
    if (cc < n_code && entry_size(ld_u64(table + 8 * cc)) != len_of(uint32_t(cc)))
      ctl->list[atomicAdd(&ctl->nlist, 1u)] = uint32_t(cc);
    __syncthreads();
    const uint32_t nl = ctl->nlist;
#pragma unroll 1
    for (uint32_t i = 0; i < nl; ++i) {
      const uint32_t c = ctl->list[i];
      const uint64_t e = ld_u64(table + 8 * uint64_t(c)), off = entry_offset(e);
      const uint32_t size = entry_size(e), len = len_of(c), pipe = entry_pipe(e);
      const bool good = len == uint32_t(kChunk) && (pipe == 0 || pipe == 2) &&
                        size >= (pipe ? uint32_t(kBitmap2) : uint32_t(kBitmap)) && size < len &&
                        base + off + round16(size) <= limit;
      if (tid == 0) {
        if (good) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&ctl->zbar, uint32_t(round16(size)));
          bulk_g2s(chunk, a.in + base + off, uint32_t(round16(size)), &ctl->zbar);
        } else {
          set_status(a.status, KVC_ERR_CORRUPT);
        }
      }
      if (!good) continue;  // uniform over the CTA
      if (!mbar_wait(&ctl->zbar, zphase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
      zphase ^= 1;
      const bool ok = lossless_decode<kElimThreads>(chunk, scr, bmp, ctl->red, size, pipe, 32u);
      if (!ok) {
        if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
        __syncthreads();
        continue;
      }
      const uint32_t nvec = len / C::CB;
#pragma unroll 1
      for (uint32_t b = warp; b * 32 < nvec; b += kElimWarps) {
        const uint32_t v0 = c * C::VC + b * 32, nv = min(32u, nvec - b * 32);
        const uint8_t *msrc = meta_src(v0, nv);
        if (!msrc) {
          if (lane == 0) set_status(a.status, KVC_ERR_CORRUPT);
          continue;
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t mbytes = uint32_t(round16(nv * C::MB));
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&ctl->mbar[warp], mbytes);
          bulk_g2s(mbuf, msrc, mbytes, &ctl->mbar[warp]);
        }
        if (!mbar_wait(&ctl->mbar[warp], mphase, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
        mphase ^= 1;
        uint32_t out[D / 2];
        const bool act = uint32_t(lane) < nv;
        if (act)
          decode_vector<D, BITS, G, kFp4>(ctl->mask, chunk + (b * 32 + lane) * C::CB,
                                    mbuf + lane * C::MB, out);
        if constexpr (!kIsPaged<Layout>) {
          if (use_tma) {
            store_block_tma<D>(lay, out, v0, stage, stage_busy, a, ctl->vec_signs, ctl->mask,
                               ctl->seed);
            continue;
          }
        }
        uint8_t *dst = nullptr;
        if (act) {
          bool vok;
          dst = vec_addr(lay, cum, v0 + lane, vok);
          if (!vok) {
            set_status(a.status, KVC_ERR_CORRUPT);
            dst = nullptr;
          }
        }
        __syncwarp();  // the previous block's scatter has read the buffer
        stage_row<D>(out, stage);
        if (ctl->vec_signs) fix_row_signs<D>(stage, ctl->mask, ctl->seed, fdiv(a.tdiv, v0 + lane));
        __syncwarp();
        scatter_rows<D>(stage, dst);
      }
      fence_proxy_async_smem();
      __syncthreads();  // the chunk buffer is reused
    }
  }
  if (lane == 0) bulk_wait_all<0>();
}

template <int D, class Layout>
__global__ void __launch_bounds__(kElimThreads, 1)
    elim_decode_kernel(const __grid_constant__ DecArgs a, const __grid_constant__ Layout lay) {
  grid_dependency_wait();  // the meta pre-pass
  using S = ElimSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  ElimCtl *ctl = reinterpret_cast<ElimCtl *>(smem + S::ctl);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(smem + S::cum);
  const int tid = threadIdx.x;
  if (a.in_bytes < kHeader || (a.in[11] & 1u) == 0) return;  // no code chunk uses elimination
  if (tid < kElimWarps) {
    mbar_init(&ctl->mbar[tid], 1);
    mbar_fence_init();
  }
  if (tid == 0) {
    mbar_init(&ctl->zbar, 1);
    mbar_fence_init();
    const StreamHdr h = parse_header<D>(a);
    ctl->ok = h.ok;
    ctl->bits = h.bits;
    ctl->group = h.group;
    ctl->base = h.data_base;
    ctl->limit = min(a.in_bytes, h.stream_bytes);
    ctl->vec_signs = h.vec_signs;
    ctl->quant = h.quant;
    ctl->seed = h.seed;
    if (h.ok) sign_masks(h.seed, D, ctl->mask);
  }
  if constexpr (kIsPaged<Layout>) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
  }
  __syncthreads();
  if (!ctl->ok) return;  // decode_kernel reports the header
  const uint32_t bits = ctl->bits, group = ctl->group;
  if (ctl->quant == 2) {  // FP4
    if constexpr (D == 128) {
      if (group == 128)
        elim_body<128, 4, 128, Layout, true>(a, lay, ctl, smem, s_cum);
      else if (group == 64)
        elim_body<128, 4, 64, Layout, true>(a, lay, ctl, smem, s_cum);
      else
        elim_body<128, 4, 32, Layout, true>(a, lay, ctl, smem, s_cum);
    } else {
      if (group == 64)
        elim_body<64, 4, 64, Layout, true>(a, lay, ctl, smem, s_cum);
      else
        elim_body<64, 4, 32, Layout, true>(a, lay, ctl, smem, s_cum);
    }
    return;
  }
  if constexpr (D == 128) {
    if (bits == 8 && group == 128)
      elim_body<128, 8, 128>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 64)
      elim_body<128, 8, 64>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 32)
      elim_body<128, 8, 32>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 128)
      elim_body<128, 4, 128>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 64)
      elim_body<128, 4, 64>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 32)
      elim_body<128, 4, 32>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 128)
      elim_body<128, 2, 128>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 64)
      elim_body<128, 2, 64>(a, lay, ctl, smem, s_cum);
    else
      elim_body<128, 2, 32>(a, lay, ctl, smem, s_cum);
  } else {
    if (bits == 8 && group == 64)
      elim_body<64, 8, 64>(a, lay, ctl, smem, s_cum);
    else if (bits == 8 && group == 32)
      elim_body<64, 8, 32>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 64)
      elim_body<64, 4, 64>(a, lay, ctl, smem, s_cum);
    else if (bits == 4 && group == 32)
      elim_body<64, 4, 32>(a, lay, ctl, smem, s_cum);
    else if (bits == 2 && group == 64)
      elim_body<64, 2, 64>(a, lay, ctl, smem, s_cum);
    else
      elim_body<64, 2, 32>(a, lay, ctl, smem, s_cum);
  }
}

}  // namespace kvc
