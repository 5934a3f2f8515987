// Fused decode kernel: parse and validate the stream -> per tile (one code
// chunk): bulk-async load of the code chunk and of the tile's meta -> undo
// zero-byte elimination and the bit-plane shuffle when the chunk used them ->
// unpack -> dequantize -> fp32 Walsh-Hadamard (same butterfly as the encoder)
// -> scale by 2^-log2(d) -> unsign -> bf16 -> bulk store (dense) or scatter
// through the receiver's page table (paged). The decoder is the inverse path
// the podcast page "FastKVComp: checking whether high-throughput KV
// compression pays off" (episode notes) places on the decode GPU.
//
// The chunk table stores every chunk's offset, so each CTA takes a contiguous
// range of tiles and reads its chunks directly: no scan, no inter-CTA waits.
// Every table entry is checked against its predecessor (offset = previous
// offset + padded previous size), so a consistent table is a prefix sum.
#pragma once

#include "kvc_encode.cuh"

namespace kvc {

struct TileIO {
  uint32_t ok;        // chunk entries valid
  uint32_t code_mode; // 0 raw, 1 zero-byte eliminated
  uint32_t code_size;
  uint32_t meta_mode;
  uint32_t meta_size;
};

struct DecCtl {
  uint64_t full[2];
  TileIO io[2];
  uint32_t red[kThreads / 32];
  uint32_t hdr_ok;
  uint32_t bits, group, n_req_stream, n_chunks;
  uint64_t data_base, stream_bytes, seed;
  alignas(16) uint32_t mask[128];  // read as uint4
};

template <int D>
constexpr size_t dec_smem_bytes(bool paged) {
  return size_t(2) * kThreads * (2 * D + 16) + 5 * size_t(kChunk) + sizeof(DecCtl) +
         (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
}

__device__ __forceinline__ uint32_t ld_u32(const uint8_t *p) {
  return *reinterpret_cast<const uint32_t *>(p);
}
__device__ __forceinline__ uint64_t ld_u64(const uint8_t *p) {
  return *reinterpret_cast<const uint64_t *>(p);
}

template <int D, int BITS, int G>
struct Dec : Cfg<D, BITS, G, kThreads> {
  using C = Cfg<D, BITS, G, kThreads>;

  // Reading R9: y^ = fl(zf + fl(q*sf)), the encoder's butterfly, then
  // x^ = bf16_RNE(sign * (u * 2^-log2 d)). Computed here in an exactly
  // equivalent order: zf and sf are pre-scaled by 2^-log2 d (exact), so every
  // value of the butterfly is the reference value times 2^-log2 d; no value
  // can become subnormal (all are 0 or at least 2^-28 in magnitude: fp16
  // meta values are multiples of 2^-24), so scaling commutes with every
  // rounding. q*sf is exact (q < 16 times an fp16 value needs at most 15
  // significant bits), so one fused multiply-add equals fl(zf + fl(q*sf)).
  static __device__ __forceinline__ void vector(const uint8_t *codes, const uint8_t *meta,
                                                const uint32_t *mask, uint32_t (&out)[D / 2]) {
    uint32_t cw[C::CW];
    const uint4 *c4 = reinterpret_cast<const uint4 *>(codes);
#pragma unroll
    for (int q = 0; q < C::CW / 4; ++q) {
      const uint4 v = c4[q];
      cw[4 * q] = v.x, cw[4 * q + 1] = v.y, cw[4 * q + 2] = v.z, cw[4 * q + 3] = v.w;
    }
    float zf[C::NG], sf[C::NG];
    const float up = float(1 << C::K) / float(D);
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      const uint32_t m = reinterpret_cast<const uint32_t *>(meta)[g];
      sf[g] = __fmul_rn(__half2float(__ushort_as_half(uint16_t(m & 0xFFFFu))), up);
      zf[g] = __fmul_rn(__half2float(__ushort_as_half(uint16_t(m >> 16))), up);
    }
    // Code -> float: a byte permute puts the code in the low byte of the bit
    // pattern 0x4B4000qq = 1.5*2^23 + q, and subtracting 1.5*2^23 gives q
    // exactly.
    constexpr uint32_t kMagicBits = 0x4B400000u;
    constexpr float kMagic = 12582912.0f;
    float y[D];
#pragma unroll
    for (int W = 0; W < C::CW; ++W) {
      constexpr int per_byte = 8 / BITS;
      uint32_t part[per_byte];  // part[e] byte k = code of channel (4W + k)*per_byte + e
#pragma unroll
      for (int e = 0; e < per_byte; ++e)
        part[e] = (cw[W] >> (e * BITS)) & (BITS == 4 ? 0x0F0F0F0Fu : 0x03030303u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int e = 0; e < per_byte; ++e) {
          const int c = (4 * W + k) * per_byte + e, g = c / G;
          const float qf = __fsub_rn(__uint_as_float(__byte_perm(part[e], kMagicBits, 0x7640 | k)), kMagic);
          y[c] = __fmaf_rn(qf, sf[g], zf[g]);
        }
      }
    }
    fwht<D>(y);
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
      const uint4 m4 = reinterpret_cast<const uint4 *>(mask)[q];
      const uint32_t m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * q + e;
        const __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
        out[j] = *reinterpret_cast<const uint32_t *>(&b) ^ m[e];
      }
    }
  }
};

template <int D, int BITS, int G, class Layout>
__device__ void decode_body(const DecArgs &a, const Layout &lay, DecCtl *ctl, uint8_t *s_out,
                            uint8_t *s_cbuf, uint8_t *s_mbuf, uint8_t *s_scr,
                            const uint32_t *cum) {
  using C = Cfg<D, BITS, G, kThreads>;
  using Dc = Dec<D, BITS, G>;
  const int tid = threadIdx.x;
  const uint32_t V = a.V;
  const uint32_t n_tiles = (V + C::VC - 1) / C::VC;
  const uint32_t t0 = uint32_t(uint64_t(blockIdx.x) * n_tiles / gridDim.x);
  const uint32_t t1 = uint32_t(uint64_t(blockIdx.x + 1) * n_tiles / gridDim.x);
  const uint8_t *in = a.in;
  const uint64_t base = ctl->data_base;
  const uint64_t limit = min(a.in_bytes, ctl->stream_bytes);

  // Thread 0: check the table entries of `tile`, then start its loads.
  auto prefetch = [&](uint32_t tile, int b) {
    uint64_t *bar = &ctl->full[b];
    TileIO io{1, 0, 0, 0, 0};
    uint32_t bytes = 0;
    const uint32_t nvec = min(uint32_t(C::VC), V - tile * C::VC);
    const uint32_t seg = tile / C::R, tis = tile - seg * C::R;
    // reading R13: code chunk c is entry c, meta chunk s is entry n_code + s
    const uint64_t ic = tile;
    const uint64_t im = uint64_t(n_tiles) + seg;
    auto entry = [&](uint64_t i, uint64_t &off, uint32_t &size) {
      const uint64_t e = ld_u64(in + kHeader + 8 * i);
      off = (e >> 16) << 4;
      size = uint32_t(e & 0xFFFFu);
      uint64_t expect = 0;
      if (i > 0) {
        const uint64_t p = ld_u64(in + kHeader + 8 * (i - 1));
        expect = ((p >> 16) << 4) + round16(p & 0xFFFFu);
      }
      return off == expect && base + off + round16(size) <= limit;
    };
    uint64_t oc, om;
    uint32_t sc, sm;
    const uint32_t code_len = nvec * C::CB;
    const uint32_t seg_vec = min(uint32_t(C::VM), V - seg * C::VM);
    const uint32_t meta_len = seg_vec * C::MB;
    bool ok = entry(ic, oc, sc) && entry(im, om, sm);
    if (ok) {
      if (sc == code_len)
        io.code_mode = 0;
      else if (code_len == kChunk && sc >= kBitmap && sc < kChunk)
        io.code_mode = 1;
      else
        ok = false;
      if (sm == meta_len)
        io.meta_mode = 0;
      else if (meta_len == kChunk && sm >= kBitmap && sm < kChunk)
        io.meta_mode = 1;
      else
        ok = false;
      // the last chunk must end the stream
      if (im + 1 == ctl->n_chunks && base + om + round16(sm) != ctl->stream_bytes) ok = false;
    }
    io.ok = ok;
    io.code_size = sc;
    io.meta_size = sm;
    ctl->io[b] = io;
    if (!ok) {
      set_status(a.status, KVC_ERR_CORRUPT);
      mbar_arrive(bar);
      return;
    }
    const uint32_t cbytes = uint32_t(round16(sc));
    uint32_t mbytes, moff;
    if (io.meta_mode == 0) {  // only this tile's slice
      moff = tis * C::SLICE;
      mbytes = uint32_t(round16(uint64_t(nvec) * C::MB));
    } else {
      moff = 0;
      mbytes = uint32_t(round16(sm));
    }
    bytes = cbytes + mbytes;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(s_cbuf + b * kChunk, in + base + oc, cbytes, bar);
    bulk_g2s(s_mbuf + b * kChunk + moff, in + base + om + moff, mbytes, bar);
  };

  if (t0 < t1 && tid == 0) prefetch(t0, 0);
  uint32_t outbuf = 0;
#pragma unroll 1
  for (uint32_t tile = t0, i = 0; tile < t1; ++tile, ++i) {
    const int b = i & 1;
    if (tile + 1 < t1 && tid == 0) prefetch(tile + 1, b ^ 1);
    if (!mbar_wait(&ctl->full[b], (i >> 1) & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
    const TileIO io = ctl->io[b];
    if (!io.ok) {
      named_bar_sync(1, kThreads);
      continue;
    }
    uint8_t *cb = s_cbuf + b * kChunk, *mb = s_mbuf + b * kChunk;
    bool good = true;
    if (io.code_mode) good &= ze_decode<kThreads>(cb, s_scr, ctl->red, io.code_size);
    if (io.meta_mode) good &= ze_decode<kThreads>(mb, s_scr, ctl->red, io.meta_size);
    if (!good) {
      if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
      named_bar_sync(1, kThreads);
      continue;
    }
    const uint32_t nvec = min(uint32_t(C::VC), V - tile * C::VC);
    const uint32_t seg = tile / C::R, tis = tile - seg * C::R;
#pragma unroll 1
    for (int sub = 0; sub < C::NSUB; ++sub) {
      const uint32_t j = sub * kThreads + tid;
      if (j >= nvec) break;
      bool ok;
      uint8_t *dst = vec_addr(lay, cum, tile * C::VC + j, ok);
      if (!ok) {
        set_status(a.status, KVC_ERR_CORRUPT);
        continue;
      }
      uint32_t out[D / 2];
      Dc::vector(cb + j * C::CB, mb + tis * C::SLICE + j * C::MB, ctl->mask, out);
      uint8_t *row = s_out + (outbuf * kThreads + tid) * C::ROWP;
      bulk_wait_read<1>();  // the store issued two rows ago has read this buffer
      uint4 *r4 = reinterpret_cast<uint4 *>(row);
#pragma unroll
      for (int q = 0; q < D / 8; ++q)
        r4[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
      fence_proxy_async_smem();
      bulk_s2g(dst, row, C::ROW);
      bulk_commit();
      outbuf ^= 1;
    }
    named_bar_sync(1, kThreads);  // buffers b free for the prefetch two tiles on
  }
  bulk_wait_all<0>();
}

template <int D, class Layout>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecArgs a, const __grid_constant__ Layout lay) {
  constexpr bool kPaged = kIsPaged<Layout>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *s_out = smem;
  uint8_t *s_cbuf = s_out + 2 * kThreads * (2 * D + 16);
  uint8_t *s_mbuf = s_cbuf + 2 * kChunk;
  uint8_t *s_scr = s_mbuf + 2 * kChunk;
  DecCtl *ctl = reinterpret_cast<DecCtl *>(s_scr + kChunk);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(ctl + 1);
  const int tid = threadIdx.x;
  constexpr uint32_t kLog2D = D == 64 ? 6 : D == 128 ? 7 : 8;

  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
  }
  if (tid == 0) {
    mbar_init(&ctl->full[0], 1);
    mbar_init(&ctl->full[1], 1);
    mbar_fence_init();
    // D1: header (reading R12) against the receiver's description.
    const uint8_t *h = a.in;
    bool ok = a.in_bytes >= kHeader;
    if (ok) {
      const uint32_t bits = h[8], k = h[9], group = ld_u32(h + 12);
      ok = ld_u32(h) == kMagic && (ld_u32(h + 4) & 0xFFFFu) == 1 &&
           (ld_u32(h + 4) >> 16) == kHeader && (bits == 2 || bits == 4) && k == kLog2D / 2 &&
           (group == 32 || group == 64 || group == 128) && group <= D &&
           ld_u32(h + 16) == a.layers && ld_u32(h + 20) == 2 && ld_u32(h + 24) == a.kv_heads &&
           ld_u32(h + 28) == a.head_dim && ld_u64(h + 32) == a.tokens;
      const uint32_t n_req = ld_u32(h + 48), n_chunks = ld_u32(h + 52);
      const uint64_t stream_bytes = ld_u64(h + 56);
      if (ok) {
        const uint64_t cb = uint64_t(D) * bits / 8, mbv = uint64_t(D / group) * 4;
        const uint64_t n_code = (uint64_t(a.V) * cb + kChunk - 1) / kChunk;
        const uint64_t n_meta = (uint64_t(a.V) * mbv + kChunk - 1) / kChunk;
        const uint64_t base = round16(kHeader + 8ull * n_chunks + 4ull * n_req);
        ok = n_chunks == n_code + n_meta && base <= stream_bytes && stream_bytes <= a.in_bytes &&
             (!a.paged_receiver || n_req == a.n_req);
        ctl->bits = bits;
        ctl->group = group;
        ctl->n_req_stream = n_req;
        ctl->n_chunks = n_chunks;
        ctl->data_base = base;
        ctl->stream_bytes = stream_bytes;
        ctl->seed = ld_u64(h + 40);
      }
    }
    ctl->hdr_ok = ok;
    if (ok) sign_masks(ctl->seed, D, ctl->mask);
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
    const uint32_t hi = block_sum<kThreads>(uint32_t(sum >> 32), ctl->red);
    const uint32_t lo_bad = block_sum<kThreads>(bad, ctl->red);
    // low 32 bits: sum of low halves may carry; recombine in 64 bits
    uint32_t lo32 = uint32_t(sum);
    const uint32_t lo_sum = block_sum<kThreads>(lo32 & 0xFFFFu, ctl->red);
    const uint32_t lo_hi = block_sum<kThreads>(lo32 >> 16, ctl->red);
    const uint64_t total = (uint64_t(hi) << 32) + (uint64_t(lo_hi) << 16) + lo_sum;
    ok = !lo_bad && total == a.tokens;
  }
  if (!ok) {
    if (tid == 0) set_status(a.status, KVC_ERR_CORRUPT);
    return;
  }
  const uint32_t bits = ctl->bits, group = ctl->group;
  if constexpr (D == 128) {
    if (bits == 4 && group == 128)
      decode_body<128, 4, 128>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 4 && group == 64)
      decode_body<128, 4, 64>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 4 && group == 32)
      decode_body<128, 4, 32>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 2 && group == 128)
      decode_body<128, 2, 128>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 2 && group == 64)
      decode_body<128, 2, 64>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else
      decode_body<128, 2, 32>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
  } else {
    if (bits == 4 && group == 64)
      decode_body<64, 4, 64>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 4 && group == 32)
      decode_body<64, 4, 32>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else if (bits == 2 && group == 64)
      decode_body<64, 2, 64>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
    else
      decode_body<64, 2, 32>(a, lay, ctl, s_out, s_cbuf, s_mbuf, s_scr, s_cum);
  }
}

}  // namespace kvc
