// Fused encode kernel: load/gather -> signs -> fp32 Walsh-Hadamard -> group
// min/max -> fp16 meta -> quantize -> pack -> lossless (bit-plane shuffle +
// zero-byte elimination on 16 KB chunks) -> device-wide prefix sum of chunk
// sizes -> compaction into the stream. One launch; the transformed tensor and
// the raw payload never reach HBM (the fusion of "Beyond Compression Ratio:
// High-Throughput KV Compression for Disaggregated LLM Serving", Abstract:
// transform and quantization in one kernel with no intermediate tensor; LC-
// style lossless backend of composable primitives).
//
// CTA = 8 compute warps (one vector per thread) + 1 publisher warp.
//  compute warps: per unit of 256 vectors, bulk-async loads of each vector's
//    row (dense or paged) into a padded shared-memory stage (two stages in
//    flight), the register pipeline, codes/meta into a 16 KB chunk slot; per
//    tile (one code chunk) the raw/zero-byte decision and, when it pays, the
//    bit-plane shuffle + elimination; per segment the meta chunk.
//  publisher warp: per tile, decoupled look-back over tile tickets (taken in
//    order from a global counter, so every predecessor is already owned by a
//    running CTA), chunk table entries and bulk stores of the chunks.
#pragma once

#include <type_traits>

#include "kvc_device.cuh"

namespace kvc {

template <int D, int BITS, int G>
struct Cfg {
  static constexpr int ROW = D * 2;              // bytes of one bf16 vector
  static constexpr int ROWP = ROW + 16;          // padded smem row (no bank conflicts)
  static constexpr int HALF = D / 2;             // pair partner distance
  static constexpr int CB = D * BITS / 8;        // code bytes per vector
  static constexpr int CW = CB / 4;              // code words per vector
  static constexpr int NG = D / G;               // groups per vector
  static constexpr int MB = NG * 4;              // meta bytes per vector
  static constexpr int VC = kChunk / CB;         // vectors per code chunk
  static constexpr int R = G * BITS / 32;        // code chunks per meta chunk
  static constexpr int VM = VC * R;              // vectors per meta chunk
  static constexpr int NSUB = VC / kThreads;     // 256-vector units per tile
  static constexpr int SLICE = VC * MB;          // meta bytes per tile
  static constexpr int LOG2D = D == 64 ? 6 : D == 128 ? 7 : 8;
  static constexpr int K = LOG2D / 2;            // meta stored x 2^-K
  static constexpr int QMAX = (1 << BITS) - 1;
  static_assert(NSUB >= 1 && VC % kThreads == 0, "unit size");
  static_assert(R >= 2 && R <= 16, "segment size");
};

struct SlotInfo {
  uint32_t tile, code_size, meta_size, has_meta;
};

struct EncCtl {
  uint64_t full[2];   // input stage filled (kThreads arrivals + bytes)
  uint64_t ready[2];  // chunk slot filled by compute warps (1 arrival)
  uint64_t freed[2];  // chunk slot stored by the publisher (1 arrival)
  SlotInfo info[2];
  uint32_t tick[4];  // ticket broadcast ring
  uint32_t red[kThreads / 32];
};

template <int D, int BITS, int G>
constexpr size_t enc_smem_bytes(bool paged) {
  using C = Cfg<D, BITS, G>;
  return size_t(2) * kThreads * C::ROWP + 5 * size_t(kChunk) + sizeof(EncCtl) +
         (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
}

template <class L>
constexpr bool kIsPaged = std::is_same<L, PagedLayout>::value;

// ------------------------------------------------------------------------
// One vector: registers in, codes + meta out. Returns error bits.
// ------------------------------------------------------------------------
template <int D, int BITS, int G>
struct Enc : Cfg<D, BITS, G> {
  using C = Cfg<D, BITS, G>;
  static constexpr int D8 = D / 8;  // 16-byte pieces per row

  // Reading R5: asymmetric min/max group quantization, fp16 zero (round
  // down) and scale (round up), both stored x 2^-K.
  // E1/E2: read the row from shared memory, widen bf16 exactly, flip the
  // sign bit of negative channels. p[i] = (channel i, channel i + d/2).
  static __device__ __forceinline__ void unpack(const uint8_t *row, const uint32_t *__restrict__ mask,
                                                float2 (&p)[C::HALF]) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
#pragma unroll
    for (int q = 0; q < D8 / 2; ++q) {
      const uint4 lo = r4[q], hi = r4[q + D8 / 2];  // channels 8q.. and 8q + d/2 ..
      const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ja = 4 * q + e, jb = ja + C::HALF / 2;
        const uint32_t a = wl[e] ^ mask[ja], b = wh[e] ^ mask[jb];
        p[2 * ja] = make_float2(__uint_as_float(a << 16), __uint_as_float(b << 16));
        p[2 * ja + 1] = make_float2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u));
      }
    }
  }

  static __device__ __forceinline__ uint32_t vector(float2 (&p)[C::HALF], uint32_t (&code)[C::CW],
                                                    uint32_t (&meta)[C::NG]) {
    // E3: butterfly (reading R2 order).
    fwht_pairs<C::HALF>(p);
    // E4/E5: per-group min/max (NaN-propagating) and meta.
    uint32_t err = 0;
    float nzf[C::NG], rr[C::NG];
#pragma unroll
    for (int g = 0; g < C::NG; ++g) {
      float mn = min2n(val_dyn(p, g * G), val_dyn(p, g * G + 1));
      float mx = max2n(val_dyn(p, g * G), val_dyn(p, g * G + 1));
#pragma unroll
      for (int c = g * G + 2; c < (g + 1) * G; c += 2) {
        mn = min3n(mn, val_dyn(p, c), val_dyn(p, c + 1));
        mx = max3n(mx, val_dyn(p, c), val_dyn(p, c + 1));
      }
      mn = __fadd_rn(mn, 0.0f);  // -0 -> +0
      mx = __fadd_rn(mx, 0.0f);
      if (!(isfinite(mn) && isfinite(mx))) err |= 1u;
      const float down = 1.0f / float(1 << C::K), up = float(1 << C::K);
      const __half zh = __float2half_rd(__fmul_rn(mn, down));
      const float zf = __fmul_rn(__half2float(zh), up);
      const float s32 = __fdiv_rn(__fsub_rn(mx, zf), float(C::QMAX));
      const __half sh = __float2half_ru(__fmul_rn(s32, down));
      const float sf = __fmul_rn(__half2float(sh), up);
      const uint16_t zb = __half_as_ushort(zh), sb = __half_as_ushort(sh);
      if ((zb & 0x7FFFu) == 0x7C00u || (sb & 0x7FFFu) == 0x7C00u) err |= 2u;
      rr[g] = ((sb & 0x7FFFu) == 0) ? 0.0f : __frcp_rn(sf);
      nzf[g] = zf;
      meta[g] = uint32_t(sb) | (uint32_t(zb) << 16);
    }
    // E6: q = RNE(fl(fl(y - zf) * r)) by cvt.rni on the rounded product. The
    // clamp to [0, 2^b - 1] never acts for a finite group: y - zf >= 0 since
    // zf <= min, and sf >= (max - zf)/(2^b - 1) bounds the product below
    // 2^b - 1 + 2^-20, so the integers are stored as they come.
#pragma unroll
    for (int i = 0; i < C::HALF; ++i) {
      const int ga = i / G, gb = (i + C::HALF) / G;
      const float2 t = mul2(sub2(p[i], make_float2(nzf[ga], nzf[gb])), make_float2(rr[ga], rr[gb]));
      p[i] = make_float2(__int_as_float(__float2int_rn(t.x)), __int_as_float(__float2int_rn(t.y)));
    }
    // E7: pack (reading R6), channel order, LSB first.
#pragma unroll
    for (int W = 0; W < C::CW; ++W) {
      uint32_t b[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        constexpr int per = 8 / BITS;  // codes per byte
        const int c0 = (W * 4 + k) * per;
        uint32_t acc = __float_as_uint(val_dyn(p, c0));
#pragma unroll
        for (int e = 1; e < per; ++e) acc += __float_as_uint(val_dyn(p, c0 + e)) << (e * BITS);
        b[k] = acc;
      }
      code[W] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    }
    return err;
  }

  static __device__ __forceinline__ float val_dyn(const float2 (&p)[C::HALF], int c) {
    return c < C::HALF ? p[c].x : p[c - C::HALF].y;
  }
};

// ------------------------------------------------------------------------
// Zero-byte elimination of one 16 KB chunk in shared memory (compute
// threads). buf holds the chunk; on return it holds bitmap + nonzero bytes.
// Reading R10 (bit planes of 32-bit little-endian words) and R11.
// ------------------------------------------------------------------------
__device__ __forceinline__ void ze_encode(uint8_t *buf, uint8_t *scr, uint32_t *red,
                                          uint32_t expect, uint32_t *status) {
  const int tid = threadIdx.x;
  if (tid < 128) {  // bit-plane shuffle: block m = words 32m .. 32m+31
    uint32_t a[32];
    const uint4 *src = reinterpret_cast<const uint4 *>(buf + tid * 128);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 v = src[q];
      a[4 * q] = v.x, a[4 * q + 1] = v.y, a[4 * q + 2] = v.z, a[4 * q + 3] = v.w;
    }
    transpose32(a);
    uint32_t *dst = reinterpret_cast<uint32_t *>(scr);
#pragma unroll
    for (int p = 0; p < 32; ++p) dst[p * 128 + tid] = a[p];
  }
  named_bar_sync(1, kThreads);
  // each thread: shuffled bytes [64 tid, 64 tid + 64)
  uint32_t w[16];
  const uint4 *s4 = reinterpret_cast<const uint4 *>(scr + tid * 64);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = s4[q];
    w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
  }
  uint32_t m0 = 0, m1 = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) m0 |= (((w[i / 4] >> (8 * (i % 4))) & 0xFFu) ? 1u : 0u) << i;
#pragma unroll
  for (int i = 0; i < 32; ++i) m1 |= (((w[8 + i / 4] >> (8 * (i % 4))) & 0xFFu) ? 1u : 0u) << i;
  uint32_t total;
  const uint32_t pos = block_excl_scan(__popc(m0) + __popc(m1), red, total);
  reinterpret_cast<uint2 *>(buf)[tid] = make_uint2(m0, m1);
  uint32_t o = kBitmap + pos;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const uint32_t byte = (w[i / 4] >> (8 * (i % 4))) & 0xFFu;
    if (byte && o < uint32_t(kChunk)) buf[o++] = uint8_t(byte);
  }
  (void)expect;
  (void)status;
  named_bar_sync(1, kThreads);
}

// Number of nonzero bytes the shuffle of a 16 KB chunk would have: byte i of
// plane p is nonzero iff bit p of (w[8i] | ... | w[8i+7]) is set, so the count
// is the sum of popcounts of 8-word ORs (no shuffle needed to decide).
__device__ __forceinline__ uint32_t chunk_nnz_part(const uint8_t *buf) {
  const uint4 *s = reinterpret_cast<const uint4 *>(buf + threadIdx.x * 64);
  const uint4 a = s[0], b = s[1], c = s[2], d = s[3];
  return __popc(a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w) +
         __popc(c.x | c.y | c.z | c.w | d.x | d.y | d.z | d.w);
}

// ------------------------------------------------------------------------
// Publisher warp: look-back, chunk table, bulk stores, header.
// ------------------------------------------------------------------------
constexpr uint64_t kFlagAgg = 1ull << 62, kFlagPre = 2ull << 62;
constexpr uint64_t kValMask = (1ull << 62) - 1;

__device__ __forceinline__ uint64_t lookback(const EncArgs &a, uint32_t tile, uint64_t agg) {
  const int lane = threadIdx.x & 31;
  uint64_t *st = a.tile_state;
  if (tile == 0) {
    if (lane == 0) st_release_u64(&st[0], kFlagPre | agg);
    return 0;
  }
  if (lane == 0) st_release_u64(&st[tile], kFlagAgg | agg);
  uint64_t excl = 0;
  int64_t look = int64_t(tile) - 1;
  const uint64_t t0 = globaltimer();
  while (true) {
    const int64_t idx = look - lane;
    uint64_t v = kFlagPre;  // before tile 0: prefix 0
    if (idx >= 0) {
      v = ld_acquire_u64(&st[idx]);
      for (uint32_t it = 0; (v >> 62) == 0; ++it) {
        if (spin_expired(it, t0, a.status)) {
          set_status(a.status, KVC_ERR_TIMEOUT);
          v = kFlagPre;
          break;
        }
        __nanosleep(32);
        v = ld_acquire_u64(&st[idx]);
      }
    }
    const uint32_t pre = __ballot_sync(0xFFFFFFFFu, (v >> 62) == 2);
    const int first = pre ? __ffs(pre) - 1 : 32;
    uint64_t c = lane <= first ? (v & kValMask) : 0;
#pragma unroll
    for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    excl += c;
    if (pre) break;
    look -= 32;
  }
  if (lane == 0) st_release_u64(&st[tile], kFlagPre | (excl + agg));
  return excl;
}

__device__ __forceinline__ void st_u16(uint8_t *p, uint32_t v) {
  *reinterpret_cast<uint16_t *>(p) = uint16_t(v);
}
__device__ __forceinline__ void st_u32(uint8_t *p, uint32_t v) {
  *reinterpret_cast<uint32_t *>(p) = v;
}
__device__ __forceinline__ void st_u64(uint8_t *p, uint64_t v) {
  *reinterpret_cast<uint64_t *>(p) = v;
}

// Header (reading R12) without stream_bytes, token table and zero padding.
template <class Layout>
__device__ void write_header(const EncArgs &a, const Layout &lay, const uint32_t *cum) {
  uint8_t *o = a.out;
  st_u32(o + 0, kMagic);
  st_u16(o + 4, 1);
  st_u16(o + 6, kHeader);
  st_u32(o + 8, a.bits | (a.k << 8) | (a.origin << 16));
  st_u32(o + 12, a.group);
  st_u32(o + 16, a.layers);
  st_u32(o + 20, 2);
  st_u32(o + 24, a.kv_heads);
  st_u32(o + 28, a.head_dim);
  st_u64(o + 32, a.tokens);
  st_u64(o + 40, a.seed);
  st_u32(o + 48, a.n_req);
  st_u32(o + 52, a.n_chunks);
  uint8_t *tt = o + kHeader + 8ull * a.n_chunks;
  for (uint32_t r = 0; r < a.n_req; ++r) {
    uint32_t n;
    if constexpr (kIsPaged<Layout>)
      n = cum[r + 1] - cum[r];
    else
      n = uint32_t(a.tokens);
    st_u32(tt + 4ull * r, n);
  }
  for (uint64_t b = kHeader + 8ull * a.n_chunks + 4ull * a.n_req; b < a.data_base; ++b) o[b] = 0;
}

template <int D, int BITS, int G, class Layout>
__device__ void publisher(const EncArgs &a, const Layout &lay, EncCtl *ctl, uint8_t *s_code,
                          uint8_t *s_meta, const uint32_t *cum) {
  using C = Cfg<D, BITS, G>;
  const int lane = threadIdx.x & 31;
  for (uint32_t k = 0;; ++k) {
    const uint32_t slot = k & 1;
    if (!mbar_wait(&ctl->ready[slot], (k >> 1) & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
    const SlotInfo info = ctl->info[slot];
    if (info.tile == kNoTile) break;
    const uint64_t pc = round16(info.code_size);
    const uint64_t agg = pc + (info.has_meta ? round16(info.meta_size) : 0);
    const uint64_t excl = lookback(a, info.tile, agg);
    if (lane == 0) {
      const uint64_t code_idx = uint64_t(info.tile) + info.tile / C::R;
      const uint64_t dst = a.data_base + excl;
      if (dst + agg <= a.out_capacity) {
        st_u64(a.out + kHeader + 8 * code_idx, ((excl >> 4) << 16) | info.code_size);
        bulk_s2g(a.out + dst, s_code + slot * kChunk, uint32_t(pc));
        if (info.has_meta) {
          st_u64(a.out + kHeader + 8 * (code_idx + 1), (((excl + pc) >> 4) << 16) | info.meta_size);
          bulk_s2g(a.out + dst + pc, s_meta + slot * kChunk, uint32_t(round16(info.meta_size)));
        }
        bulk_commit();
      } else {
        set_status(a.status, KVC_ERR_CAPACITY);
      }
      if (info.tile == 0) write_header(a, lay, cum);
      if (info.tile == a.n_tiles - 1) {
        const uint64_t total = a.data_base + excl + agg;
        st_u64(a.out + 56, total);
        if (a.out_bytes_dev) *a.out_bytes_dev = total;
      }
      bulk_wait_read<0>();
      mbar_arrive(&ctl->freed[slot]);
    }
    __syncwarp();
  }
  if (lane == 0) bulk_wait_all<0>();
}

// ------------------------------------------------------------------------
// The kernel.
// ------------------------------------------------------------------------
template <int D, int BITS, int G, class Layout>
__global__ void __launch_bounds__(kThreads + 32, 1)
    encode_kernel(const __grid_constant__ EncArgs a, const __grid_constant__ Layout lay) {
  using C = Cfg<D, BITS, G>;
  using E = Enc<D, BITS, G>;
  constexpr bool kPaged = kIsPaged<Layout>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *s_in = smem;
  uint8_t *s_code = s_in + 2 * kThreads * C::ROWP;
  uint8_t *s_meta = s_code + 2 * kChunk;
  uint8_t *s_scr = s_meta + 2 * kChunk;
  EncCtl *ctl = reinterpret_cast<EncCtl *>(s_scr + kChunk);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(ctl + 1);
  const int tid = threadIdx.x;

  if (a.n_tiles == 0) {  // empty input: header and tables only
    if (blockIdx.x == 0 && tid == 0) {
      if constexpr (kPaged) {
        for (uint32_t r = 0; r <= lay.n_req; ++r) s_cum[r] = lay.cum[r];
      }
      write_header(a, lay, s_cum);
      st_u64(a.out + 56, a.data_base);
      if (a.out_bytes_dev) *a.out_bytes_dev = a.data_base;
    }
    return;
  }
  if (tid == 0) {
    mbar_init(&ctl->full[0], kThreads);
    mbar_init(&ctl->full[1], kThreads);
    mbar_init(&ctl->ready[0], 1);
    mbar_init(&ctl->ready[1], 1);
    mbar_init(&ctl->freed[0], 1);
    mbar_init(&ctl->freed[1], 1);
    mbar_fence_init();
  }
  if constexpr (kPaged) {
    for (uint32_t r = tid; r <= lay.n_req; r += blockDim.x) s_cum[r] = lay.cum[r];
  }
  __syncthreads();

  if (tid >= kThreads) {
    publisher<D, BITS, G>(a, lay, ctl, s_code, s_meta, s_cum);
    return;
  }

  // ---------------------------------------------------- compute warps --
  const uint32_t n_tiles = a.n_tiles, V = a.V;
  uint32_t tick_next = kNoTile;  // thread 0: prefetched ticket
  auto grab = [&]() -> uint32_t {
    const uint32_t t = atomicAdd(a.ticket, 1u);
    return t < n_tiles ? t : kNoTile;
  };
  constexpr uint32_t kNeed = 0xFFFFFFFEu;  // issue pointer waits for a ticket

  auto issue = [&](int stage, uint32_t tile, uint32_t sub) {
    uint64_t *bar = &ctl->full[stage];
    const uint32_t j = sub * kThreads + tid;
    const uint32_t nvec = min(uint32_t(C::VC), V - tile * C::VC);
    if (j < nvec) {
      bool ok;
      const uint8_t *src = vec_addr(lay, s_cum, tile * C::VC + j, ok);
      if (ok) {
        mbar_arrive_expect_tx(bar, C::ROW);
        bulk_g2s(s_in + (stage * kThreads + tid) * C::ROWP, src, C::ROW, bar);
      } else {
        set_status(a.status, KVC_ERR_CORRUPT);
        mbar_arrive(bar);
      }
    } else {
      mbar_arrive(bar);
    }
  };

  uint32_t iss_tile = kNeed, iss_sub = 0, n_need = 0;
  uint32_t qt[2] = {kNoTile, kNoTile}, qs[2] = {0, 0};
  // prologue: fill both stages
  if (tid == 0) tick_next = grab();
#pragma unroll 1
  for (int s = 0; s < 2; ++s) {
    if (iss_tile == kNeed) {
      if (tid == 0) {
        ctl->tick[n_need & 3] = tick_next;
        tick_next = tick_next == kNoTile ? kNoTile : grab();
      }
      named_bar_sync(1, kThreads);
      iss_tile = ctl->tick[n_need & 3];
      ++n_need;
    }
    qt[s] = iss_tile;
    qs[s] = iss_sub;
    if (iss_tile != kNoTile) {
      issue(s, iss_tile, iss_sub);
      if (++iss_sub == C::NSUB) iss_sub = 0, iss_tile = kNeed;
    }
  }

  uint32_t u = 0, k = 0, nnz = 0, err = 0;
#pragma unroll 1
  while (true) {
    const int stage = u & 1;
    const uint32_t tile = stage ? qt[1] : qt[0];
    const uint32_t sub = stage ? qs[1] : qs[0];
    if (tile == kNoTile) break;
    const uint32_t slot = k & 1;
    if (sub == 0 && k >= 2 && !mbar_wait(&ctl->freed[slot], ((k >> 1) - 1) & 1, a.status))
      set_status(a.status, KVC_ERR_TIMEOUT);
    if (!mbar_wait(&ctl->full[stage], (u >> 1) & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
    const uint32_t nvec = min(uint32_t(C::VC), V - tile * C::VC);
    const uint32_t j = sub * kThreads + tid;
    const bool valid = j < nvec;
    float2 pv[C::HALF];
    if (valid) E::unpack(s_in + (stage * kThreads + tid) * C::ROWP, a.sign_mask, pv);
    const bool need = iss_tile == kNeed;
    if (need && tid == 0) {
      ctl->tick[n_need & 3] = tick_next;
      tick_next = tick_next == kNoTile ? kNoTile : grab();
    }
    named_bar_sync(1, kThreads);  // stage consumed; ticket visible
    if (need) iss_tile = ctl->tick[n_need++ & 3];
    if (stage) {
      qt[1] = iss_tile == kNeed ? kNoTile : iss_tile;
      qs[1] = iss_sub;
    } else {
      qt[0] = iss_tile == kNeed ? kNoTile : iss_tile;
      qs[0] = iss_sub;
    }
    if (iss_tile != kNoTile) {
      issue(stage, iss_tile, iss_sub);
      if (++iss_sub == C::NSUB) iss_sub = 0, iss_tile = kNeed;
    }

    const uint32_t seg = tile / C::R, tis = tile - seg * C::R;
    uint8_t *cslot = s_code + slot * kChunk;
    uint8_t *mslot = s_meta + slot * kChunk;
    uint32_t code[C::CW] = {};
    if (valid) {
      uint32_t meta[C::NG];
      err |= E::vector(pv, code, meta);
      uint4 *cd = reinterpret_cast<uint4 *>(cslot + j * C::CB);
#pragma unroll
      for (int q = 0; q < C::CW / 4; ++q)
        cd[q] = make_uint4(code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
      uint32_t *md = reinterpret_cast<uint32_t *>(mslot + tis * C::SLICE + j * C::MB);
      if constexpr (C::NG == 1) {
        md[0] = meta[0];
      } else if constexpr (C::NG == 2) {
        *reinterpret_cast<uint2 *>(md) = make_uint2(meta[0], meta[1]);
      } else {
        *reinterpret_cast<uint4 *>(md) = make_uint4(meta[0], meta[1], meta[2], meta[3]);
      }
    }
    // shuffled-byte count of this vector's 8-word groups
    {
      uint32_t orv[C::CW / 4 > 0 ? (C::CW + 7) / 8 : 1] = {};
#pragma unroll
      for (int W = 0; W < C::CW; ++W) orv[W / 8] |= code[W];
      if constexpr (C::CW >= 8) {
#pragma unroll
        for (int q = 0; q < C::CW / 8; ++q) nnz += __popc(orv[q]);
      } else {
        const uint32_t o = orv[0] | __shfl_xor_sync(0xFFFFFFFFu, orv[0], 1);
        if ((tid & 1) == 0) nnz += __popc(o);
      }
    }

    if (sub == C::NSUB - 1) {
      // ------------------------------------------------ finalize tile --
      const uint32_t total_nnz = block_sum(nnz, ctl->red);
      nnz = 0;
      const uint32_t code_len = nvec * C::CB;
      uint32_t code_size = code_len;
      if (code_len == kChunk && kBitmap + total_nnz < kChunk) {
        ze_encode(cslot, s_scr, ctl->red, total_nnz, a.status);
        code_size = kBitmap + total_nnz;
        for (uint32_t b = code_size + tid; b < round16(code_size); b += kThreads) cslot[b] = 0;
      }
      const uint32_t seg_tiles = min(uint32_t(C::R), n_tiles - seg * C::R);
      const bool last = tis == seg_tiles - 1;
      uint32_t meta_size = 0;
      if (!last) {
        uint8_t *wm = a.ws_meta + size_t(seg) * kChunk + tis * C::SLICE;
        for (uint32_t o = tid * 16; o < uint32_t(C::SLICE); o += kThreads * 16)
          __stcg(reinterpret_cast<uint4 *>(wm + o),
                 *reinterpret_cast<const uint4 *>(mslot + tis * C::SLICE + o));
        __threadfence();
      } else {
        if (tid < tis) {  // siblings of this segment published their meta
          const uint64_t *st = a.tile_state + seg * C::R + tid;
          const uint64_t t0 = globaltimer();
          for (uint32_t it = 0; (ld_acquire_u64(st) >> 62) == 0; ++it) {
            if (spin_expired(it, t0, a.status)) {
              set_status(a.status, KVC_ERR_TIMEOUT);
              break;
            }
            __nanosleep(64);
          }
        }
        named_bar_sync(1, kThreads);
        const uint8_t *wm = a.ws_meta + size_t(seg) * kChunk;
        for (uint32_t o = tid * 16; o < tis * C::SLICE; o += kThreads * 16)
          *reinterpret_cast<uint4 *>(mslot + o) = __ldcg(reinterpret_cast<const uint4 *>(wm + o));
        named_bar_sync(1, kThreads);
        const uint32_t seg_vec = min(uint32_t(C::VM), V - seg * C::VM);
        const uint32_t meta_len = seg_vec * C::MB;
        meta_size = meta_len;
        if (meta_len == kChunk) {
          const uint32_t mnnz = block_sum(chunk_nnz_part(mslot), ctl->red);
          if (kBitmap + mnnz < kChunk) {
            ze_encode(mslot, s_scr, ctl->red, mnnz, a.status);
            meta_size = kBitmap + mnnz;
          }
        }
        for (uint32_t b = meta_size + tid; b < round16(meta_size); b += kThreads) mslot[b] = 0;
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kThreads);
      if (tid == 0) {
        ctl->info[slot] = SlotInfo{tile, code_size, meta_size, last ? 1u : 0u};
        mbar_arrive(&ctl->ready[slot]);
      }
      ++k;
    }
    ++u;
  }
  if (err & 1u) set_status(a.status, KVC_ERR_NONFINITE);
  if (err & 2u) set_status(a.status, KVC_ERR_RANGE);
  // tell the publisher there is nothing more
  const uint32_t slot = k & 1;
  if (k >= 2 && !mbar_wait(&ctl->freed[slot], ((k >> 1) - 1) & 1, a.status))
    set_status(a.status, KVC_ERR_TIMEOUT);
  if (tid == 0) {
    ctl->info[slot] = SlotInfo{kNoTile, 0, 0, 0};
    mbar_arrive(&ctl->ready[slot]);
  }
}

}  // namespace kvc
