// Finishing kernels of kvc_compress (after the main encode kernel):
//
// finish_kernel: every chunk's stored size, from the shuffled-byte nonzero
//   counts the encode kernel accumulated (reading R11: zero-byte elimination
//   only for full chunks and only when strictly shorter), the device-wide
//   prefix sum of the padded sizes (readings R12, R13: every code chunk, then
//   every meta chunk), the meta chunks' lossless stage and their placement,
//   the chunk table and the header. CTA b takes a contiguous range of meta
//   chunks and of code-table entries; the prefix sums a CTA needs are block
//   reductions over the count arrays, so CTAs never wait on one another.
//
// compact_kernel: runs only when some code chunk shrinks (zero-byte
//   elimination makes it shorter, reading R11) and eliminating pays for the
//   shift of the later code chunks (reading R16), which is rare for
//   Hadamard-rotated codes. The encode
//   kernel left every code chunk raw at data base + c * 16 KB; chunks are
//   re-encoded and moved left in ticket order, a chunk only after every chunk
//   whose raw bytes its destination overlaps has been read; the meta chunks
//   (parked in the workspace by finish_kernel) are placed after every code
//   chunk has been read. All waits are bounded.
#pragma once

#include "kvc_encode.cuh"

namespace kvc {

constexpr int kFinThreads = 256;

struct FinCtl {
  uint64_t full[2];
  uint32_t red[kFinThreads / 32];
  uint32_t flag;
  uint32_t tick;
};

// Shared memory: two chunk buffers | plane-word scratch | 2 KB bitmap of the
// two-level form | FinCtl | request prefix (paged).
constexpr size_t kFinBm = 3 * size_t(kChunk);
constexpr size_t kFinCtl = kFinBm + kBitmap;
constexpr size_t fin_smem_bytes(bool paged) {
  return kFinCtl + sizeof(FinCtl) + (paged ? sizeof(uint32_t) * (KVC_MAX_REQUESTS + 1) : 0);
}

// 64-bit block sum over the first NT threads.
template <int NT>
__device__ __forceinline__ uint64_t block_sum64(uint64_t x, uint32_t *red) {
  const uint32_t hi = block_sum<NT>(uint32_t(x >> 32), red);
  const uint32_t mid = block_sum<NT>(uint32_t(x >> 16) & 0xFFFFu, red);
  const uint32_t lo = block_sum<NT>(uint32_t(x) & 0xFFFFu, red);
  return (uint64_t(hi) << 32) + (uint64_t(mid) << 16) + lo;
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

__device__ __forceinline__ uint32_t code_len(const FinArgs &a, uint32_t c) {
  return min(a.vc, a.V - c * a.vc) * a.cb;
}
// How a chunk is stored (readings R11, R17): size, pipeline id and, for the
// two-level form, its nonzero bitmap bytes. Only full chunks are coded, only
// when strictly shorter; the search mode takes the shortest candidate (code:
// pipelines 0, 2; meta: 0..3, or 0, 1 with one meta word per vector), ties
// to the lower id; the NONE mode stores everything raw.
struct Stored {
  uint32_t size, pipe, bnz;
};
__device__ __forceinline__ Stored code_stored(const FinArgs &a, uint32_t c) {
  const uint32_t len = code_len(a, c);
  if (len != uint32_t(kChunk) || a.mode == KVC_LOSSLESS_NONE) return {len, 0u, 0u};
  const unsigned long long n = a.code_nnz[c];
  const uint32_t n0 = uint32_t(n) & 0xFFFFu, b0 = (uint32_t(n) >> 16) & 0xFFFFu;
  Stored r{kBitmap + n0, 0u, 0u};
  if (a.mode == KVC_LOSSLESS_SEARCH && kBitmap2 + b0 + n0 < r.size) r = {kBitmap2 + b0 + n0, 2u, b0};
  return r.size < len ? r : Stored{len, 0u, 0u};
}
__device__ __forceinline__ uint32_t code_stored_size(const FinArgs &a, uint32_t c) {
  return code_stored(a, c).size;
}
__device__ __forceinline__ uint32_t meta_len(const FinArgs &a, uint32_t s) {
  return min(a.vm, a.V - s * a.vm) * a.mb;
}
__device__ __forceinline__ Stored meta_stored(const FinArgs &a, uint32_t s) {
  const uint32_t len = meta_len(a, s);
  if (len != uint32_t(kChunk) || a.mode == KVC_LOSSLESS_NONE) return {len, 0u, 0u};
  const unsigned long long n = a.meta_nnz[s];
  const uint32_t n0 = uint32_t(n) & 0xFFFFu, n1 = uint32_t(n) >> 16;
  const uint32_t b0 = uint32_t(n >> 32) & 0xFFFFu, b1 = uint32_t(n >> 48);
  Stored r{kBitmap + n0, 0u, 0u};
  if (a.mode == KVC_LOSSLESS_SEARCH) {
    if (kBitmap + n1 < r.size) r = {kBitmap + n1, 1u, 0u};
    if (a.mb >= 8) {  // the two-level form needs at least two meta words per vector
      if (kBitmap2 + b0 + n0 < r.size) r = {kBitmap2 + b0 + n0, 2u, b0};
      if (kBitmap2 + b1 + n1 < r.size) r = {kBitmap2 + b1 + n1, 3u, b1};
    }
  }
  return r.size < len ? r : Stored{len, 0u, 0u};
}
__device__ __forceinline__ uint32_t meta_stored_size(const FinArgs &a, uint32_t s) {
  return meta_stored(a, s).size;
}

// Reading R16: some code chunk shrank (flag bit 0); keep zero-byte
// elimination in the code region only if the padded bytes it saves are at
// least 1/64 of the padded bytes from the first shrinking code chunk to the
// region's end, the bytes the compaction would move. Otherwise every code
// chunk stays raw where the encode kernel wrote it.
// Both kernels that call this read the encode kernel's counters after
// grid_dependency_wait(), which returns only once the encode kernel (and the
// kernels before it) has completed and its memory operations, atomics
// included, are visible to this grid; plain volatile loads then see the final
// values, so no acquire ordering is needed here.
__device__ __forceinline__ bool code_elim_kept(const FinArgs &a, uint32_t flags) {
  if (!(flags & 1u) || a.n_code == 0) return false;
  const uint32_t c0 = ~*reinterpret_cast<const volatile uint32_t *>(a.first_inv);
  const uint64_t saved = *reinterpret_cast<const volatile unsigned long long *>(a.saved);
  const uint64_t moved =
      uint64_t(a.n_code - 1 - c0) * kChunk + round16(code_len(a, a.n_code - 1));
  return 64 * saved >= moved;
}

// Header (reading R12); byte 11 bit 0: some code chunk uses zero-byte
// elimination (`code_elim`).
template <class Layout>
__device__ void fin_header(const FinArgs &a, const uint32_t *cum, uint64_t stream_bytes,
                           uint32_t code_elim) {
  uint8_t *o = a.out;
  st_u32(o + 0, kMagic);
  st_u16(o + 4, 1);
  st_u16(o + 6, kHeader);
  // flags: bit 0 code chunks eliminated, bits 1..2 quantizer, bit 3 signs
  const uint32_t flags = code_elim | (a.quant << 1) | (a.signs << 3);
  st_u32(o + 8, a.bits | (a.k << 8) | (a.origin << 16) | (flags << 24));
  st_u32(o + 12, a.group);
  st_u32(o + 16, a.layers);
  st_u32(o + 20, 2);
  st_u32(o + 24, a.kv_heads);
  st_u32(o + 28, a.head_dim);
  st_u64(o + 32, a.tokens);
  st_u64(o + 40, a.seed);
  st_u32(o + 48, a.n_req);
  st_u32(o + 52, a.n_chunks);
  st_u64(o + 56, stream_bytes);
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
  if (a.out_bytes_dev) *a.out_bytes_dev = stream_bytes;
}

template <class Layout>
__global__ void __launch_bounds__(kFinThreads, 4)
    finish_kernel(const __grid_constant__ FinArgs a, const __grid_constant__ Layout lay) {
  grid_dependency_wait();  // the encode kernel's counts and meta
  constexpr int NT = kFinThreads;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *scr = smem + 2 * kChunk;  // buffers 0 and 1 below it
  uint8_t *bm = smem + kFinBm;
  FinCtl *ctl = reinterpret_cast<FinCtl *>(smem + kFinCtl);
  uint32_t *s_cum = reinterpret_cast<uint32_t *>(ctl + 1);
  const int tid = threadIdx.x;
  const uint32_t nb = gridDim.x, b = blockIdx.x;
  // this CTA's meta chunks s0 .. s1 - 1; the first one starts loading at once
  // (its raw bytes need none of the prefix sums below)
  const uint32_t s0 = uint32_t(uint64_t(b) * a.n_meta / nb);
  const uint32_t s1 = uint32_t(uint64_t(b + 1) * a.n_meta / nb);
  if (tid == 0) {
    mbar_init(&ctl->full[0], 1);
    mbar_init(&ctl->full[1], 1);
    mbar_fence_init();
    if (s0 < s1) {
      const uint32_t bytes = uint32_t(round16(meta_len(a, s0)));
      mbar_arrive_expect_tx(&ctl->full[0], bytes);
      bulk_g2s(smem, a.ws_meta + uint64_t(s0) * kChunk, bytes, &ctl->full[0]);
    }
    ctl->flag = code_elim_kept(a, *reinterpret_cast<volatile uint32_t *>(a.flags)) ? 1u : 0u;
  }
  if constexpr (kIsPaged<Layout>) {
    for (uint32_t r = tid; r <= lay.n_req; r += NT) s_cum[r] = lay.cum[r];
  }
  __syncthreads();

  // Bytes of all code chunks, padded. Unless some code chunk shrank and
  // eliminating pays (reading R16), every code chunk is raw and the code
  // region is the plain array of codes.
  const bool shrank = ctl->flag & 1u;
  uint64_t total_code = 0;
  if (!shrank) {
    if (a.n_code)
      total_code = uint64_t(a.n_code - 1) * kChunk + round16(code_len(a, a.n_code - 1));
  } else {
    uint64_t part = 0;
    for (uint32_t c = tid; c < a.n_code; c += NT) part += round16(code_stored_size(a, c));
    total_code = block_sum64<NT>(part, ctl->red);
  }

  // -------------------------------------------------- this CTA's meta chunks --
  uint64_t prefix = 0;
  {
    uint64_t part = 0;
    for (uint32_t s = tid; s < s0; s += NT) part += round16(meta_stored_size(a, s));
    prefix = block_sum64<NT>(part, ctl->red);
  }
  // Two buffers: the raw meta of chunk s + 1 loads while chunk s is encoded;
  // a buffer is refilled only after its store has read it.
  auto load = [&](uint32_t s, uint32_t k) {
    if (tid == 0) {
      const uint32_t bytes = uint32_t(round16(meta_len(a, s)));
      mbar_arrive_expect_tx(&ctl->full[k], bytes);
      bulk_g2s(smem + k * kChunk, a.ws_meta + uint64_t(s) * kChunk, bytes, &ctl->full[k]);
    }
  };
  uint32_t phase = 0;  // bit k: phase of buffer k
#pragma unroll 1
  for (uint32_t s = s0, k = 0; s < s1; ++s, k ^= 1) {
    uint8_t *buf = smem + k * kChunk;
    if (s + 1 < s1) {
      if (tid == 0) bulk_wait_read<0>();  // the store of chunk s - 1 has read buffer k ^ 1
      load(s + 1, k ^ 1);
    }
    if (!mbar_wait(&ctl->full[k], (phase >> k) & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
    phase ^= 1u << k;
    const uint32_t len = meta_len(a, s);
    const Stored so = meta_stored(a, s);
    const uint32_t size = so.size;
    if (size < len) lossless_encode<NT>(buf, scr, bm, ctl->red, so.pipe, 8 * a.mb, so.bnz, a.status);
    for (uint32_t i = size + tid; i < round16(size); i += NT) buf[i] = 0;
    fence_proxy_async_smem();
    named_bar_sync(1, NT);
    if (tid == 0) {
      const uint64_t off = total_code + prefix;
      if (a.data_base + off + round16(size) <= a.out_capacity) {
        // Without a shrunken code chunk the code region is final, so the
        // chunk goes to its place; otherwise it is parked in its workspace
        // slot until compact_kernel has moved the code chunks.
        uint8_t *dst = shrank ? a.ws_meta + uint64_t(s) * kChunk : a.out + a.data_base + off;
        bulk_s2g(dst, buf, uint32_t(round16(size)));
        bulk_commit();
        st_u64(a.out + kHeader + 8ull * (a.n_code + s), make_entry(off, size, so.pipe));
      } else {
        set_status(a.status, KVC_ERR_CAPACITY);
      }
      a.meta_size[s] = size;
    }
    prefix += round16(size);
  }

  // -------------------------------------------------- code-table entries --
  const uint32_t c0 = uint32_t(uint64_t(b) * a.n_code / nb);
  const uint32_t c1 = uint32_t(uint64_t(b + 1) * a.n_code / nb);
  if (!shrank) {
    for (uint32_t c = c0 + tid; c < c1; c += NT)
      st_u64(a.out + kHeader + 8ull * c, make_entry(uint64_t(c) * kChunk, code_len(a, c), 0u));
  } else {
    uint64_t part = 0;
    for (uint32_t c = tid; c < c0; c += NT) part += round16(code_stored_size(a, c));
    uint64_t base = block_sum64<NT>(part, ctl->red);
    for (uint32_t c = c0; c < c1; c += NT) {  // block-wide scan, NT chunks at a time
      const uint32_t me = c + tid;
      const Stored so = me < c1 ? code_stored(a, me) : Stored{0u, 0u, 0u};
      const uint32_t sz = so.size;
      if (me < c1) a.code_size[me] = sz;
      uint32_t total;
      const uint32_t ex = block_excl_scan<NT>(uint32_t(round16(sz)) >> 4, ctl->red, total);
      if (me < c1) {
        const uint64_t off = base + (uint64_t(ex) << 4);
        a.code_off[me] = off;
        st_u64(a.out + kHeader + 8ull * me, make_entry(off, sz, so.pipe));
      }
      base += uint64_t(total) << 4;
    }
  }

  // -------------------------------------------------------------- header --
  if (b == 0) {
    uint64_t part = 0;
    for (uint32_t s = tid; s < a.n_meta; s += NT) part += round16(meta_stored_size(a, s));
    const uint64_t total_meta = block_sum64<NT>(part, ctl->red);
    if (tid == 0) fin_header<Layout>(a, s_cum, a.data_base + total_code + total_meta, shrank ? 1u : 0u);
  }
  if (tid == 0) bulk_wait_all<0>();
}

// Re-encodes and moves code chunks when some code chunk shrank, then places
// the meta chunks. Chunk c (raw bytes at data_base + c * 16 KB, destination
// data_base + code_off[c] <= that) may overwrite only raw bytes of chunks
// j <= c whose 16 KB slot overlaps its destination; it waits for their read
// flags. Chunks before the first shrinking chunk c0 stay where they are
// (every destination lies at or above c0's slot).
__global__ void __launch_bounds__(kFinThreads, 4) compact_kernel(const __grid_constant__ FinArgs a) {
  grid_dependency_wait();  // finish_kernel's sizes, offsets and parked meta
  constexpr int NT = kFinThreads;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *buf = smem;
  uint8_t *scr = smem + kChunk;
  uint8_t *bm = smem + kFinBm;
  FinCtl *ctl = reinterpret_cast<FinCtl *>(smem + kFinCtl);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&ctl->full[0], 1);
    mbar_fence_init();
    ctl->flag = code_elim_kept(a, *reinterpret_cast<volatile uint32_t *>(a.flags)) ? 1u : 0u;
  }
  __syncthreads();
  if (!(ctl->flag & 1u)) return;
  // Chunks before the first shrinking one keep their place: tickets start
  // there. The next ticket is taken while the current chunk moves.
  const uint32_t c0 = ~*reinterpret_cast<volatile uint32_t *>(a.first_inv);
  uint32_t phase = 0;
  if (tid == 0) ctl->tick = atomicAdd(a.ticket, 1u);
#pragma unroll 1
  while (true) {
    named_bar_sync(1, NT);
    const uint32_t c = c0 + a.ticket_skip + ctl->tick;
    named_bar_sync(1, NT);
    if (c >= a.n_code) break;
    if (tid == 0) ctl->tick = atomicAdd(a.ticket, 1u);
    const uint32_t len = code_len(a, c), size = a.code_size[c];
    const uint64_t src = uint64_t(c) * kChunk, dst = a.code_off[c];
    if (dst != src || size != len) {
      // The raw bytes of chunk c are never overwritten before it reads them
      // (chunk j < c writes below code_off[j + 1] <= code_off[c] <= c * 16 KB),
      // so every chunk loads at once; only its store waits, for the chunks
      // whose raw bytes [dst, dst + padded size) overlaps to have been read.
      if (tid == 0) {
        mbar_arrive_expect_tx(&ctl->full[0], len);
        bulk_g2s(buf, a.out + a.data_base + src, len, &ctl->full[0]);
      }
      if (!mbar_wait(&ctl->full[0], phase & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
      ++phase;
      if (tid == 0) {
        __threadfence();
        atomicExch(a.done + c, 1u);  // raw bytes read
        atomicAdd(a.ticket + 1, 1u);
      }
      if (size != len) {  // shrinks: its lossless pipeline (0 or 2 for code chunks)
        const Stored so = code_stored(a, c);
        lossless_encode<NT>(buf, scr, bm, ctl->red, so.pipe, 0u, so.bnz, a.status);
        for (uint32_t i = size + tid; i < round16(size); i += NT) buf[i] = 0;
      }
      const uint32_t j0 = uint32_t(dst / kChunk);
      const uint32_t j1 = uint32_t((dst + round16(size) - 1) / kChunk);  // <= c
      for (uint32_t j = j0 + tid; j <= j1 && j < c; j += NT) {
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0; *reinterpret_cast<volatile uint32_t *>(a.done + j) == 0; ++it) {
          if (spin_expired(it, t0, a.status, a.wait_ns)) {
            set_status(a.status, KVC_ERR_TIMEOUT);
            break;
          }
          __nanosleep(64);
        }
      }
      __threadfence();
      fence_proxy_async_smem();
      named_bar_sync(1, NT);
      if (tid == 0) {
        bulk_s2g(a.out + a.data_base + dst, buf, uint32_t(round16(size)));
        bulk_commit();
        bulk_wait_read<0>();
      }
      named_bar_sync(1, NT);
    } else if (tid == 0) {
      atomicExch(a.done + c, 1u);
      atomicAdd(a.ticket + 1, 1u);
    }
  }
  // meta chunks, parked in the workspace, go after the code region once
  // every code chunk has been read (their destinations overlap old sources)
  if (tid == 0) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0; *reinterpret_cast<volatile uint32_t *>(a.ticket + 1) < a.n_code - c0; ++it) {
      if (spin_expired(it, t0, a.status, a.wait_ns)) {
        set_status(a.status, KVC_ERR_TIMEOUT);
        break;
      }
      __nanosleep(128);
    }
    __threadfence();
  }
  named_bar_sync(1, NT);
#pragma unroll 1
  for (uint32_t s = blockIdx.x; s < a.n_meta; s += gridDim.x) {
    if (tid == 0) {
      const uint32_t size = a.meta_size[s];
      const uint64_t e = *reinterpret_cast<const uint64_t *>(a.out + kHeader + 8ull * (a.n_code + s));
      mbar_arrive_expect_tx(&ctl->full[0], uint32_t(round16(size)));
      bulk_g2s(buf, a.ws_meta + uint64_t(s) * kChunk, uint32_t(round16(size)), &ctl->full[0]);
      if (!mbar_wait(&ctl->full[0], phase & 1, a.status)) set_status(a.status, KVC_ERR_TIMEOUT);
      bulk_s2g(a.out + a.data_base + entry_offset(e), buf, uint32_t(round16(size)));
      bulk_commit();
      bulk_wait_read<0>();
    }
    ++phase;
  }
  if (tid == 0) bulk_wait_all<0>();
}

}  // namespace kvc
