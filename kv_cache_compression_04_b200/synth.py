"""Seeded synthetic KV caches shaped like the workloads the codec targets.

This module draws inputs only. It holds none of the codec's arithmetic, and
both the CUDA path and the CPU oracle receive the very same bytes from it
(generated once, then copied where each side needs them).

The pages evaluate on unnamed serving workloads and print no data, so the
inputs are synthetic: model names below fix shapes only. Distributions follow
the usual shape of real KV caches: keys with strong per-channel scale
differences (outlier channels), values close to Gaussian or heavy-tailed.

Workloads (logical shape [layers, 2 (K, V), kv_heads, tokens, head_dim], bf16):
  tiny    [1, 2, 8, 64, 128]      K = N(0,1) * exp(N(0,1)) per (layer, head,
                                  channel); V = N(0,1); 4-bit, group 128
  llama8b [32, 2, 8, 4096, 128]   K = N(0,1) * exp(1.5 N(0,1)) per (layer,
                                  head, channel); V = N(0,1); 4-bit, group 128
  qwen7b  [28, 2, 4, 32768, 128]  K = N(0,1) with 4 outlier channels x20 (same
                                  channels for every layer and head); V =
                                  Student-t(5); 2-bit, group 32
  paged   80 layers, 8 heads, d 128, 16 requests of U{512..8192} tokens in
          16-token pages placed by a seeded permutation of the pool; llama8b
          distributions; 4-bit, group 64
  paged-L the paged batch with L layers (a smaller case of the same kernels)
  sweep   [32, 2, 8, T, 128], T = 8 * 2^i (1 MiB .. 4 GiB), llama8b
          distributions; 4-bit/group 128 and 2-bit/group 32
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

PAGE_SEED = 1234


@dataclass
class Workload:
    name: str
    layers: int
    kv_heads: int
    head_dim: int
    bits: int
    group: int
    seed: int
    kind: str                      # "lognormal" or "outlier_t"
    scale_sigma: float = 1.0       # lognormal sigma of the key channel scales
    tokens: int = 0                # dense
    seq_lens: list = field(default_factory=list)  # paged
    page_tokens: int = 16
    sign_seed: int = 0

    @property
    def paged(self) -> bool:
        return bool(self.seq_lens)

    @property
    def total_tokens(self) -> int:
        return sum(self.seq_lens) if self.paged else self.tokens

    @property
    def vectors(self) -> int:
        return self.layers * 2 * self.kv_heads * self.total_tokens

    @property
    def raw_bytes(self) -> int:
        return self.vectors * self.head_dim * 2


def paged_seq_lens(seed: int, n: int = 16, lo: int = 512, hi: int = 8192) -> list:
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def workload(name: str) -> Workload:
    if name == "tiny":
        return Workload("tiny", 1, 8, 128, 4, 128, 0, "lognormal", 1.0, tokens=64)
    if name == "llama8b":
        return Workload("llama8b", 32, 8, 128, 4, 128, 1, "lognormal", 1.5,
                        tokens=4096)
    if name == "qwen7b":
        return Workload("qwen7b", 28, 4, 128, 2, 32, 2, "outlier_t", tokens=32768)
    if name == "paged":
        return Workload("paged", 80, 8, 128, 4, 64, 3, "lognormal", 1.5,
                        seq_lens=paged_seq_lens(3))
    if name.startswith("paged-"):
        # paged-<layers>: the paged batch with fewer layers (profiling size)
        return Workload(name, int(name.split("-")[1]), 8, 128, 4, 64, 3, "lognormal", 1.5,
                        seq_lens=paged_seq_lens(3))
    if name.startswith("sweep"):
        # sweep-<i>-<bits>: T = 8 * 2^i tokens
        _, i, bits = name.split("-")
        bits = int(bits)
        return Workload(name, 32, 8, 128, bits, 128 if bits == 4 else 32, 4,
                        "lognormal", 1.5, tokens=8 * (1 << int(i)))
    raise KeyError(name)


def _gen(seed: int, device) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(seed)


def _key_scale(w: Workload, layers: int, g: torch.Generator, device) -> torch.Tensor:
    """Per-(layer, head, channel) multiplier of the keys, [layers, H, d]."""
    if w.kind == "lognormal":
        z = torch.randn(layers, w.kv_heads, w.head_dim, generator=g, device=device)
        return torch.exp(w.scale_sigma * z)
    m = torch.ones(layers, w.kv_heads, w.head_dim, device=device)
    ch = torch.randperm(w.head_dim, generator=g, device=device)[:4]
    m[:, :, ch] = 20.0
    return m


def _values(shape, w: Workload, g: torch.Generator, device) -> torch.Tensor:
    if w.kind == "outlier_t":
        z = torch.randn(shape, generator=g, device=device)
        chi2 = torch.zeros(shape, device=device)
        for _ in range(5):
            chi2 += torch.randn(shape, generator=g, device=device) ** 2
        return z / torch.sqrt(chi2 / 5.0)
    return torch.randn(shape, generator=g, device=device)


def dense_kv(w: Workload, device="cpu", tokens: int | None = None) -> torch.Tensor:
    """Contiguous bf16 tensor [layers, 2, kv_heads, tokens, head_dim]."""
    T = w.tokens if tokens is None else tokens
    g = _gen(w.seed, device)
    out = torch.empty(w.layers, 2, w.kv_heads, T, w.head_dim, dtype=torch.bfloat16,
                      device=device)
    for l in range(w.layers):  # one layer at a time bounds the fp32 temporaries
        m = _key_scale(w, 1, g, device)[0]
        k = torch.randn(w.kv_heads, T, w.head_dim, generator=g, device=device)
        out[l, 0] = (k * m[:, None, :]).to(torch.bfloat16)
        out[l, 1] = _values((w.kv_heads, T, w.head_dim), w, g, device).to(torch.bfloat16)
    return out


@dataclass
class PagedKV:
    pool: torch.Tensor        # bf16 [layers, n_pages, 2, kv_heads, page_tokens, d]
    page_table: torch.Tensor  # int32 [n_requests, max_pages]
    seq_lens: list

    def strides(self):
        """(layer, page, kv, head, slot) strides in elements."""
        s = self.pool.stride()
        return s[0], s[1], s[2], s[3], s[4]


def page_table_for(seq_lens, page_tokens: int, n_pages: int, seed: int,
                   device="cpu") -> torch.Tensor:
    """Assigns pool pages to requests through a seeded permutation."""
    need = [(n + page_tokens - 1) // page_tokens for n in seq_lens]
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(seed))
    maxp = max(need) if need else 1
    pt = torch.full((len(seq_lens), max(maxp, 1)), -1, dtype=torch.int32)
    pos = 0
    for r, n in enumerate(need):
        pt[r, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    return pt.to(device)


def paged_kv(w: Workload, device="cpu", spare_pages: int = 3,
             fill: str = "random") -> PagedKV:
    """A pool holding every request's pages (plus a few spare), filled with
    the workload's distributions; unused slots hold random data as well."""
    need = sum((n + w.page_tokens - 1) // w.page_tokens for n in w.seq_lens)
    n_pages = need + spare_pages
    pool = torch.empty(w.layers, n_pages, 2, w.kv_heads, w.page_tokens, w.head_dim,
                       dtype=torch.bfloat16, device=device)
    if fill == "random":
        g = _gen(w.seed, device)
        for l in range(w.layers):
            m = _key_scale(w, 1, g, device)[0]
            k = torch.randn(n_pages, w.kv_heads, w.page_tokens, w.head_dim,
                            generator=g, device=device)
            pool[l, :, 0] = (k * m[None, :, None, :]).to(torch.bfloat16)
            pool[l, :, 1] = _values((n_pages, w.kv_heads, w.page_tokens, w.head_dim),
                                    w, g, device).to(torch.bfloat16)
    pt = page_table_for(w.seq_lens, w.page_tokens, n_pages, PAGE_SEED, device)
    return PagedKV(pool, pt, list(w.seq_lens))


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 view (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
