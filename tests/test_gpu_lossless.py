"""GPU parity of the lossless-stage modes (reading R17): the search mode
(per chunk the shortest of the composed pipelines: XOR of words in runs of
32 vectors, one- or two-level zero-byte elimination) and the none mode (no
lossless stage) give the oracle's streams byte for byte, with the same
pipeline ids in the chunk table, and every stream decodes on the GPU to the
oracle's values: dense shapes over both head dimensions and every group
size, structured inputs whose chunks take the two-level form, paged pools
with eliminated code chunks, and the full-size workloads."""
import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import (chunk_table, first_diff, gpu_compress, gpu_decompress, oracle_desc,
                          pipelines, u16)

pytestmark = pytest.mark.gpu

SEARCH, NONE = kvc.KVC_LOSSLESS_SEARCH, kvc.KVC_LOSSLESS_NONE


def _roundtrip(kv, bits, g, mode, seed=0):
    L, _, H, T, D = kv.shape
    x = u16(kv.contiguous()).reshape(-1, D)
    od = oracle_desc(bits, g, D, L, H, [T], seed, lossless=mode)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.dense_desc(kv), bits, g, seed, lossless=mode)
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    out = torch.zeros_like(kv)
    assert gpu_decompress(ostream, kvc.dense_desc(out)) == kvc.KVC_OK
    _, ox = oracle.decompress(ostream, od)
    assert np.array_equal(u16(out).reshape(-1, D), ox)
    return od, ostream


SHAPES = [(128, 4, 128, 2, 3, 4096), (128, 4, 64, 2, 3, 2000), (128, 4, 32, 1, 5, 1777),
          (128, 2, 128, 3, 2, 3333), (128, 2, 64, 2, 2, 4100), (128, 2, 32, 2, 4, 3000),
          (64, 4, 64, 2, 3, 4000), (64, 4, 32, 1, 4, 4500), (64, 2, 64, 2, 2, 5000),
          (64, 2, 32, 3, 3, 2999)]


@pytest.mark.parametrize("mode", [SEARCH, NONE])
@pytest.mark.parametrize("d,bits,g,L,H,T", SHAPES)
def test_modes_dense_parity(d, bits, g, L, H, T, mode):
    w = synth.Workload("t", L, H, d, bits, g, seed=L * 100 + T, kind="lognormal",
                       scale_sigma=1.5, tokens=T)
    od, s = _roundtrip(synth.dense_kv(w).cuda(), bits, g, mode, seed=T)
    lay = od.layout()
    ids = pipelines(s, lay.n_chunks)
    if mode == NONE:
        sizes, _ = chunk_table(s, lay.n_chunks)
        assert not ids.any() and s[11] == 0
        assert s.size == od.max_bytes()                 # every chunk raw
    else:
        meta = [oracle.meta_chunk_index(lay, k) for k in range(lay.n_meta)]
        full = [m for m in meta[:-1]]
        if full:
            assert (ids[full] % 2 == 1).all()           # the XOR pays on these inputs


@pytest.mark.parametrize("kind", ["zeros", "half_zero_tokens", "sparse_channels",
                                  "constant_groups"])
@pytest.mark.parametrize("bits,g,d", [(4, 128, 128), (2, 32, 128), (4, 64, 64)])
def test_search_structured(kind, bits, g, d):
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(2, 2, 2, 2048, d, generator=gen)
    if kind == "zeros":
        x.zero_()
    elif kind == "half_zero_tokens":
        x[:, :, :, :1024] = 0
    elif kind == "sparse_channels":
        x[..., 8:] = 0
    elif kind == "constant_groups":
        v = torch.randn(2, 2, 2, 2048, 1, generator=gen)
        x.zero_()
        x[..., :1] = v
    od, s = _roundtrip(x.to(torch.bfloat16).cuda(), bits, g, SEARCH)
    if kind in ("zeros", "half_zero_tokens"):
        ids = pipelines(s, od.layout().n_chunks)
        assert (ids[:od.layout().n_code] == 2).any()    # two-level code chunks


@pytest.mark.parametrize("mode", [SEARCH, NONE])
@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32)])
def test_modes_paged_with_eliminated_code_chunks(bits, g, mode):
    seq = [700, 600, 300]
    w = synth.Workload("p", 2, 3, 128, bits, g, seed=3, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    pages = pk.page_table[1, :(600 + 15) // 16].long()
    pk.pool[:, pages] = 0
    x = oracle.gather_paged(u16(pk.pool).reshape(-1), w.layers, w.kv_heads, 128,
                            pk.strides(), 16, seq, pk.page_table.cpu().numpy(), 0, w.vectors)
    od = oracle_desc(bits, g, 128, w.layers, w.kv_heads, seq, origin=1, lossless=mode)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK and ostream[11] == (1 if mode == SEARCH else 0)
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), bits, g,
                                     lossless=mode)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    _, ox = oracle.decompress(ostream, od)
    pt2 = synth.page_table_for(seq, 16, pk.pool.shape[1], 41, device="cuda")
    pool2 = torch.full_like(pk.pool, 1.5)
    assert gpu_decompress(ostream, kvc.paged_desc(pool2, pt2, seq)) == kvc.KVC_OK
    got = oracle.gather_paged(u16(pool2).reshape(-1), w.layers, w.kv_heads, 128,
                              [s for s in pool2.stride()][:5], 16, seq, pt2.cpu().numpy(), 0,
                              w.vectors)
    assert np.array_equal(got, ox)


def test_lossless_mode_argument_checked():
    kv = torch.zeros(1, 2, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    desc = kvc.dense_desc(kv)
    for bad in (kvc.params(4, 128, 0, 3), kvc.params(4, 128, 0, -1)):
        assert kvc.kvc_max_compressed_bytes(desc, bad) == 0
    p = kvc.params(4, 128, 0)
    p.reserved = 1
    assert kvc.kvc_workspace_bytes(desc, p) == 0


@pytest.mark.parametrize("wname", ["llama8b", "qwen7b"])
def test_full_size_search_mode(wname):
    """Full-size streams in the search mode, whole stream and whole decode."""
    import os
    w = synth.workload(wname)
    threads = max(1, min(os.cpu_count() or 1, 128))
    kv = synth.dense_kv(w, device="cuda")
    x = u16(kv).reshape(-1, 128)
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, [w.tokens], lossless=SEARCH)
    st, gstream, gbuf, n = gpu_compress(kvc.dense_desc(kv), w.bits, w.group, lossless=SEARCH)
    assert st == kvc.KVC_OK
    ost, ostream = oracle.compress(od, x, threads=threads)
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    out = torch.empty_like(kv)
    assert gpu_decompress(gbuf, kvc.dense_desc(out), n) == kvc.KVC_OK
    dst, ox = oracle.decompress(ostream, od, threads=threads)
    assert dst == oracle.OK and np.array_equal(u16(out).reshape(-1, 128), ox)
