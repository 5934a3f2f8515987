"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded bytes. Streams must be byte-identical (codes, meta, chunk table,
lossless chunks); decoded bf16 must be bit-identical (the 1-ulp tolerance
allowed for decoded values is not needed: both sides run the same fp32
operation sequence with round-to-nearest-even and no contraction).

Sizes: small shapes that still span several tiles, segments and a ragged tail
(oracle in seconds), structured inputs that exercise zero-byte elimination,
and every full-size workload in the benchmark's launch configuration (llama8b,
qwen7b, the paged batch and all 26 points of the message-size sweep), each
compared whole: every stream byte and every decoded value."""
import os

import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import (chunk_table, first_diff, gpu_compress, gpu_decompress, oracle_desc,
                          u16)

pytestmark = pytest.mark.gpu

SHAPES = [  # d, bits, group, layers, heads, tokens
    (128, 4, 128, 1, 8, 64),
    (128, 4, 128, 2, 3, 1000),
    (128, 4, 64, 2, 3, 1000),
    (128, 4, 32, 1, 5, 777),
    (128, 2, 128, 3, 2, 1111),
    (128, 2, 64, 2, 2, 2049),
    (128, 2, 32, 2, 4, 3000),
    (64, 4, 64, 2, 3, 900),
    (64, 4, 32, 1, 4, 1500),
    (64, 2, 64, 2, 2, 2500),
    (64, 2, 32, 3, 3, 999),
]


def _roundtrip_dense(kv: torch.Tensor, bits, group, seed=0, logical=None):
    """Encode kv (any strides) on the GPU and with the oracle; compare streams;
    decode the oracle's stream on the GPU and compare with the oracle's
    decode."""
    L, _, H, T, D = kv.shape
    x = u16(kv.contiguous()).reshape(-1, D) if logical is None else logical
    od = oracle_desc(bits, group, D, L, H, [T], seed)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    desc = kvc.dense_desc(kv)
    st, gstream, _, n = gpu_compress(desc, bits, group, seed)
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    # decode the oracle's bytes on the GPU
    out = torch.zeros((L, 2, H, T, D), dtype=torch.bfloat16, device="cuda")
    assert gpu_decompress(ostream, kvc.dense_desc(out)) == kvc.KVC_OK
    dst, ox = oracle.decompress(ostream, od)
    assert dst == oracle.OK
    got = u16(out).reshape(-1, D)
    assert np.array_equal(got, ox), f"{np.count_nonzero(got != ox)} decoded values differ"
    return ostream


@pytest.mark.parametrize("d,bits,g,L,H,T", SHAPES)
def test_dense_parity(d, bits, g, L, H, T):
    w = synth.Workload("t", L, H, d, bits, g, seed=L * 100 + T, kind="lognormal",
                       scale_sigma=1.5, tokens=T)
    kv = synth.dense_kv(w).cuda()
    _roundtrip_dense(kv, bits, g, seed=T)


def test_tiny_workload_parity():
    w = synth.workload("tiny")
    kv = synth.dense_kv(w).cuda()
    s = _roundtrip_dense(kv, w.bits, w.group, w.sign_seed)
    assert s.size == 69744                      # all chunks raw on Gaussian-like data


def test_outlier_t_distribution_parity():
    w = synth.Workload("q", 2, 4, 128, 2, 32, seed=2, kind="outlier_t", tokens=2000)
    _roundtrip_dense(synth.dense_kv(w).cuda(), 2, 32)


def test_strided_dense_input():
    """A tensor stored [tokens, layers, 2, heads, d] and viewed as [layers, 2,
    heads, tokens, d]: the gather follows the strides."""
    w = synth.Workload("s", 3, 2, 128, 4, 64, seed=9, kind="lognormal", tokens=333)
    kv = synth.dense_kv(w)
    store = kv.permute(3, 0, 1, 2, 4).contiguous().cuda()       # [T, L, 2, H, D]
    view = store.permute(1, 2, 3, 0, 4)
    assert not view.is_contiguous()
    _roundtrip_dense(view, 4, 64, logical=u16(kv).reshape(-1, 128))


def test_empty_input():
    kv = torch.zeros((2, 2, 3, 0, 128), dtype=torch.bfloat16, device="cuda")
    od = oracle_desc(4, 128, 128, 2, 3, [0])
    st, gstream, _, n = gpu_compress(kvc.dense_desc(kv), 4, 128)
    _, ostream = oracle.compress(od, np.zeros((0, 128), np.uint16))
    assert st == kvc.KVC_OK and np.array_equal(gstream, ostream)
    assert gpu_decompress(ostream, kvc.dense_desc(kv)) == kvc.KVC_OK


# --------------------------------------------------------------- structured --
def _structured(kind, T=1024, L=2, H=2, D=128):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(L, 2, H, T, D, generator=g)
    if kind == "zeros":
        x.zero_()
    elif kind == "half_zero_tokens":
        x[:, :, :, : T // 2] = 0
    elif kind == "neg_zero":
        return torch.full((L, 2, H, T, D), -0.0, dtype=torch.bfloat16)
    elif kind == "constant_groups":
        v = torch.randn(L, 2, H, T, 1, generator=g)
        x.zero_()
        x[..., :1] = v                           # one-hot at channel 0: every group constant
    elif kind == "tiny_values":
        x = x * 1e-30
    elif kind == "large_values":
        x = x * 3000.0
    elif kind == "sparse_channels":
        x[..., 8:] = 0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("kind", ["zeros", "half_zero_tokens", "neg_zero", "constant_groups",
                                  "tiny_values", "large_values", "sparse_channels"])
@pytest.mark.parametrize("bits,g", [(4, 128), (2, 32)])
def test_structured_inputs(kind, bits, g):
    kv = _structured(kind).cuda()
    s = _roundtrip_dense(kv, bits, g)
    if kind in ("zeros", "neg_zero", "half_zero_tokens"):
        od = oracle_desc(bits, g, 128, 2, 2, [1024])
        sizes, _ = chunk_table(s, od.layout().n_chunks)
        assert (sizes < 16384).any()              # zero-byte elimination was exercised


@pytest.mark.parametrize("bits,g", [(4, 128), (2, 32)])
@pytest.mark.parametrize("zero_chunk,kept", [(8, True), (7, False), (63, True), (0, False)])
def test_code_elimination_threshold(bits, g, zero_chunk, kept):
    """Reading R16 on the GPU: 64 code chunks, one of them all-zero codes.
    Its elimination saves 56 * 256 padded bytes, so it is kept only if at most
    56 code chunks (itself included) follow from it: 8 and 63 keep it (8 is
    the tie), 7 and 0 store every code chunk raw, with the flag clear and no
    compaction. Stream bytes and decoded values equal the oracle's."""
    per = 16384 * 8 // (128 * bits)                           # vectors per code chunk
    V = per * 64
    x = torch.randn(V, 128, generator=torch.Generator().manual_seed(11))
    x[zero_chunk * per:(zero_chunk + 1) * per] = 0
    kv = x.to(torch.bfloat16).reshape(1, 2, V // 2048, 1024, 128).cuda()
    s = _roundtrip_dense(kv, bits, g)
    od = oracle_desc(bits, g, 128, 1, V // 2048, [1024])
    lay = od.layout()
    sizes, _ = chunk_table(s, lay.n_chunks)
    code = [int(sizes[oracle.code_chunk_index(lay, c)]) for c in range(64)]
    assert code[zero_chunk] == (2048 if kept else 16384)
    assert s[11] == (1 if kept else 0)


def test_compaction_many_chunks_mixed():
    """Shrunken code chunks scattered through more code chunks than CTAs (each
    CTA moves several): a random half of the 16 KB code chunks are all-zero
    codes, so later chunks move left by varying distances."""
    L, H, T, D = 4, 8, 4096, 128
    g = torch.Generator().manual_seed(11)
    x = torch.randn(L, 2, H, T, D, generator=g)
    blocks = x.view(L, 2, H, T // 256, 256, D)
    zero = torch.rand(L, 2, H, T // 256, generator=g) < 0.5
    blocks[zero] = 0
    s = _roundtrip_dense(x.to(torch.bfloat16).cuda(), 4, 128)
    od = oracle_desc(4, 128, D, L, H, [T])
    sizes, _ = chunk_table(s, od.layout().n_chunks)
    n_code = od.layout().n_code
    assert n_code > 2 * 148
    assert 0.3 < (sizes[:n_code] < 16384).mean() < 0.7


# -------------------------------------------------------------------- paged --
def _paged_setup(seq, L=2, H=3, D=128, bits=4, g=64, seed=3, page_tokens=16):
    w = synth.Workload("p", L, H, D, bits, g, seed=seed, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq, page_tokens=page_tokens)
    pk = synth.paged_kv(w, device="cuda")
    pool = u16(pk.pool)
    x = oracle.gather_paged(pool.reshape(-1), L, H, D, pk.strides(), page_tokens, seq,
                            pk.page_table.cpu().numpy(), 0, w.vectors)
    return w, pk, x


def _used_slots(pk, seq, page_tokens=16):
    used = torch.zeros(pk.pool.shape[1], page_tokens, dtype=torch.bool)
    pt = pk.page_table.cpu()
    for r, n in enumerate(seq):
        for t in range(n):
            used[pt[r, t // page_tokens], t % page_tokens] = True
    return used


@pytest.mark.parametrize("seq,bits,g", [([20, 0, 33, 700, 16, 257], 4, 64),
                                        ([1, 1500, 3], 2, 32), ([4096, 4095], 4, 128)])
def test_paged_parity_and_cross_layout_decode(seq, bits, g):
    w, pk, x = _paged_setup(seq, bits=bits, g=g)
    od = oracle_desc(bits, g, 128, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), bits, g)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    _, ox = oracle.decompress(ostream, od)
    # decode into a differently shuffled pool pre-filled with a canary
    pt2 = synth.page_table_for(seq, 16, pk.pool.shape[1], 777, device="cuda")
    pool2 = torch.full_like(pk.pool, 1.5)
    desc2 = kvc.paged_desc(pool2, pt2, seq)
    assert gpu_decompress(ostream, desc2) == kvc.KVC_OK
    got = oracle.gather_paged(u16(pool2).reshape(-1), w.layers, w.kv_heads, 128,
                              [s for s in pool2.stride()][:5], 16, seq, pt2.cpu().numpy(), 0,
                              w.vectors)
    assert np.array_equal(got, ox)
    pk2 = synth.PagedKV(pool2, pt2, seq)
    unused = ~_used_slots(pk2, seq)
    canary = pool2.cpu().float().permute(1, 4, 0, 2, 3, 5)[unused]
    assert torch.all(canary == 1.5), "decode wrote outside the described slots"
    # decode into a dense tensor of the same logical shape
    dense = torch.zeros((w.layers, 2, w.kv_heads, sum(seq), 128), dtype=torch.bfloat16,
                        device="cuda")
    assert gpu_decompress(ostream, kvc.dense_desc(dense)) == kvc.KVC_OK
    assert np.array_equal(u16(dense).reshape(-1, 128), ox)


@pytest.mark.parametrize("page_tokens", [8, 32, 64, 24])
def test_paged_page_sizes(page_tokens):
    """Pages of 8, 32 and 64 slots (tensor-map runs of 8 or 16 slots, a run's
    page and slot taken from its index in the request) and of 24 (not a power
    of two: every block gathered row by row), with requests that start and end
    inside pages; decode scatters through another page table."""
    seq = [300, 1025, 77, 2000, 33]
    w, pk, x = _paged_setup(seq, L=2, H=2, page_tokens=page_tokens)
    od = oracle_desc(4, 64, 128, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), 4, 64)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    _, ox = oracle.decompress(ostream, od)
    pt2 = synth.page_table_for(seq, page_tokens, pk.pool.shape[1], 5, device="cuda")
    pool2 = torch.full_like(pk.pool, 1.5)
    assert gpu_decompress(ostream, kvc.paged_desc(pool2, pt2, seq)) == kvc.KVC_OK
    got = oracle.gather_paged(u16(pool2).reshape(-1), w.layers, w.kv_heads, 128,
                              [s for s in pool2.stride()][:5], page_tokens, seq,
                              pt2.cpu().numpy(), 0, w.vectors)
    assert np.array_equal(got, ox)
    unused = ~_used_slots(synth.PagedKV(pool2, pt2, seq), seq, page_tokens)
    canary = pool2.cpu().float().permute(1, 4, 0, 2, 3, 5)[unused]
    assert torch.all(canary == 1.5), "decode wrote outside the described slots"


# permutation from a slot-major pool's storage order to the logical
# [layers, pages, kv, heads, slots, d] view the descriptor takes
_SLOT_MAJOR = {
    # [layers][pages][slot][kv][head][d]: kv and head still merge (tensor-map runs)
    "slot_kv_head": ((0, 1, 4, 2, 3, 5), (0, 1, 3, 4, 2, 5)),
    # [layers][pages][kv][slot][head][d]: they do not (row gathers)
    "kv_slot_head": ((0, 1, 2, 4, 3, 5), (0, 1, 2, 4, 3, 5)),
}


@pytest.mark.parametrize("order", sorted(_SLOT_MAJOR))
def test_paged_slot_major_pools(order):
    """Pools stored slot-major (the layouts of serving engines that keep a
    page's heads together per token) through strided views: parity with the
    oracle's gather of the same strides, decode into another such pool."""
    seq = [300, 1025, 77]
    to_store, to_view = _SLOT_MAJOR[order]
    w, pk, _ = _paged_setup(seq, L=2, H=2)
    store = pk.pool.permute(*to_store).contiguous()
    view = store.permute(*to_view)
    assert view.shape == pk.pool.shape and torch.equal(view, pk.pool)
    x = oracle.gather_paged(u16(store).reshape(-1), w.layers, w.kv_heads, 128,
                            [st for st in view.stride()][:5], 16, seq,
                            pk.page_table.cpu().numpy(), 0, w.vectors)
    od = oracle_desc(4, 64, 128, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(view, pk.page_table, seq), 4, 64)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    _, ox = oracle.decompress(ostream, od)
    pt2 = synth.page_table_for(seq, 16, pk.pool.shape[1], 8, device="cuda")
    store2 = torch.full_like(store, 1.5)
    view2 = store2.permute(*to_view)
    assert gpu_decompress(ostream, kvc.paged_desc(view2, pt2, seq)) == kvc.KVC_OK
    got = oracle.gather_paged(u16(store2).reshape(-1), w.layers, w.kv_heads, 128,
                              [st for st in view2.stride()][:5], 16, seq, pt2.cpu().numpy(), 0,
                              w.vectors)
    assert np.array_equal(got, ox)


@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32)])
def test_paged_parity_eliminated_code_chunks(bits, g):
    """A paged batch whose middle request is all zeros: the code chunks inside
    it are stored eliminated (they save far more than 1/64 of what follows,
    reading R16) between raw ones, so the paged gather feeds the compaction,
    and the eliminated-chunk decode scatters through another page table."""
    seq = [700, 600, 300]
    w, pk, _ = _paged_setup(seq, bits=bits, g=g)
    pages = pk.page_table[1, :(600 + 15) // 16].long()
    pk.pool[:, pages] = 0
    x = oracle.gather_paged(u16(pk.pool).reshape(-1), w.layers, w.kv_heads, 128,
                            pk.strides(), 16, seq, pk.page_table.cpu().numpy(), 0, w.vectors)
    od = oracle_desc(bits, g, 128, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK and ostream[11] == 1
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), bits, g)
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


@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32)])
def test_paged_parity_head_dim_64(bits, g):
    """head_dim 64 through the paged gather (encode) and scatter (decode)."""
    seq = [300, 17, 1025]
    w, pk, x = _paged_setup(seq, D=64, bits=bits, g=g)
    od = oracle_desc(bits, g, 64, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), bits, g)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    _, ox = oracle.decompress(ostream, od)
    pt2 = synth.page_table_for(seq, 16, pk.pool.shape[1], 99, device="cuda")
    pool2 = torch.full_like(pk.pool, 1.5)
    assert gpu_decompress(ostream, kvc.paged_desc(pool2, pt2, seq)) == kvc.KVC_OK
    got = oracle.gather_paged(u16(pool2).reshape(-1), w.layers, w.kv_heads, 64,
                              [s for s in pool2.stride()][:5], 16, seq, pt2.cpu().numpy(), 0,
                              w.vectors)
    assert np.array_equal(got, ox)


@pytest.mark.parametrize("kind", ["zeros", "half_zero_tokens"])
@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32)])
def test_structured_head_dim_64(kind, bits, g):
    """Zero-byte-eliminated code chunks at head_dim 64 (the eliminated-chunk
    decode kernel's 64-channel bodies)."""
    kv = _structured(kind, D=64).cuda()
    s = _roundtrip_dense(kv, bits, g)
    od = oracle_desc(bits, g, 64, 2, 2, [1024])
    sizes, _ = chunk_table(s, od.layout().n_chunks)
    assert (sizes[:od.layout().n_code] < 16384).any()


# ----------------------------------------------------------- full workloads --
# Whole streams and whole decodes at the benchmark's sizes, in its launch
# configuration, against the oracle's thread pool over segments (the same
# bytes as its single-thread calls). Host memory is checked first: a full
# comparison holds the input, the oracle's stream and its decode on the host.
THREADS = max(1, min(os.cpu_count() or 1, 128))


def _need_host_ram(nbytes: int):
    import psutil
    avail = psutil.virtual_memory().available
    if avail < nbytes:
        pytest.skip(f"needs {nbytes / 2**30:.1f} GiB of free host memory, "
                    f"{avail / 2**30:.1f} GiB available")


def _compare_decode(out_rows, ox, piece=1 << 22):
    """out_rows(a, b) -> uint16 [b - a, d] of the GPU decode; ox the oracle's."""
    V = ox.shape[0]
    for a in range(0, V, piece):
        b = min(V, a + piece)
        got = out_rows(a, b)
        if not np.array_equal(got, ox[a:b]):
            i = int(np.flatnonzero((got != ox[a:b]).any(axis=1))[0])
            raise AssertionError(f"decoded vector {a + i} differs from the oracle's")


def _full_dense(w):
    """GPU stream == oracle stream, and GPU decode of it == oracle decode,
    over the whole tensor."""
    _need_host_ram(int(w.raw_bytes * 2.2))
    kv = synth.dense_kv(w, device="cuda")
    x = u16(kv).reshape(-1, w.head_dim)
    od = oracle_desc(w.bits, w.group, w.head_dim, w.layers, w.kv_heads, [w.tokens])
    st, gstream, gbuf, n = gpu_compress(kvc.dense_desc(kv), w.bits, w.group)
    assert st == kvc.KVC_OK
    ost, ostream = oracle.compress(od, x, threads=THREADS)
    assert ost == oracle.OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    del x, gstream
    out = torch.empty_like(kv)
    del kv
    assert gpu_decompress(gbuf, kvc.dense_desc(out), n) == kvc.KVC_OK
    dst, ox = oracle.decompress(ostream, od, threads=THREADS)
    assert dst == oracle.OK
    flat = out.view(-1, w.head_dim)
    _compare_decode(lambda a, b: u16(flat[a:b]), ox)
    del out, flat, gbuf
    torch.cuda.empty_cache()
    return ostream


def test_full_llama8b():
    _full_dense(synth.workload("llama8b"))


def test_full_qwen7b():
    _full_dense(synth.workload("qwen7b"))


def _paged_rows(pk, w, cum):
    """Logical vectors [a, b) of a paged pool by torch indexing on the GPU
    (independent of both codecs)."""
    T = int(cum[-1])
    pt = pk.page_table
    cum_d = torch.tensor(cum, device=pt.device)

    def rows(a, b):
        v = torch.arange(a, b, device=pt.device)
        lkh, u = v // T, v % T
        r = torch.searchsorted(cum_d[1:], u, right=True)
        t = u - cum_d[r]
        page = pt[r, t // w.page_tokens].long()
        lk, h = lkh // w.kv_heads, lkh % w.kv_heads
        return u16(pk.pool[lk // 2, page, lk % 2, h, t % w.page_tokens])
    return rows


def test_full_paged():
    """The paged batch (80 layers, 16 ragged requests, shuffled page table) at
    full size: the whole stream against the oracle's, then the whole decode
    into a second, differently shuffled page table against the oracle's
    decode, with every slot outside the requests left untouched."""
    w = synth.workload("paged")
    _need_host_ram(int(w.raw_bytes * 2.4))
    pk = synth.paged_kv(w, device="cuda")
    seq = w.seq_lens
    cum = np.concatenate([[0], np.cumsum(seq)]).astype(np.int64)
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, seq, origin=1)
    st, gstream, gbuf, n = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), w.bits,
                                        w.group)
    assert st == kvc.KVC_OK
    rows = _paged_rows(pk, w, cum)
    x = np.empty((w.vectors, 128), np.uint16)
    for a in range(0, w.vectors, 1 << 22):
        b = min(w.vectors, a + (1 << 22))
        x[a:b] = rows(a, b)
    ost, ostream = oracle.compress(od, x, threads=THREADS)
    assert ost == oracle.OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    del x, gstream
    # decode into a second pool with another page table, pre-filled with a canary
    pool_shape, n_pages = pk.pool.shape, pk.pool.shape[1]
    del pk
    torch.cuda.empty_cache()
    pt2 = synth.page_table_for(seq, 16, n_pages, 4321, device="cuda")
    pool2 = torch.full(pool_shape, 1.5, dtype=torch.bfloat16, device="cuda")
    assert gpu_decompress(gbuf, kvc.paged_desc(pool2, pt2, seq), n) == kvc.KVC_OK
    del gbuf
    dst, ox = oracle.decompress(ostream, od, threads=THREADS)
    assert dst == oracle.OK
    pk2 = synth.PagedKV(pool2, pt2, seq)
    _compare_decode(_paged_rows(pk2, w, cum), ox)
    # slots that belong to no request still hold the canary
    used = torch.zeros(n_pages, 16, dtype=torch.bool, device="cuda")
    for r, ln in enumerate(seq):
        t = torch.arange(ln, device="cuda")
        used[pt2[r, t // 16].long(), t % 16] = True
    for l in range(w.layers):
        sl = pool2[l].permute(0, 3, 1, 2, 4)[~used]           # [unused slots, 2, H, d]
        assert torch.all(sl == 1.5), f"decode wrote an unused slot in layer {l}"
    del pool2, pk2
    torch.cuda.empty_cache()


# -------------------------------------------------------------------- sweep --
@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("i", list(range(13)))
def test_sweep_full(i, bits):
    """Message-size sweep, every point (T = 8 * 2^i tokens, 1 MiB .. 4 GiB):
    whole streams and whole decodes compared."""
    _full_dense(synth.workload(f"sweep-{i}-{bits}"))
