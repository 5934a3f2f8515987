"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded bytes. Streams must be byte-identical (codes, meta, chunk table,
lossless chunks); decoded bf16 must be bit-identical (the 1-ulp tolerance
allowed for decoded values is not needed: both sides run the same fp32
operation sequence with round-to-nearest-even and no contraction).

Sizes: small shapes that still span several tiles, segments and a ragged tail
(oracle in seconds), structured inputs that exercise zero-byte elimination,
and the full-size workloads in the benchmark's launch configuration (full
comparison for llama8b, sampled segments for qwen7b and the paged batch)."""
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
def _paged_setup(seq, L=2, H=3, D=128, bits=4, g=64, seed=3):
    w = synth.Workload("p", L, H, D, bits, g, seed=seed, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    pool = u16(pk.pool)
    x = oracle.gather_paged(pool.reshape(-1), L, H, D, pk.strides(), 16, seq,
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
def _segment_check(w, od, gstream, x_of_range, segs):
    """Compare the chunks of sampled segments with the oracle's, and the table's
    offsets with the prefix sum of padded sizes."""
    lay = od.layout()
    sizes, offs = chunk_table(gstream, lay.n_chunks)
    padded = (sizes + 15) // 16 * 16
    assert np.array_equal(offs[1:], np.cumsum(padded)[:-1]) and offs[0] == 0
    assert gstream.size == lay.data_base + offs[-1] + padded[-1]
    for s in segs:
        v0, v1 = oracle.segment_vectors(lay, s)
        st, chunks = oracle.encode_segment(od, s, x_of_range(v0, v1))
        assert st == oracle.OK
        idx = [oracle.code_chunk_index(lay, s * lay.code_per_seg + i)
               for i in range(len(chunks) - 1)] + [oracle.meta_chunk_index(lay, s)]
        for ch, ci in zip(chunks, idx):
            assert sizes[ci] == ch.size, (s, ci)
            a = lay.data_base + offs[ci]
            assert np.array_equal(gstream[a:a + ch.size], ch), (s, ci)
    return sizes, offs


def test_full_llama8b():
    w = synth.workload("llama8b")
    kv = synth.dense_kv(w, device="cuda")
    x = u16(kv).reshape(-1, 128)
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, [w.tokens])
    st, gstream, _, _ = gpu_compress(kvc.dense_desc(kv), w.bits, w.group)
    assert st == kvc.KVC_OK
    ost, ostream = oracle.compress(od, x)
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    out = torch.empty_like(kv)
    assert gpu_decompress(gstream, kvc.dense_desc(out)) == kvc.KVC_OK
    lay = od.layout()
    got = u16(out).reshape(-1, 128)
    for s in [0, 1, 77, 255, lay.n_seg - 1]:
        v0, v1 = oracle.segment_vectors(lay, s)
        _, chunks = oracle.encode_segment(od, s, x[v0:v1])
        dst, ref = oracle.decode_segment(od, s, chunks, v1 - v0)
        assert dst == oracle.OK and np.array_equal(got[v0:v1], ref), s


def test_full_qwen7b_sampled():
    w = synth.workload("qwen7b")
    kv = synth.dense_kv(w, device="cuda")
    flat = kv.view(-1, 128)
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, [w.tokens])
    st, gstream, _, _ = gpu_compress(kvc.dense_desc(kv), w.bits, w.group)
    assert st == kvc.KVC_OK
    lay = od.layout()
    rng = np.random.default_rng(0)
    segs = sorted({0, 1, int(lay.n_seg) - 1, *rng.integers(0, lay.n_seg, 12).tolist()})
    _segment_check(w, od, gstream, lambda a, b: u16(flat[a:b]), segs)
    out = torch.empty_like(kv)
    assert gpu_decompress(gstream, kvc.dense_desc(out)) == kvc.KVC_OK
    oflat = out.view(-1, 128)
    for s in segs[:6]:
        v0, v1 = oracle.segment_vectors(lay, s)
        _, chunks = oracle.encode_segment(od, s, u16(flat[v0:v1]))
        _, ref = oracle.decode_segment(od, s, chunks, v1 - v0)
        assert np.array_equal(u16(oflat[v0:v1]), ref), s


def test_full_paged_sampled():
    w = synth.workload("paged")
    pk = synth.paged_kv(w, device="cuda")
    seq = w.seq_lens
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, seq, origin=1)
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), w.bits,
                                     w.group)
    assert st == kvc.KVC_OK
    lay = od.layout()
    # logical vectors of a range via torch indexing (independent of both sides)
    cum = np.concatenate([[0], np.cumsum(seq)])
    T = int(cum[-1])
    pt = pk.page_table

    def rows(a, b):
        v = torch.arange(a, b, device="cuda")
        lkh, u = v // T, v % T
        r = torch.searchsorted(torch.tensor(cum[1:], device="cuda"), u, right=True)
        t = u - torch.tensor(cum, device="cuda")[r]
        page = pt[r, t // 16].long()
        lk, h = lkh // w.kv_heads, lkh % w.kv_heads
        return u16(pk.pool[lk // 2, page, lk % 2, h, t % 16])

    rng = np.random.default_rng(1)
    segs = sorted({0, int(lay.n_seg) - 1, *rng.integers(0, lay.n_seg, 10).tolist()})
    _segment_check(w, od, gstream, rows, segs)
    del pk
    torch.cuda.empty_cache()


# -------------------------------------------------------------------- sweep --
@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("i", [0, 2, 5])
def test_sweep_small_sizes_full(i, bits):
    """Message-size sweep, small end (T = 8 * 2^i tokens): whole streams and
    whole decodes compared."""
    w = synth.workload(f"sweep-{i}-{bits}")
    kv = synth.dense_kv(w, device="cuda")
    _roundtrip_dense(kv, w.bits, w.group)


@pytest.mark.parametrize("bits", [4, 2])
def test_sweep_largest_size_sampled(bits):
    """Message-size sweep, 4 GiB end (T = 32768): chunk table consistency over
    the whole stream, sampled segments against the oracle, sampled decode."""
    w = synth.workload(f"sweep-12-{bits}")
    kv = synth.dense_kv(w, device="cuda")
    flat = kv.view(-1, 128)
    od = oracle_desc(w.bits, w.group, 128, w.layers, w.kv_heads, [w.tokens])
    st, gstream, _, _ = gpu_compress(kvc.dense_desc(kv), w.bits, w.group)
    assert st == kvc.KVC_OK
    lay = od.layout()
    rng = np.random.default_rng(12 + bits)
    segs = sorted({0, int(lay.n_seg) - 1, *rng.integers(0, lay.n_seg, 6).tolist()})
    _segment_check(w, od, gstream, lambda a, b: u16(flat[a:b]), segs)
    out = torch.empty_like(kv)
    assert gpu_decompress(gstream, kvc.dense_desc(out)) == kvc.KVC_OK
    oflat = out.view(-1, 128)
    for s in segs[:3]:
        v0, v1 = oracle.segment_vectors(lay, s)
        _, chunks = oracle.encode_segment(od, s, u16(flat[v0:v1]))
        _, ref = oracle.decode_segment(od, s, chunks, v1 - v0)
        assert np.array_equal(u16(oflat[v0:v1]), ref), s
    del kv, out, flat, oflat
    torch.cuda.empty_cache()
