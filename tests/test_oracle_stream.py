"""Pins of the oracle's stream layer: the header against a hand-written golden,
layout counts against hand arithmetic, the whole-codec error bound, corrupt
streams, and the logical vector order of dense and paged gathers against
independent numpy/torch indexing."""
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_04_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _u(b, off, n):
    return int.from_bytes(bytes(b[off:off + n]), "little")


def tiny_desc_and_vectors():
    w = synth.workload("tiny")
    kv = synth.dense_kv(w)
    x = synth.bf16_bits(kv).reshape(-1, w.head_dim)   # contiguous = logical order
    d = oracle.StreamDesc(w.bits, w.group, w.head_dim, w.layers, w.kv_heads,
                          [w.tokens], w.sign_seed)
    return w, d, x


def test_header_golden():
    _, d, x = tiny_desc_and_vectors()
    st, s = oracle.compress(d, x)
    assert st == oracle.OK
    rows = {}
    with open(os.path.join(GOLDEN, "header_tiny.txt")) as f:
        for l in f:
            l = l.split("#")[0].split()
            if l:
                rows[l[0]] = l[1:]
    for key, val in rows.items():
        if key.isdigit():
            assert _u(s, int(key), int(val[0])) == int(val[1], 0), key
    lay = d.layout()
    assert lay.data_base == int(rows["data_base"][0])
    assert d.max_bytes() == int(rows["max_bytes"][0])
    assert _u(s, 56, 8) == s.size                               # stream_bytes
    assert _u(s, 64 + 8 * 5, 4) == 64                           # token length
    assert not s[64 + 8 * 5 + 4:112].any()                      # zero padding


@pytest.mark.parametrize("zero_chunk", [False, True])
def test_header_flag_code_elimination(zero_chunk):
    """Header byte 11, bit 0 says whether some code chunk uses zero-byte
    elimination: an all-zero tensor's 16 KB code chunks are all-zero codes
    (2048-byte bitmap only); random data gives none."""
    w, d, x = tiny_desc_and_vectors()
    if zero_chunk:
        x = x.copy()
        x[:256] = 0                      # the first code chunk's 256 vectors
    st, s = oracle.compress(d, x)
    assert st == oracle.OK
    sizes = np.frombuffer(bytes(s[64:64 + 8 * 5]), "<u8") & 0xFFFF
    assert (sizes[:4] < 16384).any() == zero_chunk
    assert s[11] == (1 if zero_chunk else 0)
    st, y = oracle.decompress(s, d)
    assert st == oracle.OK


def test_code_elim_rule_arithmetic():
    """Reading R16 by hand: S = padded bytes saved, T = padded bytes from the
    first shrinking code chunk on; elimination is kept iff 64 * S >= T."""
    F = 16384
    pays = oracle.code_elim_pays
    assert not pays([F] * 5, [F] * 5)                         # nothing shrinks
    assert not pays([], [])
    # one all-zero chunk (bitmap only, saves 14336 = 56 * 256) at position 1:
    # T = 56 chunks -> 64 * 14336 = 917504 = T, kept (tie); 57 chunks -> not
    assert pays([F, 2048] + [F] * 55, [F] * 57)
    assert not pays([F, 2048] + [F] * 56, [F] * 58)
    # chunks before the first shrinking one are not part of T
    assert pays([F] * 1000 + [2048] + [F] * 55, [F] * 1056)
    # sizes count padded: 2049 -> 2064 saves 14320, so 56 chunks no longer pay
    assert not pays([2049] + [F] * 55, [F] * 56)
    assert pays([2049] + [F] * 54, [F] * 55)
    # a short last chunk counts with its padded length: 55 full + 1000 -> 1008
    assert pays([2048] + [F] * 54 + [1000], [F] * 55 + [1000])
    # two shrinking chunks: S adds up
    assert pays([2048, F, 2048] + [F] * 109, [F] * 112)
    assert not pays([2048, F, 2048] + [F] * 110, [F] * 113)


def _one_zero_chunk(bits, group, zero_chunk, n_code=64, seed=11):
    """Random vectors except the `zero_chunk`-th code chunk's vectors, which
    are zero: all-zero codes, stored as the 2048-byte bitmap alone when
    eliminated."""
    per = 16384 * 8 // (128 * bits)                           # vectors per code chunk
    V = per * n_code
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(V, 128, generator=g)
    x[zero_chunk * per:(zero_chunk + 1) * per] = 0
    x = synth.bf16_bits(x.to(torch.bfloat16)).reshape(V, 128)
    d = oracle.StreamDesc(bits, group, 128, 1, V // 2048, [1024], 0)
    return d, x


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 32)])
@pytest.mark.parametrize("zero_chunk,kept", [(8, True), (7, False), (63, True), (0, False)])
def test_code_elim_rule_in_stream(bits, group, zero_chunk, kept):
    """64 code chunks, one of them all-zero codes: eliminated (and the later
    chunks shifted) only if the 56 * 256 saved bytes are at least 1/64 of the
    code chunks from it to the end, i.e. if at most 56 chunks remain."""
    d, x = _one_zero_chunk(bits, group, zero_chunk)
    lay = d.layout()
    assert lay.n_code == 64
    st, s = oracle.compress(d, x)
    assert st == oracle.OK
    table = np.frombuffer(bytes(s[64:64 + 8 * lay.n_chunks]), "<u8")
    code = [int(table[oracle.code_chunk_index(lay, c)] & 0xFFFF) for c in range(64)]
    assert code[zero_chunk] == (2048 if kept else 16384)
    assert all(code[c] == 16384 for c in range(64) if c != zero_chunk)
    assert s[11] == (1 if kept else 0)
    st, y = oracle.decompress(s, d)
    assert st == oracle.OK
    zero = y[zero_chunk * (lay.V // 64):(zero_chunk + 1) * (lay.V // 64)]
    assert not (zero & 0x7FFF).any()                          # +-0 (signs flip zeros)


@pytest.mark.parametrize("pattern", range(6))
def test_code_elim_rule_matches_per_chunk_sizes(pattern):
    """The stream's code sizes and flag follow from the separately pinned
    parts: each code chunk's own lossless encoding (raw codes from the
    quantizer) and the rule on those sizes; random sets of all-zero chunks
    among 64, some of which keep elimination and some not."""
    rng = np.random.default_rng(100 + pattern)
    zeros = sorted(rng.choice(64, size=int(rng.integers(1, 5)), replace=False).tolist())
    if pattern == 0:
        zeros = [3]                                           # a long tail: raw
    if pattern == 1:
        zeros = [60, 61, 62]                                  # a short tail: kept
    d, x = _one_zero_chunk(4, 128, zeros[0], seed=20 + pattern)
    for z in zeros[1:]:
        x[z * 256:(z + 1) * 256] = 0
    lay = d.layout()
    st, codes, _ = oracle.quantize_vectors(x, 4, 128, 0)
    assert st == oracle.OK
    lens = [16384] * 64
    sizes = [oracle.lossless_encode_chunk(codes[c * 256:(c + 1) * 256].reshape(-1)).size
             for c in range(64)]
    keep = oracle.code_elim_pays(sizes, lens)
    st, s = oracle.compress(d, x)
    assert st == oracle.OK
    table = np.frombuffer(bytes(s[64:64 + 8 * lay.n_chunks]), "<u8")
    got = [int(table[oracle.code_chunk_index(lay, c)] & 0xFFFF) for c in range(64)]
    assert got == (sizes if keep else lens)
    assert s[11] == int(keep)
    if pattern == 0:
        assert not keep
    if pattern == 1:
        assert keep
    assert oracle.decompress(s, d)[0] == oracle.OK


@pytest.mark.parametrize("name,n_code,n_meta", [("tiny", 4, 1), ("llama8b", 8192, 512),
                                                ("qwen7b", 14336, 7168)])
def test_layout_counts(name, n_code, n_meta):
    """Hand arithmetic: code chunks = V*d*b/8/16384, meta chunks =
    V*(d/g)*4/16384 (rounded up)."""
    w = synth.workload(name)
    d = oracle.StreamDesc(w.bits, w.group, w.head_dim, w.layers, w.kv_heads,
                          [w.tokens])
    lay = d.layout()
    assert lay.V == w.vectors
    assert (lay.n_code, lay.n_meta, lay.n_chunks) == (n_code, n_meta, n_code + n_meta)
    assert lay.code_per_seg == w.group * w.bits // 32


def test_chunk_order_codes_then_meta():
    lay = oracle.StreamDesc(2, 32, 128, 1, 1, [1250]).layout()   # V = 2500, R = 2
    assert lay.code_per_seg == 2 and lay.n_code == 5 and lay.n_meta == 3
    idx = sorted([("c", c, oracle.code_chunk_index(lay, c)) for c in range(5)] +
                 [("m", s, oracle.meta_chunk_index(lay, s)) for s in range(3)],
                 key=lambda t: t[2])
    assert [(k, i) for k, i, _ in idx] == [("c", 0), ("c", 1), ("c", 2), ("c", 3),
                                           ("c", 4), ("m", 0), ("m", 1), ("m", 2)]
    assert [t[2] for t in idx] == list(range(8))


def test_roundtrip_error_bound_tiny():
    """x^ - x = D H (y^ - y) / d up to the final bf16 rounding, and H/sqrt(d)
    is orthonormal, so ||x^ - x||_2 <= ||y^ - y||_2 / sqrt(d) + bf16 term,
    with |y^ - y| <= sf/2 per element in each group."""
    w, d, x = tiny_desc_and_vectors()
    st, s = oracle.compress(d, x)
    assert st == oracle.OK and s.size <= d.max_bytes()
    st, xh = oracle.decompress(s, d)
    assert st == oracle.OK
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).double().numpy()
    xhf = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).double().numpy()
    _, codes, meta = oracle.quantize_vectors(x, w.bits, w.group, 0)
    sh = meta.reshape(x.shape[0], -1, 4)
    sh = (sh[..., 0].astype(np.uint16) | (sh[..., 1].astype(np.uint16) << 8)).view(np.float16)
    sf = sh.astype(np.float64) * 8
    ybound = np.sqrt((sf / 2) ** 2 * w.group).sum(axis=1) if sf.shape[1] == 1 else \
        np.sqrt(((sf / 2) ** 2 * w.group).sum(axis=1))
    err = np.linalg.norm(xhf - xf, axis=1)
    bf16_term = np.linalg.norm(xhf, axis=1) * 2.0 ** -8
    assert np.all(err <= ybound / np.sqrt(w.head_dim) * (1 + 1e-4) + bf16_term)
    # and it is a real codec: 4-bit relative error well below 1
    assert err.mean() / np.linalg.norm(xf, axis=1).mean() < 0.15


def test_stream_is_deterministic_and_segments_agree():
    """Three segments (R = 2 code chunks per meta chunk at 2-bit, group 32):
    each chunk of encode_segment sits in the stream at the index the layout
    gives it, and offsets are the prefix sum of padded sizes."""
    w = synth.Workload("t", 1, 2, 128, 2, 32, seed=3, kind="lognormal", tokens=600)
    x = synth.bf16_bits(synth.dense_kv(w)).reshape(-1, 128)
    d = oracle.StreamDesc(2, 32, 128, 1, 2, [600])
    st1, s1 = oracle.compress(d, x)
    st2, s2 = oracle.compress(d, x)
    assert st1 == oracle.OK and np.array_equal(s1, s2)
    lay = d.layout()
    assert lay.n_code == 5 and lay.n_seg == 3       # 2400 vectors, 512 per code chunk
    sizes = [_u(s1, 64 + 8 * i, 8) & 0xFFFF for i in range(lay.n_chunks)]
    offs = [(_u(s1, 64 + 8 * i, 8) >> 16) * 16 for i in range(lay.n_chunks)]
    assert offs == [sum((z + 15) // 16 * 16 for z in sizes[:i]) for i in range(lay.n_chunks)]
    for seg in range(lay.n_seg):
        v0, v1 = oracle.segment_vectors(lay, seg)
        st, chunks, _ = oracle.encode_segment(d, seg, x[v0:v1])
        idx = [oracle.code_chunk_index(lay, seg * lay.code_per_seg + i)
               for i in range(len(chunks) - 1)] + [oracle.meta_chunk_index(lay, seg)]
        for i, ch in zip(idx, chunks):
            a = lay.data_base + offs[i]
            assert sizes[i] == ch.size and np.array_equal(s1[a:a + ch.size], ch)


def test_corrupt_streams():
    _, d, x = tiny_desc_and_vectors()
    _, s = oracle.compress(d, x)
    assert oracle.decompress(s[:-16], d)[0] == oracle.CORRUPT       # truncated
    for off, val in ((0, 0x4A), (8, 2), (12, 64), (24, 4), (52, 6)):
        bad = s.copy()
        bad[off] = val
        assert oracle.decompress(bad, d)[0] == oracle.CORRUPT, off
    bad = s.copy()
    bad[64] ^= 0x10                                                   # chunk 0 size
    assert oracle.decompress(bad, d)[0] == oracle.CORRUPT
    bad = s.copy()
    bad[64 + 8 + 2] ^= 0x01                                           # chunk 1 offset
    assert oracle.decompress(bad, d)[0] == oracle.CORRUPT
    bad = s.copy()
    bad[11] = 2                                                       # unknown flag bit
    assert oracle.decompress(bad, d)[0] == oracle.CORRUPT
    bad[11] = 1                   # announced elimination that no chunk uses: accepted
    assert oracle.decompress(bad, d)[0] == oracle.OK


def test_mode1_chunks_roundtrip():
    """Half of the tokens zero: code chunks of zero vectors compress to a
    bitmap plus few bytes; the stream still decodes bit-exactly to what the
    per-vector decode gives."""
    w, d, x = tiny_desc_and_vectors()
    x = x.copy()
    x[: x.shape[0] // 2] = 0
    st, s = oracle.compress(d, x)
    assert st == oracle.OK
    lay = d.layout()
    sizes = [_u(s, 64 + 8 * i, 8) & 0xFFFF for i in range(lay.n_chunks)]
    assert min(sizes[:2]) < 16384                                     # mode-1 chunks
    assert s[11] == 1
    bad = s.copy()
    bad[11] = 0                                  # not announced: corrupt
    assert oracle.decompress(bad, d)[0] == oracle.CORRUPT
    st, xh = oracle.decompress(s, d)
    _, codes, meta = oracle.quantize_vectors(x, w.bits, w.group, 0)
    ref = oracle.dequantize_vectors(codes, meta, 128, w.bits, w.group, 0)
    assert st == oracle.OK and np.array_equal(xh, ref)


def test_empty_stream():
    d = oracle.StreamDesc(4, 128, 128, 2, 8, [0])
    st, s = oracle.compress(d, np.zeros((0, 128), np.uint16))
    assert st == oracle.OK and s.size == d.layout().data_base == 80
    st, xh = oracle.decompress(s, d)
    assert st == oracle.OK and xh.shape == (0, 128)


def test_gather_dense_matches_permuted_indexing():
    rng = np.random.default_rng(0)
    L, H, T, D = 2, 3, 5, 64
    store = rng.integers(0, 65536, (T, L, H, 2, D)).astype(np.uint16)   # odd layout
    st = [s // 2 for s in store.strides]                              # elements
    strides = (st[1], st[3], st[2], st[0])                            # layer, kv, head, token
    out = oracle.gather_dense(store.reshape(-1), L, H, T, D, strides, 0, L * 2 * H * T)
    ref = store.transpose(1, 3, 2, 0, 4).reshape(-1, D)               # [l][kv][h][t]
    assert np.array_equal(out, ref)
    out2 = oracle.gather_dense(store.reshape(-1), L, H, T, D, strides, 7, 23)
    assert np.array_equal(out2, ref[7:23])


def test_gather_paged_matches_python_walk():
    w = synth.Workload("t", 2, 2, 64, 4, 64, 5, "lognormal", seq_lens=[20, 0, 33, 16])
    pk = synth.paged_kv(w)
    pool = synth.bf16_bits(pk.pool)
    pt = pk.page_table.numpy()
    ref = []
    for l in range(2):
        for kv in range(2):
            for h in range(2):
                for r, n in enumerate(w.seq_lens):
                    for t in range(n):
                        ref.append(pool[l, pt[r, t // 16], kv, h, t % 16])
    ref = np.array(ref)
    out = oracle.gather_paged(pool.reshape(-1), 2, 2, 64, pk.strides(), 16, w.seq_lens,
                              pt, 0, len(ref))
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("threads", [2, 3, 8])
def test_threaded_oracle_equals_single_thread(threads):
    """The thread-pool compress/decompress (the per-segment loop spread over
    POSIX threads) give the single-thread calls' bytes and status: a mixed
    lognormal input with all-zero stretches (eliminated code and meta chunks,
    reading R16 both ways), a ragged tail, and more segments than threads."""
    w = synth.Workload("m", 3, 2, 128, 2, 32, seed=5, kind="lognormal", scale_sigma=1.5,
                       tokens=1500)
    x = synth.bf16_bits(synth.dense_kv(w)).reshape(-1, 128).copy()
    x[4000:6200] = 0
    for bits, g in [(2, 32), (4, 64), (4, 128)]:
        d = oracle.StreamDesc(bits, g, 128, 3, 2, [1500], 7)
        st1, s1 = oracle.compress(d, x)
        stn, sn = oracle.compress(d, x, threads=threads)
        assert st1 == stn == oracle.OK and np.array_equal(s1, sn)
        dst1, x1 = oracle.decompress(s1, d)
        dstn, xn = oracle.decompress(s1, d, threads=threads)
        assert dst1 == dstn == oracle.OK and np.array_equal(x1, xn)


def test_threaded_oracle_first_error_in_segment_order():
    """With errors in several segments the threaded call reports the one of
    the lowest segment, as the single-thread loop does: RANGE in segment 1,
    NONFINITE in segment 3 -> RANGE; swapped -> NONFINITE."""
    d = oracle.StreamDesc(4, 128, 128, 1, 1, [2048 * 4], 0)
    lay = d.layout()
    assert lay.n_seg == 4
    s0 = -1 if oracle.sign_words(0, 128)[0] & 1 else 1     # sign of channel 0
    big = np.float32(-s0 * 655360.0).view(np.uint32) >> 16   # one-hot -> RANGE
    for rng_seg, nan_seg, want in [(1, 3, oracle.RANGE), (3, 1, oracle.NONFINITE)]:
        x = np.zeros((lay.V, 128), np.uint16)
        v0, _ = oracle.segment_vectors(lay, rng_seg)
        x[v0, 0] = big
        v1, _ = oracle.segment_vectors(lay, nan_seg)
        x[v1, 5] = 0x7FC0
        st1, s1 = oracle.compress(d, x)
        st4, s4 = oracle.compress(d, x, threads=4)
        assert st1 == st4 == want and np.array_equal(s1, s4)


def _search_desc(bits, g, L, H, T, seed=0, mode=None):
    return oracle.StreamDesc(bits, g, 128, L, H, [T], seed,
                             lossless=oracle.LOSSLESS_SEARCH if mode is None else mode)


def _entries(stream, n_chunks):
    e = stream[64:64 + 8 * n_chunks].view("<u8").astype(np.uint64)
    return (e & 0xFFFF).astype(np.int64), (e >> 60).astype(np.int64)


@pytest.mark.parametrize("bits,g", [(4, 128), (4, 64), (2, 32)])
def test_search_mode_round_trip_and_table_ids(bits, g):
    """Search-mode streams decode to the fixed-mode decode (the lossless
    stage is exact), their meta chunks use the XOR pipelines on these inputs
    and are shorter than in the fixed mode, and each table entry's id equals
    the one encode_segment chose for that chunk."""
    w = synth.Workload("s", 2, 4, 128, bits, g, seed=3, kind="lognormal", scale_sigma=1.5,
                       tokens=4096)
    x = synth.bf16_bits(synth.dense_kv(w)).reshape(-1, 128)
    ds, df = _search_desc(bits, g, 2, 4, 4096), _search_desc(bits, g, 2, 4, 4096,
                                                              mode=oracle.LOSSLESS_FIXED)
    st, s = oracle.compress(ds, x)
    stf, sf = oracle.compress(df, x)
    assert st == stf == oracle.OK
    lay = ds.layout()
    sizes, ids = _entries(s, lay.n_chunks)
    fsizes, fids = _entries(sf, lay.n_chunks)
    meta = [oracle.meta_chunk_index(lay, k) for k in range(lay.n_meta)]
    assert not fids.any()
    assert set(ids[meta].tolist()) <= {1, 3} and sizes[meta].sum() < fsizes[meta].sum()
    for seg in (0, lay.n_seg - 1):
        v0, v1 = oracle.segment_vectors(lay, seg)
        _, chunks, pipes = oracle.encode_segment(ds, seg, x[v0:v1])
        assert pipes[-1] == ids[oracle.meta_chunk_index(lay, seg)]
        assert chunks[-1].size == sizes[oracle.meta_chunk_index(lay, seg)]
    dst, y = oracle.decompress(s, ds)
    dstf, yf = oracle.decompress(sf, df)
    assert dst == dstf == oracle.OK and np.array_equal(y, yf)
    # the thread pool gives the same bytes in search mode
    st4, s4 = oracle.compress(ds, x, threads=4)
    assert st4 == oracle.OK and np.array_equal(s4, s)


@pytest.mark.parametrize("zero_chunk,fixed_kept,search_kept", [(1, False, True), (7, False, True),
                                                                (8, True, True), (0, False, False)])
def test_code_rule_threshold_moves_with_search(zero_chunk, fixed_kept, search_kept):
    """Reading R16 with the chosen sizes: an all-zero code chunk saves
    16384 - 2048 padded bytes in the fixed mode and 16384 - 256 in the search
    mode (two-level form), so among 64 code chunks elimination is kept when
    at most 56 (fixed) or 63 (search) chunks follow from it, itself
    included: 64 * 14336 = 917504 >= 56 * 16384, 64 * 16128 = 1032192 ==
    63 * 16384."""
    per = 16384 * 8 // (128 * 4)
    V = per * 64
    x = torch.randn(V, 128, generator=torch.Generator().manual_seed(11))
    x[zero_chunk * per:(zero_chunk + 1) * per] = 0
    xb = synth.bf16_bits(x.to(torch.bfloat16))
    for mode, kept, size in [(oracle.LOSSLESS_FIXED, fixed_kept, 2048),
                             (oracle.LOSSLESS_SEARCH, search_kept, 256)]:
        d = oracle.StreamDesc(4, 128, 128, 1, V // 2048, [1024], 0, lossless=mode)
        st, s = oracle.compress(d, xb)
        assert st == oracle.OK
        sizes, ids = _entries(s, d.layout().n_chunks)
        assert sizes[zero_chunk] == (size if kept else 16384), mode
        assert ids[zero_chunk] == (2 if kept and size == 256 else 0)
        assert s[11] == (1 if kept else 0)
        dst, y = oracle.decompress(s, d)
        assert dst == oracle.OK and np.array_equal(y, oracle.decompress(
            oracle.compress(oracle.StreamDesc(4, 128, 128, 1, V // 2048, [1024], 0), xb)[1],
            oracle.StreamDesc(4, 128, 128, 1, V // 2048, [1024], 0))[1])


def test_decoder_rejects_bad_pipeline_ids():
    """A table id above 3, a nonzero id on a raw chunk, and an XOR id on a
    code chunk are corrupt streams."""
    w = synth.Workload("s", 1, 2, 128, 2, 32, seed=4, kind="lognormal", scale_sigma=1.5,
                       tokens=4096)
    x = synth.bf16_bits(synth.dense_kv(w)).reshape(-1, 128).copy()
    x[:512] = 0                                         # an all-zero code chunk (id 2)
    d = _search_desc(2, 32, 1, 2, 4096)
    st, s = oracle.compress(d, x)
    lay = d.layout()
    sizes, ids = _entries(s, lay.n_chunks)
    assert st == oracle.OK and ids[0] == 2 and s[11] == 1
    m = oracle.meta_chunk_index(lay, 0)
    raw = next(i for i in range(lay.n_code) if sizes[i] == 16384)

    def with_id(i, new_id):
        t = s.copy()
        e = t[64 + 8 * i:72 + 8 * i].view("<u8")
        e[0] = (int(e[0]) & ((1 << 60) - 1)) | (new_id << 60)
        return t
    assert oracle.decompress(s, d)[0] == oracle.OK
    for i, new_id in [(m, 4), (m, 15), (raw, 2), (0, 1), (0, 3)]:
        assert oracle.decompress(with_id(i, new_id), d)[0] == oracle.CORRUPT, (i, new_id)
