"""Data-dependent errors on the GPU: non-finite input, fp16 meta overflow,
corrupt or mismatched streams and page indices outside the pool set the
workspace status word; nothing is written outside the caller's buffers
(guard bytes around them stay intact). No case here faults, traps or hangs:
every bad input is one the library's own checks turn into a status."""
import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import gpu_compress, gpu_decompress, u16

pytestmark = pytest.mark.gpu


def _kv(T=512, L=2, H=2, seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(L, 2, H, T, 128, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_input(bad):
    kv = _kv()
    kv[1, 0, 1, 100, 17] = bad
    st, _, _, _ = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    assert st == kvc.KVC_ERR_NONFINITE


def test_transform_overflow_is_nonfinite():
    kv = torch.full((1, 2, 1, 256, 128), 3.0e38, dtype=torch.bfloat16)
    st, _, _, _ = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    assert st == kvc.KVC_ERR_NONFINITE


def test_meta_range():
    # one-hot at channel 0 makes y constant = s_0 * x_0; |y| / 8 > 65504 with
    # y negative rounds the fp16 zero point down to -inf
    s0 = -1 if int(oracle.sign_words(0, 128)[0]) & 1 else 1
    kv = torch.zeros((1, 2, 1, 256, 128), dtype=torch.bfloat16)
    kv[..., 0] = -s0 * 655360.0
    st, _, _, _ = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    assert st == kvc.KVC_ERR_RANGE


def test_output_guard_after_capacity():
    kv = _kv().cuda()
    st, host, out, n = gpu_compress(kvc.dense_desc(kv), 4, 128, slack=4096)
    assert st == kvc.KVC_OK
    cap = kvc.kvc_max_compressed_bytes(kvc.dense_desc(kv), kvc.params(4, 128))
    tail = out[cap:].cpu().numpy()
    assert np.all(tail == 0xA5)


def _good_stream():
    kv = _kv(T=2000)
    st, s, _, n = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    assert st == kvc.KVC_OK
    return kv, s


def _decode_guarded(stream: np.ndarray, shape=(2, 2, 2, 2000, 128), n=None):
    """Decode into the middle of a larger buffer; returns (status, guard ok)."""
    numel = int(np.prod(shape))
    big = torch.full((numel + 2 * 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    view = big[4096:4096 + numel].view(shape)
    buf = torch.from_numpy(np.ascontiguousarray(stream)).cuda()
    st = gpu_decompress(buf, kvc.dense_desc(view), nbytes=n)
    g = torch.cat([big[:4096], big[4096 + numel:]])
    return st, bool(torch.all(g == 7.0))


def test_good_stream_decodes():
    kv, s = _good_stream()
    st, guard = _decode_guarded(s)
    assert st == kvc.KVC_OK and guard


@pytest.mark.parametrize("field,offset,value", [
    ("magic", 0, 0x4A), ("version", 4, 2), ("bits", 8, 3), ("k", 9, 4), ("group", 12, 48),
    ("layers", 16, 3), ("kv", 20, 3), ("heads", 24, 5), ("head_dim", 28, 64),
    ("tokens", 32, 0x11), ("n_chunks", 52, 0x77), ("stream_bytes", 61, 0x7F),
    ("flags: an undefined bit", 11, 0x10), ("flags: quantizer id 3", 11, 6)])
def test_corrupt_header(field, offset, value):
    _, s = _good_stream()
    bad = s.copy()
    bad[offset] = value
    st, guard = _decode_guarded(bad)
    assert st == kvc.KVC_ERR_CORRUPT and guard, field


def test_corrupt_table_and_truncation():
    _, s = _good_stream()
    n_chunks = int(s[52:56].view("<u4")[0])
    for i in (0, 3, n_chunks - 1):
        bad = s.copy()
        bad[64 + 8 * i] ^= 0x10                  # size
        st, guard = _decode_guarded(bad)
        assert st == kvc.KVC_ERR_CORRUPT and guard, i
        bad = s.copy()
        bad[64 + 8 * i + 2] ^= 0x01              # offset
        st, guard = _decode_guarded(bad)
        assert st == kvc.KVC_ERR_CORRUPT and guard, i
    st, guard = _decode_guarded(s, n=s.size - 16)  # truncated
    assert st == kvc.KVC_ERR_CORRUPT and guard
    st, guard = _decode_guarded(s[:40], n=40)
    assert st == kvc.KVC_ERR_CORRUPT and guard


def test_corrupt_zero_byte_bitmap():
    kv = _kv(T=2000)
    kv[:, :, :, :1000] = 0                       # mode-1 chunks
    st, s, _, _ = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    n_chunks = int(s[52:56].view("<u4")[0])
    e = s[64:64 + 8 * n_chunks].view("<u8")
    sizes = (e & 0xFFFF).astype(int)
    offs = ((e >> 16) * 16).astype(int)
    base = (64 + 8 * n_chunks + 4 + 15) // 16 * 16
    i = int(np.flatnonzero(sizes < 16384)[0])
    bad = s.copy()
    bad[base + offs[i]] ^= 0x01                  # bitmap popcount no longer matches
    st, guard = _decode_guarded(bad)
    assert st == kvc.KVC_ERR_CORRUPT and guard


def test_code_elimination_flag_cleared():
    """Code chunks that use zero-byte elimination but a header that does not
    announce them: CORRUPT, like the oracle decoder."""
    kv = _kv(T=2000)
    kv[:, :, :, :1000] = 0                       # mode-1 code chunks
    st, s, _, _ = gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)
    assert st == kvc.KVC_OK and s[11] == 1
    bad = s.copy()
    bad[11] = 0
    st, guard = _decode_guarded(bad)
    assert st == kvc.KVC_ERR_CORRUPT and guard
    od = oracle.StreamDesc(4, 128, 128, 2, 2, [2000])
    assert oracle.decompress(bad, od)[0] == oracle.CORRUPT
    assert oracle.decompress(s, od)[0] == oracle.OK


def test_shape_mismatch():
    _, s = _good_stream()
    st, guard = _decode_guarded(s, shape=(2, 2, 2, 1999, 128))
    assert st == kvc.KVC_ERR_CORRUPT and guard


def test_page_index_outside_pool():
    seq = [40, 17]
    w = synth.Workload("p", 2, 2, 128, 4, 64, seed=1, kind="lognormal", seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    pt = pk.page_table.clone()
    pt[1, 0] = pk.pool.shape[1]                  # one past the pool
    st, _, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pt, seq), 4, 64)
    assert st == kvc.KVC_ERR_CORRUPT
    pt[1, 0] = -1
    st, _, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pt, seq), 4, 64)
    assert st == kvc.KVC_ERR_CORRUPT


@pytest.mark.parametrize("page_tokens", [16, 32])
@pytest.mark.parametrize("bad", ["past_pool", "negative"])
def test_page_index_outside_pool_inside_a_long_request(page_tokens, bad):
    """A bad page in the middle of a long request: the blocks over it lie in
    one request, so their load plan (not a row gather) meets the page first;
    the plan falls back to the row gather, which records the bad page. The
    decoder's scatter through such a page table fails the same way."""
    seq = [300, 200]
    w = synth.Workload("p", 2, 2, 128, 4, 64, seed=1, kind="lognormal", seq_lens=seq,
                       page_tokens=page_tokens)
    pk = synth.paged_kv(w, device="cuda")
    st, s, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), 4, 64)
    assert st == kvc.KVC_OK
    pt = pk.page_table.clone()
    pt[0, 96 // page_tokens] = pk.pool.shape[1] if bad == "past_pool" else -1
    st, _, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pt, seq), 4, 64)
    assert st == kvc.KVC_ERR_CORRUPT
    pool2 = torch.zeros_like(pk.pool)
    assert gpu_decompress(s, kvc.paged_desc(pool2, pt, seq)) == kvc.KVC_ERR_CORRUPT


def test_paged_receiver_request_mismatch():
    seq = [40, 17]
    w = synth.Workload("p", 2, 2, 128, 4, 64, seed=1, kind="lognormal", seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    st, s, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), 4, 64)
    assert st == kvc.KVC_OK
    other = [17, 40]                              # same total, different split
    pt2 = synth.page_table_for(other, 16, pk.pool.shape[1], 5, device="cuda")
    pool2 = torch.zeros_like(pk.pool)
    assert gpu_decompress(s, kvc.paged_desc(pool2, pt2, other)) == kvc.KVC_ERR_CORRUPT
    dense = torch.zeros((2, 2, 2, 57, 128), dtype=torch.bfloat16, device="cuda")
    assert gpu_decompress(s, kvc.dense_desc(dense)) == kvc.KVC_OK


def test_status_is_cleared_per_call():
    kv = _kv()
    kv[0, 0, 0, 0, 0] = float("nan")
    assert gpu_compress(kvc.dense_desc(kv.cuda()), 4, 128)[0] == kvc.KVC_ERR_NONFINITE
    assert gpu_compress(kvc.dense_desc(_kv().cuda()), 4, 128)[0] == kvc.KVC_OK


def test_compaction_wait_runs_out_to_timeout():
    """A bounded device wait that runs out ends the call with KVC_ERR_TIMEOUT
    and leaves the context usable. The test entry point starts the
    compaction's tickets one chunk late, so the first shrinking code chunk is
    never read and its read flag never set; the next chunk stores into that
    chunk's slot and waits for the flag, which runs out after 1 ms. Writes stay
    inside the output buffer (guard bytes after it intact), and an ordinary
    compress on the same stream afterwards still matches the oracle."""
    L, H, T, D = 2, 4, 4096, 128
    g = torch.Generator().manual_seed(21)
    x = torch.randn(L, 2, H, T, D, generator=g)
    blocks = x.view(L, 2, H, T // 256, 256, D)
    zero = torch.rand(L, 2, H, T // 256, generator=g) < 0.5
    blocks[zero] = 0
    kv = x.to(torch.bfloat16).cuda()
    desc = kvc.dense_desc(kv)
    p = kvc.params(4, 128, 0)
    cap = kvc.kvc_max_compressed_bytes(desc, p)
    wsb = kvc.kvc_workspace_bytes(desc, p)
    out = torch.full((cap + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    nb = torch.zeros(1, dtype=torch.int64, device="cuda")
    sp = kvc._stream_ptr(None)
    # invalid hook arguments are refused before anything runs
    for skip, ns in [(0, 10**6), (1, 0), (1, 2 * 10**9)]:
        assert kvc.kvc_test_compress_stalled(desc, p, out.data_ptr(), cap, nb.data_ptr(),
                                             ws.data_ptr(), wsb, skip, ns,
                                             sp) == kvc.KVC_ERR_INVALID_ARG
    st = kvc.kvc_test_compress_stalled(desc, p, out.data_ptr(), cap, nb.data_ptr(),
                                       ws.data_ptr(), wsb, 1, 10**6, sp)
    assert st == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_ERR_TIMEOUT
    assert torch.all(out[cap:] == 0xA5), "a write went past the output buffer"
    # the context is still usable: the ordinary call gives the oracle's stream
    st, gstream, _, _ = gpu_compress(desc, 4, 128)
    assert st == kvc.KVC_OK
    od = oracle.StreamDesc(4, 128, D, L, H, [T], 0)
    ost, ostream = oracle.compress(od, u16(kv.cpu()).reshape(-1, D))
    assert ost == oracle.OK and ostream[11] == 1       # code chunks stored eliminated
    assert np.array_equal(gstream, ostream)
