"""Attention over the compressed cache on the GPU (kvc_attend) against the
oracle's attention in double (reading R18): grouped-query decode attention
for every layer and request, scored and accumulated in the transformed
domain from the stream's codes and meta, no decoded vector written out.

Tolerance, from the arithmetic: the kernels work in fp32 on the decoder's
exact fp32 transformed values. The transformed query carries log2(d) = 7
roundings; each score a 128-term fp32 dot product; the softmax weights
exp(s - m) and their sums fp32 roundings over at most 256 tokens per split
plus the splits' combination; the output one 7-stage fp32 butterfly. Bounded
termwise this is below 1e-3 of the largest |value| of the head, and the
observed errors are orders of magnitude smaller, so the test asks
|out - ref| <= 2e-4 * max|v| + 1e-6 (and reports the worst ratio)."""
import os

import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import gpu_compress, u16

pytestmark = pytest.mark.gpu


def _stream(w, lossless):
    """-> (status, host stream, device stream, bytes, oracle description)."""
    if w.paged:
        pk = synth.paged_kv(w, device="cuda")
        desc = kvc.paged_desc(pk.pool, pk.page_table, w.seq_lens)
        od = oracle.StreamDesc(w.bits, w.group, 128, w.layers, w.kv_heads, w.seq_lens, 0, 1)
    else:
        desc = kvc.dense_desc(synth.dense_kv(w, device="cuda"))
        od = oracle.StreamDesc(w.bits, w.group, 128, w.layers, w.kv_heads, [w.tokens], 0)
    st, s, gbuf, n = gpu_compress(desc, w.bits, w.group, lossless=lossless)
    return st, s, gbuf, n, od


def _check(w, qpk, lossless=0, seed=3, kernel=0):
    L, H, d = w.layers, w.kv_heads, 128
    lens = list(w.seq_lens) if w.paged else [w.tokens]
    dev = torch.device("cuda", 0)
    st, s, gbuf, n, od = _stream(w, lossless)
    assert st == kvc.KVC_OK
    assert s[11] == 0, "attention needs raw code chunks"
    n_req = len(lens)
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randn(L, n_req, H * qpk, d, generator=g, device=dev).to(torch.bfloat16)
    out = torch.full((L, n_req, H * qpk, d), float("nan"), device=dev)
    scale = 1.0 / np.sqrt(d)
    ad = kvc.attn_desc(L, H, qpk, w.bits, w.group, lens, q, out, scale, kernel=kernel)
    wsb = kvc.kvc_attend_workspace_bytes(ad)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    sp = kvc._stream_ptr(None)
    assert kvc.kvc_attend(gbuf.data_ptr(), n, ad, ws.data_ptr(), wsb, sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    threads = max(1, min(os.cpu_count() or 1, 64))
    ost, ref = oracle.attend(s, od, u16(q.cpu()), qpk, scale, threads=threads)
    assert ost == oracle.OK
    _, vals = oracle.decode_values(s, od, threads=threads)
    V = vals.reshape(L, 2, H, sum(lens), d)[:, 1]
    got = out.cpu().numpy().astype(np.float64)
    cum = np.concatenate([[0], np.cumsum(lens)])
    worst = 0.0
    for r in range(n_req):
        if lens[r] == 0:
            assert not got[:, r].any()
            continue
        for h in range(H):
            vmax = np.abs(V[:, h, cum[r]:cum[r + 1]]).max()
            sl = slice(h * qpk, (h + 1) * qpk)
            err = np.abs(got[:, r, sl] - ref[:, r, sl]).max()
            worst = max(worst, err / vmax)
            assert err <= 2e-4 * vmax + 1e-6, (r, h, err, vmax)
    return worst


@pytest.mark.parametrize("kernel", [0, 1])   # tensor cores where supported / CUDA cores
@pytest.mark.parametrize("bits,g", [(4, 128), (4, 64), (4, 32), (2, 128), (2, 64), (2, 32)])
@pytest.mark.parametrize("qpk", [1, 2, 4, 8])
def test_attend_dense_one_request(bits, g, qpk, kernel):
    w = synth.Workload("a", 2, 2, 128, bits, g, seed=bits * 7 + g, kind="lognormal",
                       scale_sigma=1.5, tokens=1000)
    _check(w, qpk, kernel=kernel)


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("qpk", [3, 7])
def test_attend_several_requests_and_search_mode(qpk, kernel):
    """A paged cache with requests of 0, 1, 255, 256, 257 and 700 tokens
    (split boundaries), meta chunks through the search mode's XOR pipelines,
    and a query-head count per kv head that is not a power of two (7: the
    28 query / 4 kv heads of a Qwen2-7B-shaped model)."""
    w = synth.Workload("a", 2, 2, 128, 2, 32, seed=9, kind="outlier_t",
                       seq_lens=[0, 1, 255, 256, 257, 700])
    _check(w, qpk, lossless=kvc.KVC_LOSSLESS_SEARCH, kernel=kernel)


def test_attend_rejects_eliminated_code_chunks_and_bad_arguments():
    dev = torch.device("cuda", 0)
    kv = torch.zeros(1, 2, 2, 2048, 128, dtype=torch.bfloat16, device=dev)
    st, s, gbuf, n = gpu_compress(kvc.dense_desc(kv), 4, 128)
    assert st == kvc.KVC_OK and s[11] == 1             # code chunks stored eliminated
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16, device=dev)
    out = torch.zeros(1, 1, 4, 128, device=dev)
    ad = kvc.attn_desc(1, 2, 2, 4, 128, [2048], q, out, 0.1)
    ws = torch.empty(kvc.kvc_attend_workspace_bytes(ad), dtype=torch.uint8, device=dev)
    sp = kvc._stream_ptr(None)
    assert kvc.kvc_attend(gbuf.data_ptr(), n, ad, ws.data_ptr(), ws.numel(), sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_ERR_CORRUPT
    bad = kvc.attn_desc(1, 2, 9, 4, 128, [2048], q, out, 0.1)   # q_per_kv 9
    assert kvc.kvc_attend_workspace_bytes(bad) == 0
    assert kvc.kvc_attend(gbuf.data_ptr(), n, bad, ws.data_ptr(), ws.numel(),
                          sp) == kvc.KVC_ERR_UNSUPPORTED
    wrong_bits = kvc.attn_desc(1, 2, 2, 2, 128, [2048], q, out, 0.1)
    ws2 = torch.empty(kvc.kvc_attend_workspace_bytes(wrong_bits), dtype=torch.uint8, device=dev)
    assert kvc.kvc_attend(gbuf.data_ptr(), n, wrong_bits, ws2.data_ptr(), ws2.numel(),
                          sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws2.data_ptr(), sp) == kvc.KVC_ERR_CORRUPT


@pytest.mark.parametrize("kernel", [0, 1])
def test_attend_full_llama8b(kernel):
    """The Llama-3-8B-shaped cache (32 layers, 8 kv heads, 4096 tokens) with
    32 query heads (4 per kv head)."""
    w = synth.workload("llama8b")
    worst = _check(w, 4, kernel=kernel)
    print(f"worst error / max|v|: {worst:.3g}")


def test_attend_full_qwen7b():
    """The Qwen-7B-shaped cache (28 layers, 4 kv heads, 32768 tokens, 2-bit
    group 32) with 28 query heads (7 per kv head): 128 splits per head."""
    w = synth.workload("qwen7b")
    worst = _check(w, 7)
    print(f"worst error / max|v|: {worst:.3g}")
