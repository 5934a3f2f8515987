"""The measurement entry points kvc_compress_timed / kvc_decompress_timed do
the ordinary calls' work (same stream bytes, same decode) and record their
five events in order around the four kernels of each call."""
import numpy as np
import pytest
import torch

import bench
import kv_cache_compression_04_b200 as kvc
from kv_cache_compression_04_b200 import synth
from kvc_testutil import gpu_compress, u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("paged", [False, True])
def test_timed_calls_match_ordinary_calls(paged):
    w = synth.Workload("t", 2, 4, 128, 4, 64, seed=8, kind="lognormal", scale_sigma=1.5,
                       tokens=3000, seq_lens=[700, 1200, 33] if paged else [])
    dev = torch.device("cuda", 0)
    if paged:
        pk = synth.paged_kv(w, device=dev)
        desc = kvc.paged_desc(pk.pool, pk.page_table, w.seq_lens)
    else:
        kv = synth.dense_kv(w, device=dev)
        desc = kvc.dense_desc(kv)
    st, ref, _, _ = gpu_compress(desc, 4, 64)
    assert st == kvc.KVC_OK
    codec = kvc.Codec(4, 64, 0)
    out, ws, nb = codec.buffers(desc, dev)
    stream = torch.cuda.current_stream(dev)
    sp = kvc._stream_ptr(stream)
    ce = bench.new_events(5, stream)
    assert kvc.kvc_compress_timed(desc, codec.params, out.data_ptr(), out.numel(), nb.data_ptr(),
                                  ws.data_ptr(), ws.numel(), ce, sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    n = int(nb.item())
    assert np.array_equal(out[:n].cpu().numpy(), ref)
    dst = torch.empty(w.layers, 2, w.kv_heads, w.total_tokens, 128, dtype=torch.bfloat16,
                      device=dev)
    odesc = kvc.dense_desc(dst)
    dws = torch.empty(kvc.kvc_decompress_workspace_bytes(odesc), dtype=torch.uint8, device=dev)
    de = bench.new_events(5, stream)
    assert kvc.kvc_decompress_timed(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(), de,
                                    sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK
    ref2 = torch.empty_like(dst)
    dws2 = torch.empty_like(dws)
    assert kvc.kvc_decompress(out.data_ptr(), n, kvc.dense_desc(ref2), dws2.data_ptr(),
                              dws2.numel(), sp) == kvc.KVC_OK
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), ref2.view(torch.int16))
    for ev in (ce, de):
        parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(4)]
        assert all(p >= 0 for p in parts)
        assert abs(sum(parts) - ev[0].elapsed_time(ev[4])) < 1e-3
    # the encode kernel and the decode kernel carry the work
    assert ce[1].elapsed_time(ce[2]) > 0 and de[3].elapsed_time(de[4]) > 0
