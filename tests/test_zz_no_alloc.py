"""kvc_compress_noalloc (workspace in the library's static device block)
against kvc_compress with a caller workspace: identical streams and stream
lengths on two calls in a row, status read back through status_dev, and the
size limit enforced before anything is enqueued. Collected last on purpose:
it must pass alone in a fresh process and after every other test."""
import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
from kv_cache_compression_04_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs():
    w = synth.Workload("n", 2, 4, 128, 4, 64, seed=21, kind="lognormal", tokens=3000)
    dense = synth.dense_kv(w, device="cuda")
    zeros = torch.zeros(2, 2, 2, 2048, 128, dtype=torch.bfloat16, device="cuda")  # compaction
    return [(dense, 4, 64), (zeros, 2, 32)]


def _with_workspace(desc, p, stream):
    cap = kvc.kvc_max_compressed_bytes(desc, p)
    out = torch.zeros(cap, dtype=torch.uint8, device="cuda")
    nb = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws = torch.empty(kvc.kvc_workspace_bytes(desc, p), dtype=torch.uint8, device="cuda")
    st = kvc.kvc_compress(desc, p, out.data_ptr(), cap, nb.data_ptr(), ws.data_ptr(), ws.numel(),
                          stream)
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    assert kvc.kvc_stream_status(ws.data_ptr(), stream) == kvc.KVC_OK
    n = int(nb.item())
    return out[:n].cpu().numpy(), n


def test_noalloc_matches_workspace_entry_point():
    stream = kvc._stream_ptr(torch.cuda.current_stream())
    for kv, bits, group in _inputs():
        desc, p = kvc.dense_desc(kv), kvc.params(bits, group, 7)
        assert kvc.kvc_workspace_bytes(desc, p) <= kvc.KVC_NOALLOC_SCRATCH_BYTES
        ref, n_ref = _with_workspace(desc, p, stream)
        cap = kvc.kvc_max_compressed_bytes(desc, p)
        for call in range(2):  # two calls in a row reuse the same static block
            out = torch.full((cap,), 0xA5, dtype=torch.uint8, device="cuda")
            nb = torch.zeros(1, dtype=torch.int64, device="cuda")
            status = torch.full((1,), 0xFFFFFFF, dtype=torch.int32, device="cuda")
            st = kvc.kvc_compress_noalloc(desc, p, out.data_ptr(), cap, nb.data_ptr(),
                                          status.data_ptr(), stream)
            assert st == kvc.KVC_OK, kvc.STATUS[st]
            assert kvc.kvc_stream_status(status.data_ptr(), stream) == kvc.KVC_OK
            n = int(nb.item())
            assert n == n_ref, (call, n, n_ref)
            got = out[:n].cpu().numpy()
            assert np.array_equal(got, ref), (call, int(np.argmax(got != ref)))


def test_noalloc_rejects_shapes_beyond_the_block():
    stream = kvc._stream_ptr(torch.cuda.current_stream())
    # 32 layers x 8 heads x 4096 tokens at group 64 needs 16.1 MiB of workspace
    kv = torch.empty(32, 2, 8, 4096, 128, dtype=torch.bfloat16, device="cuda")
    desc, p = kvc.dense_desc(kv), kvc.params(4, 64)
    assert kvc.kvc_workspace_bytes(desc, p) > kvc.KVC_NOALLOC_SCRATCH_BYTES
    cap = kvc.kvc_max_compressed_bytes(desc, p)
    out = torch.empty(cap, dtype=torch.uint8, device="cuda")
    st = kvc.kvc_compress_noalloc(desc, p, out.data_ptr(), cap, None, None, stream)
    assert st == kvc.KVC_ERR_CAPACITY
    # the same cache at group 128 fits
    p128 = kvc.params(4, 128)
    assert kvc.kvc_workspace_bytes(desc, p128) <= kvc.KVC_NOALLOC_SCRATCH_BYTES
