"""The unfused two-kernel baseline (transform kernel, fp32 tensor in HBM,
quantize kernel) writes the fused path's stream byte for byte: dense inputs
with and without the tensor-map path, a partial last block, both head
dimensions, a paged pool, and inputs where code chunks shrink."""
import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
from kv_cache_compression_04_b200 import synth
from kvc_testutil import gpu_compress

pytestmark = pytest.mark.gpu


def _unfused(desc, bits, group, seed=0):
    p = kvc.params(bits, group, seed)
    cap = kvc.kvc_max_compressed_bytes(desc, p)
    wsb = kvc.kvc_unfused_workspace_bytes(desc, p)
    assert wsb > kvc.kvc_workspace_bytes(desc, p)
    out = torch.full((cap,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    nb = torch.zeros(1, dtype=torch.int64, device="cuda")
    sp = kvc._stream_ptr(None)
    # one byte too little workspace is refused before anything runs
    assert kvc.kvc_compress_unfused(desc, p, out.data_ptr(), cap, nb.data_ptr(), ws.data_ptr(),
                                    wsb - 1, sp) == kvc.KVC_ERR_CAPACITY
    st = kvc.kvc_compress_unfused(desc, p, out.data_ptr(), cap, nb.data_ptr(), ws.data_ptr(), wsb,
                                  sp)
    assert st == kvc.KVC_OK
    st = kvc.kvc_stream_status(ws.data_ptr(), sp)
    n = int(nb.item())
    return st, out[:n].cpu().numpy()


@pytest.mark.parametrize("d,bits,g,T", [(128, 4, 128, 512), (128, 2, 32, 333), (64, 4, 64, 256),
                                        (64, 2, 32, 100)])
def test_unfused_matches_fused_dense(d, bits, g, T):
    gen = torch.Generator().manual_seed(d + bits + T)
    kv = (torch.randn(2, 2, 3, T, d, generator=gen) *
          torch.exp(1.5 * torch.randn(2, 1, 3, 1, d, generator=gen))).to(torch.bfloat16).cuda()
    desc = kvc.dense_desc(kv)
    st, fused, _, _ = gpu_compress(desc, bits, g)
    ust, unf = _unfused(desc, bits, g)
    assert st == ust == kvc.KVC_OK
    assert np.array_equal(fused, unf)


def test_unfused_matches_fused_with_shrinking_chunks():
    kv = torch.randn(2, 2, 2, 2048, 128, generator=torch.Generator().manual_seed(3))
    kv[:, :, :, :1024] = 0                       # code chunks that use elimination
    desc = kvc.dense_desc(kv.to(torch.bfloat16).cuda())
    st, fused, _, _ = gpu_compress(desc, 4, 128)
    ust, unf = _unfused(desc, 4, 128)
    assert st == ust == kvc.KVC_OK and fused[11] == 1
    assert np.array_equal(fused, unf)


def test_unfused_matches_fused_paged():
    seq = [20, 700, 33, 257]
    w = synth.Workload("p", 2, 3, 128, 4, 64, seed=3, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    desc = kvc.paged_desc(pk.pool, pk.page_table, seq)
    st, fused, _, _ = gpu_compress(desc, 4, 64)
    ust, unf = _unfused(desc, 4, 64)
    assert st == ust == kvc.KVC_OK
    assert np.array_equal(fused, unf)


def test_unfused_reports_nonfinite():
    kv = torch.randn(1, 2, 1, 256, 128, generator=torch.Generator().manual_seed(4))
    kv[0, 1, 0, 17, 3] = float("inf")
    desc = kvc.dense_desc(kv.to(torch.bfloat16).cuda())
    st, _ = _unfused(desc, 4, 128)
    assert st == kvc.KVC_ERR_NONFINITE
