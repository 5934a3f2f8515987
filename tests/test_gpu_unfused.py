"""The unfused two-kernel baseline (transform kernel, fp32 tensor in HBM,
quantize kernel) writes the oracle's stream byte for byte (and so the fused
path's): dense inputs with and without the tensor-map path, a partial last
block, both head dimensions, a paged pool, and inputs where code chunks
shrink."""
import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import first_diff, gpu_compress, oracle_desc, u16

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


def _oracle_dense(kv, bits, g, seed=0):
    L, _, H, T, D = kv.shape
    od = oracle_desc(bits, g, D, L, H, [T], seed)
    st, s = oracle.compress(od, u16(kv.contiguous()).reshape(-1, D))
    assert st == oracle.OK
    return od, s


@pytest.mark.parametrize("d,bits,g,T", [(128, 4, 128, 512), (128, 2, 32, 333), (64, 4, 64, 256),
                                        (64, 2, 32, 100)])
def test_unfused_matches_oracle_dense(d, bits, g, T):
    gen = torch.Generator().manual_seed(d + bits + T)
    kv = (torch.randn(2, 2, 3, T, d, generator=gen) *
          torch.exp(1.5 * torch.randn(2, 1, 3, 1, d, generator=gen))).to(torch.bfloat16).cuda()
    desc = kvc.dense_desc(kv)
    od, ostream = _oracle_dense(kv, bits, g)
    ust, unf = _unfused(desc, bits, g)
    assert ust == kvc.KVC_OK
    assert np.array_equal(unf, ostream), first_diff(unf, ostream, od.layout())
    st, fused, _, _ = gpu_compress(desc, bits, g)
    assert st == kvc.KVC_OK and np.array_equal(fused, unf)


def test_unfused_matches_oracle_with_shrinking_chunks():
    kv = torch.randn(2, 2, 2, 2048, 128, generator=torch.Generator().manual_seed(3))
    kv[:, :, :, :1024] = 0                       # code chunks that use elimination
    kv = kv.to(torch.bfloat16).cuda()
    od, ostream = _oracle_dense(kv, 4, 128)
    ust, unf = _unfused(kvc.dense_desc(kv), 4, 128)
    assert ust == kvc.KVC_OK and unf[11] == 1
    assert np.array_equal(unf, ostream), first_diff(unf, ostream, od.layout())


def test_unfused_matches_oracle_paged():
    seq = [20, 700, 33, 257]
    w = synth.Workload("p", 2, 3, 128, 4, 64, seed=3, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    desc = kvc.paged_desc(pk.pool, pk.page_table, seq)
    x = oracle.gather_paged(u16(pk.pool).reshape(-1), w.layers, w.kv_heads, 128, pk.strides(),
                            16, seq, pk.page_table.cpu().numpy(), 0, w.vectors)
    od = oracle_desc(4, 64, 128, w.layers, w.kv_heads, seq, origin=1)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    ust, unf = _unfused(desc, 4, 64)
    assert ust == kvc.KVC_OK
    assert np.array_equal(unf, ostream), first_diff(unf, ostream, od.layout())


def test_unfused_reports_nonfinite():
    kv = torch.randn(1, 2, 1, 256, 128, generator=torch.Generator().manual_seed(4))
    kv[0, 1, 0, 17, 3] = float("inf")
    desc = kvc.dense_desc(kv.to(torch.bfloat16).cuda())
    st, _ = _unfused(desc, 4, 128)
    assert st == kvc.KVC_ERR_NONFINITE
