"""The layer-pipelined transfer (one compress / decompress call pair per
layer on three CUDA streams with a simulated link between them, the
benchmark's --pipeline measurement) delivers the oracle's decode of the whole
cache into the receiver, bit for bit: chunking the cache by layer changes no
decoded value, and the per-layer streams equal the oracle's per-layer
streams."""
import numpy as np
import pytest
import torch

import bench
import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import first_diff, oracle_desc, u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,g", [(4, 128), (2, 32)])
def test_layer_pipeline_receiver_equals_oracle(bits, g):
    w = synth.Workload("pipe", 6, 4, 128, bits, g, seed=17, kind="lognormal",
                       scale_sigma=1.5, tokens=1000)
    dev = torch.device("cuda", 0)
    kv = synth.dense_kv(w, device=dev)
    rx = torch.full_like(kv, 1.5)
    codec = kvc.Codec(bits, g, 0)
    pipe = bench.LayerPipeline(kv, rx, codec, dev)
    ms = pipe.transfer(400e9 / 8, 1.965e9)
    assert ms > 0 and pipe.statuses_ok()
    x = u16(kv).reshape(w.layers, -1, 128)
    od = oracle_desc(bits, g, 128, w.layers, w.kv_heads, [w.tokens])
    ost, ostream = oracle.compress(od, x.reshape(-1, 128))
    assert ost == oracle.OK
    _, ox = oracle.decompress(ostream, od)
    assert np.array_equal(u16(rx).reshape(-1, 128), ox)
    # each layer's stream is the oracle's stream of that layer alone
    od1 = oracle_desc(bits, g, 128, 1, w.kv_heads, [w.tokens])
    for l in range(w.layers):
        out, _, nb = pipe.bufs[l]
        got = out[:pipe.n[l]].cpu().numpy()
        st, want = oracle.compress(od1, x[l])
        assert st == oracle.OK
        assert np.array_equal(got, want), (l, first_diff(got, want, od1.layout()))
