"""The quantizer variants on the GPU against the oracle (readings R19-R22:
symmetric absmax, 8-bit codes, per-(layer, kv, head) sign diagonals, FP4
e2m1 codes with dual scales): every
stream byte equal, the oracle's stream decoded on the GPU to the oracle's
bf16 values bit for bit, attention over such streams within the attention
tolerance, for dense and paged inputs, every group size, both lossless
modes, and the full-size Llama-3-8B-shaped cache for each variant."""
import os

import numpy as np
import pytest
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth
from kvc_testutil import first_diff, gpu_compress, gpu_decompress, oracle_desc, u16

pytestmark = pytest.mark.gpu

SYM, FP4, VEC = kvc.KVC_QUANT_SYM, kvc.KVC_QUANT_FP4, kvc.KVC_SIGNS_PER_VECTOR
THREADS = max(1, min(os.cpu_count() or 1, 64))


def _dense(d, bits, g, L, H, T, quant=0, signs=0, lossless=0, seed=5, kind="lognormal", kv=None):
    if kv is None:
        w = synth.Workload("v", L, H, d, bits, g, seed=L * 31 + T, kind=kind, scale_sigma=1.5,
                           tokens=T)
        kv = synth.dense_kv(w).cuda()
    x = u16(kv).reshape(-1, d)
    od = oracle_desc(bits, g, d, L, H, [T], seed, 0, lossless, quant, signs)
    ost, ostream = oracle.compress(od, x, threads=THREADS)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.dense_desc(kv), bits, g, seed, lossless=lossless,
                                     quant=quant, signs=signs)
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    out = torch.zeros_like(kv)
    assert gpu_decompress(ostream, kvc.dense_desc(out)) == kvc.KVC_OK
    _, ox = oracle.decompress(ostream, od, threads=THREADS)
    got = u16(out).reshape(-1, d)
    assert np.array_equal(got, ox), f"{np.count_nonzero(got != ox)} decoded values differ"
    return ostream


@pytest.mark.parametrize("d,bits,g,L,H,T", [
    (128, 2, 32, 2, 3, 1000), (128, 4, 64, 2, 3, 777), (128, 4, 128, 1, 4, 1111),
    (128, 8, 32, 2, 2, 900), (128, 8, 64, 1, 3, 1500), (128, 8, 128, 2, 2, 2100),
    (64, 4, 32, 2, 3, 999), (64, 8, 64, 2, 2, 1300), (64, 2, 64, 1, 3, 1777)])
def test_symmetric_dense(d, bits, g, L, H, T):
    s = _dense(d, bits, g, L, H, T, quant=SYM)
    assert s[11] & 6 == 2


@pytest.mark.parametrize("d,g,L,H,T,signs", [
    (128, 32, 2, 3, 1000, 0), (128, 64, 2, 2, 777, VEC), (128, 128, 1, 4, 1111, 0),
    (64, 32, 2, 3, 999, VEC), (64, 64, 2, 2, 1300, 0)])
def test_fp4_dense(d, g, L, H, T, signs):
    s = _dense(d, 4, g, L, H, T, quant=FP4, signs=signs, kind="outlier_t")
    assert s[11] & 6 == 4


@pytest.mark.parametrize("d,bits,g,L,H,T", [
    (128, 8, 32, 2, 3, 1000), (128, 8, 64, 2, 2, 2049), (128, 8, 128, 1, 4, 4200),
    (64, 8, 32, 3, 2, 999), (64, 8, 64, 2, 2, 2500)])
def test_eight_bit_dense(d, bits, g, L, H, T):
    _dense(d, bits, g, L, H, T)


@pytest.mark.parametrize("d,bits,g,L,H,T", [
    (128, 4, 128, 2, 3, 1000), (128, 2, 32, 2, 2, 777), (128, 8, 64, 1, 3, 640),
    (64, 4, 64, 3, 2, 555), (128, 4, 32, 2, 2, 17)])
def test_per_vector_signs_dense(d, bits, g, L, H, T):
    s = _dense(d, bits, g, L, H, T, signs=VEC)
    assert s[11] & 8


def test_variants_combined_search_mode():
    """Symmetric 2-bit codes with per-vector signs and the lossless search
    (meta chunks through the XOR pipelines) on heavy-tailed input."""
    _dense(128, 2, 32, 2, 4, 3000, quant=SYM, signs=VEC, lossless=kvc.KVC_LOSSLESS_SEARCH,
           kind="outlier_t")
    _dense(128, 8, 32, 2, 2, 2100, quant=SYM, lossless=kvc.KVC_LOSSLESS_SEARCH)


@pytest.mark.parametrize("bits,g,quant,signs", [(4, 64, SYM, VEC), (8, 32, 0, VEC),
                                                (8, 128, SYM, 0), (4, 32, FP4, VEC)])
def test_variants_paged(bits, g, quant, signs):
    seq = [20, 0, 33, 700, 16, 257]
    w = synth.Workload("p", 2, 3, 128, bits, g, seed=3, kind="lognormal", scale_sigma=1.5,
                       seq_lens=seq)
    pk = synth.paged_kv(w, device="cuda")
    x = oracle.gather_paged(u16(pk.pool).reshape(-1), 2, 3, 128, pk.strides(), 16, seq,
                            pk.page_table.cpu().numpy(), 0, w.vectors)
    od = oracle_desc(bits, g, 128, 2, 3, seq, 0, 1, 0, quant, signs)
    ost, ostream = oracle.compress(od, x)
    assert ost == oracle.OK
    st, gstream, _, _ = gpu_compress(kvc.paged_desc(pk.pool, pk.page_table, seq), bits, g,
                                     quant=quant, signs=signs)
    assert st == kvc.KVC_OK
    assert np.array_equal(gstream, ostream), first_diff(gstream, ostream, od.layout())
    pool2 = torch.full_like(pk.pool, 1.5)
    assert gpu_decompress(ostream, kvc.paged_desc(pool2, pk.page_table, seq)) == kvc.KVC_OK
    got = oracle.gather_paged(u16(pool2).reshape(-1), 2, 3, 128, pk.strides(), 16, seq,
                              pk.page_table.cpu().numpy(), 0, w.vectors)
    _, ox = oracle.decompress(ostream, od)
    assert np.array_equal(got, ox)


def test_unfused_variants():
    """The unfused baseline writes the fused path's stream for the symmetric
    quantizer and 8-bit codes, and refuses per-vector diagonals."""
    w = synth.Workload("u", 2, 2, 128, 8, 64, seed=4, kind="lognormal", tokens=700)
    kv = synth.dense_kv(w).cuda()
    desc = kvc.dense_desc(kv)
    for bits, g, quant in [(8, 64, 0), (4, 32, SYM), (8, 128, SYM)]:  # FP4: refused below
        p = kvc.params(bits, g, 3, 0, quant)
        cap = kvc.kvc_max_compressed_bytes(desc, p)
        outs = []
        for unfused in (False, True):
            wsb = (kvc.kvc_unfused_workspace_bytes if unfused else kvc.kvc_workspace_bytes)(desc, p)
            ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
            out = torch.zeros(cap, dtype=torch.uint8, device="cuda")
            nb = torch.zeros(1, dtype=torch.int64, device="cuda")
            fn = kvc.kvc_compress_unfused if unfused else kvc.kvc_compress
            assert fn(desc, p, out.data_ptr(), cap, nb.data_ptr(), ws.data_ptr(), wsb,
                      kvc._stream_ptr(None)) == kvc.KVC_OK
            assert kvc.kvc_stream_status(ws.data_ptr(), kvc._stream_ptr(None)) == kvc.KVC_OK
            outs.append(out[:int(nb.item())].cpu().numpy())
        assert np.array_equal(outs[0], outs[1]), (bits, g, quant)
    p = kvc.params(4, 64, 3, 0, 0, VEC)
    wsb = kvc.kvc_unfused_workspace_bytes(desc, p)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.zeros(kvc.kvc_max_compressed_bytes(desc, p), dtype=torch.uint8, device="cuda")
    assert kvc.kvc_compress_unfused(desc, p, out.data_ptr(), out.numel(), None, ws.data_ptr(),
                                    wsb, kvc._stream_ptr(None)) == kvc.KVC_ERR_UNSUPPORTED
    p = kvc.params(4, 64, 3, 0, FP4)
    assert kvc.kvc_compress_unfused(desc, p, out.data_ptr(), out.numel(), None, ws.data_ptr(),
                                    wsb, kvc._stream_ptr(None)) == kvc.KVC_ERR_UNSUPPORTED


@pytest.mark.parametrize("bits,g,quant,signs", [(4, 128, SYM, VEC), (4, 64, FP4, VEC),
                                                (8, 32, 0, VEC), (4, 32, FP4, 0)])
def test_variants_with_eliminated_code_chunks(bits, g, quant, signs):
    """Half of the 256-token blocks all zero: code chunks stored eliminated
    (header flag bit 0 next to the variant's bits), compacted by the encoder
    and expanded by the eliminated-chunk decoder."""
    L, H, T, D = 2, 8, 4096, 128
    gen = torch.Generator().manual_seed(21)
    x = torch.randn(L, 2, H, T, D, generator=gen)
    blocks = x.view(L, 2, H, T // 256, 256, D)
    blocks[torch.rand(L, 2, H, T // 256, generator=gen) < 0.5] = 0
    s = _dense(D, bits, g, L, H, T, quant=quant, signs=signs, kv=x.to(torch.bfloat16).cuda())
    assert s[11] & 1, "some code chunk stored eliminated"


@pytest.mark.parametrize("bits,g,quant,signs,qpk", [(4, 128, SYM, 0, 4), (2, 32, 0, VEC, 7),
                                                    (8, 64, SYM, VEC, 2), (8, 32, 0, 0, 8),
                                                    (4, 64, FP4, VEC, 4), (4, 32, FP4, 0, 1)])
def test_attend_over_variant_streams(bits, g, quant, signs, qpk):
    L, H, T, d = 2, 2, 900, 128
    w = synth.Workload("a", L, H, d, bits, g, seed=12, kind="lognormal", scale_sigma=1.5,
                       tokens=T)
    kv = synth.dense_kv(w).cuda()
    st, s, gbuf, n = gpu_compress(kvc.dense_desc(kv), bits, g, 9, quant=quant, signs=signs)
    assert st == kvc.KVC_OK and s[11] & 1 == 0
    q = torch.randn(L, 1, H * qpk, d, generator=torch.Generator(device="cuda").manual_seed(1),
                    device="cuda").to(torch.bfloat16)
    out = torch.full((L, 1, H * qpk, d), float("nan"), device="cuda")
    ad = kvc.attn_desc(L, H, qpk, bits, g, [T], q, out, d ** -0.5, quant=quant)
    ws = torch.empty(kvc.kvc_attend_workspace_bytes(ad), dtype=torch.uint8, device="cuda")
    sp = kvc._stream_ptr(None)
    assert kvc.kvc_attend(gbuf.data_ptr(), n, ad, ws.data_ptr(), ws.numel(), sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    od = oracle_desc(bits, g, d, L, H, [T], 9, 0, 0, quant, signs)
    ost, ref = oracle.attend(s, od, u16(q.cpu()), qpk, d ** -0.5, threads=THREADS)
    assert ost == oracle.OK
    _, vals = oracle.decode_values(s, od, threads=THREADS)
    V = vals.reshape(L, 2, H, T, d)[:, 1]
    got = out.cpu().numpy().astype(np.float64)
    for h in range(H):
        vmax = np.abs(V[:, h]).max()
        sl = slice(h * qpk, (h + 1) * qpk)
        err = np.abs(got[:, 0, sl] - ref[:, 0, sl]).max()
        assert err <= 2e-4 * vmax + 1e-6, (h, err, vmax)


@pytest.mark.parametrize("bits,g,quant,signs", [(4, 128, SYM, 0), (4, 128, 0, VEC),
                                                (8, 128, 0, 0), (4, 128, FP4, 0)])
def test_full_llama8b_variant(bits, g, quant, signs):
    """The Llama-3-8B-shaped cache (32 x 2 x 8 x 4096 x 128) in each variant,
    compared whole: stream bytes and decoded values."""
    w = synth.workload("llama8b")
    _dense(128, bits, g, w.layers, w.kv_heads, w.tokens, quant=quant, signs=signs)


def test_device_e2m1_rounding_is_the_oracles_rule():
    """The FP4 encoder's e2m1 rounding (the sm_100a conversion it uses) against
    the oracle's rule: every multiple of 1/256 in [-8, 8] (every tie of the
    e2m1 grid included: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5), the fp32
    neighbours of each tie, signed zeros, values far above 6, tiny and
    subnormal values, and random values over several binades."""
    grid = np.arange(-8 * 256, 8 * 256 + 1, dtype=np.float64) / 256
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])
    ties = np.concatenate([ties, -ties])
    t32 = ties.astype(np.float32)
    near = np.concatenate([np.nextafter(t32, np.float32(np.inf)),
                           np.nextafter(t32, np.float32(-np.inf))])
    rng = np.random.default_rng(5)
    rnd = (rng.standard_normal(20000) * np.exp2(rng.integers(-12, 6, 20000))).astype(np.float32)
    special = np.array([0.0, -0.0, 7.0, -7.0, 1e30, -1e30, 1e-40, -1e-40, 6.25, -6.25],
                       np.float32)
    x = np.concatenate([grid.astype(np.float32), t32, near, rnd, special]).astype(np.float32)
    din = torch.from_numpy(x).cuda()
    dout = torch.zeros(x.size, dtype=torch.uint8, device="cuda")
    assert kvc.lib().kvc_test_e2m1(din.data_ptr(), dout.data_ptr(), x.size,
                                   kvc._stream_ptr(None)) == kvc.KVC_OK
    got = dout.cpu().numpy()
    want = np.array([oracle.f32_to_e2m1_rne(float(v)) for v in x], np.uint8)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:10]]


@pytest.mark.parametrize("q", [1, 3, 7, 15, 127, 255])
def test_device_division_by_quantizer_constant(q):
    """The encoder's division by its quantizer's constant, on the GPU, against
    numpy's correctly rounded fp32 division: 2048 random significands in
    every binade (subnormals included), each binade's first and last value,
    and zero."""
    rng = np.random.default_rng(q)
    exps = np.repeat(np.arange(0, 255, dtype=np.uint32), 2048)
    sig = rng.integers(0, 1 << 23, exps.size, dtype=np.uint32)
    bits = np.concatenate([(exps << 23) | sig, (np.arange(0, 255, dtype=np.uint32) << 23),
                           (np.arange(0, 255, dtype=np.uint32) << 23) | 0x7FFFFF,
                           np.array([0], np.uint32)])
    x = bits.view(np.float32)
    din = torch.from_numpy(x.copy()).cuda()
    dout = torch.zeros_like(din)
    assert kvc.lib().kvc_test_div_const(din.data_ptr(), dout.data_ptr(), x.size, q,
                                        kvc._stream_ptr(None)) == kvc.KVC_OK
    got = dout.cpu().numpy()
    want = x / np.float32(q)
    bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
    assert bad.size == 0, [(float(x[i]), float(got[i]), float(want[i])) for i in bad[:10]]


def test_device_reciprocal_of_every_scale():
    """The encoder's 1 / s for every scale it can hold (each positive finite
    fp16 value times 2^3 and 2^4) against numpy's correctly rounded fp32
    division."""
    h = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    s = np.concatenate([h * np.float32(8), h * np.float32(16)]).astype(np.float32)
    din = torch.from_numpy(s.copy()).cuda()
    dout = torch.zeros_like(din)
    assert kvc.lib().kvc_test_rcp_scale(din.data_ptr(), dout.data_ptr(), s.size,
                                        kvc._stream_ptr(None)) == kvc.KVC_OK
    got = dout.cpu().numpy()
    want = np.float32(1) / s
    bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
    assert bad.size == 0, [(float(s[i]), float(got[i]), float(want[i])) for i in bad[:10]]
