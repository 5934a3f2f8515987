"""Pins of the quantizer variants and the per-vector sign diagonals (the
FP4Quant abstract's variants of the transform + quantize step), checked
against things other than the oracle itself:

  R19 symmetric absmax: hand-derived scalar cases (ties to even, clamps),
      and per group the properties that define it: the scale is the
      smallest fp16 grid value covering max|y| / (2^(b-1) - 1), the stored
      zero is exactly -2^(b-1) times it, every code is a nearest grid point,
      and a stream decodes to exactly (code - 2^(b-1)) * scale;
  R20 per-(layer, kv, head) sign diagonals: the published SplitMix64
      outputs (golden file) continued across vector indices, and a stream's
      decoded vectors inverted through the Sylvester matrix with the
      diagonal of their own index;
  R21 8-bit codes: identity packing, nearest-grid-point codes, the layout
      arithmetic, and a stream's decode on the grid."""
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_04_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [int(l.split("#")[0].strip(), 16) for l in f if l.split("#")[0].strip()]


def sylvester(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def f16(h):
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float64)


def bf16(x):
    return synth.bf16_bits(torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16))


def signs_of(words, d):
    return np.array([-1.0 if (int(words[c // 64]) >> (c % 64)) & 1 else 1.0 for c in range(d)])


def transformed(x_bits, seed=0, index=None):
    """The encoder's fp32 transformed vector y = fwht(D x) (the butterfly is
    pinned on its own against the Sylvester matrix)."""
    d = x_bits.shape[-1]
    w = oracle.sign_words(seed, d) if index is None else oracle.sign_words_at(seed, d, index)
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float32)
    return oracle.fwht((x * signs_of(w, d)).astype(np.float32)).astype(np.float64)


def meta_fields(meta_row, d, g):
    m = meta_row.reshape(d // g, 4).astype(np.uint16)
    sh, zh = m[:, 0] | (m[:, 1] << 8), m[:, 2] | (m[:, 3] << 8)
    up = 2.0 ** oracle.meta_shift(d)
    return sh, zh, f16(sh) * up, f16(zh) * up


def codes_of(codes_row, d, bits):
    b = np.unpackbits(codes_row[:, None], axis=1, bitorder="little").reshape(-1)
    return b.reshape(d, bits) @ (1 << np.arange(bits))


# --------------------------------------------------------------- R20 --
def test_sign_words_at_continue_the_published_generator():
    want = _golden("splitmix64_seed0.txt")            # outputs 0..4 from state 0
    for i in range(5):
        assert int(oracle.sign_words_at(0, 64, i)[0]) == want[i]
    for i in range(2):
        assert [int(w) for w in oracle.sign_words_at(0, 128, i)] == want[2 * i:2 * i + 2]
    assert int(oracle.sign_words_at(0, 128, 2)[0]) == want[4]
    for seed in (0, 7, 2 ** 63 + 5):               # index 0 is the global diagonal
        assert (oracle.sign_words_at(seed, 128, 0) == oracle.sign_words(seed, 128)).all()
    # seed s, index i: SplitMix64 from state s + 2*i*gamma (d = 128, two words)
    g = 0x9E3779B97F4A7C15
    assert [int(w) for w in oracle.sign_words_at(5, 128, 3)] == oracle.splitmix64(
        (5 + 6 * g) % 2 ** 64, 2)


def _raw_stream(bits, g, L, H, lens, quant=oracle.QUANT_ASYM, signs=oracle.SIGNS_GLOBAL,
                seed=11, d=128, kind="lognormal"):
    w = synth.Workload("v", L, H, d, bits, g, seed=3, kind=kind, scale_sigma=1.5,
                       tokens=sum(lens))
    x = synth.bf16_bits(synth.dense_kv(w)).reshape(-1, d)
    desc = oracle.StreamDesc(bits, g, d, L, H, lens, seed, 0, oracle.LOSSLESS_NONE, quant, signs)
    st, s = oracle.compress(desc, x)
    assert st == oracle.OK
    lay = desc.layout()
    e = s[64:64 + 8 * lay.n_chunks].view("<u8")
    off = (((e >> 16) & 0xFFFFFFFFFFF) * 16).astype(np.int64) + lay.data_base
    size = (e & 0xFFFF).astype(np.int64)
    codes = np.concatenate([s[off[i]:off[i] + size[i]] for i in range(lay.n_code)])
    meta = np.concatenate([s[off[i]:off[i] + size[i]] for i in range(lay.n_code, lay.n_chunks)])
    return desc, s, x, codes.reshape(lay.V, -1), meta.reshape(lay.V, -1)


def _grid_values(codes, meta, d, bits, g):
    """zf + q*sf per channel from a stream's codes and meta (float64; the
    fp32 product and sum are exact here, see the decoder's reading R9)."""
    V = codes.shape[0]
    out = np.empty((V, d))
    for v in range(V):
        q = codes_of(codes[v], d, bits)
        _, _, sf, zf = meta_fields(meta[v], d, g)
        out[v] = np.repeat(zf, g) + q * np.repeat(sf, g)
    return out


@pytest.mark.parametrize("d", [64, 128])
def test_per_vector_signs_decode_through_each_vectors_own_diagonal(d):
    L, H, lens, seed = 2, 3, [40], 11
    desc, s, x, codes, meta = _raw_stream(4, 32, L, H, lens, signs=oracle.SIGNS_PER_VECTOR,
                                          seed=seed, d=d)
    assert s[11] == 8                               # flags: bit 3
    st, xh = oracle.decode_values(s, desc)
    assert st == oracle.OK
    grid = _grid_values(codes, meta, d, 4, 32)
    Hm = sylvester(d)
    T = sum(lens)
    for v in range(codes.shape[0]):
        D = signs_of(oracle.sign_words_at(seed, d, v // T), d)
        np.testing.assert_allclose(Hm @ (D * xh[v]), grid[v], rtol=0, atol=1e-9 * abs(grid[v]).max())
    # the global diagonal does not explain the vectors of index > 0
    D0 = signs_of(oracle.sign_words(seed, d), d)
    assert not np.allclose(Hm @ (D0 * xh[T]), grid[T], atol=1e-6)
    # a receiver expecting the global diagonal refuses the stream
    bad = oracle.StreamDesc(4, 32, d, L, H, lens, seed, 0, oracle.LOSSLESS_NONE)
    assert oracle.decompress(s, bad)[0] == oracle.CORRUPT
    # the codes differ from the global-diagonal stream's (same input)
    _, _, _, codes_g, _ = _raw_stream(4, 32, L, H, lens, seed=seed, d=d)
    assert (codes_g[:T] == codes[:T]).all() and not (codes_g[T:] == codes[T:]).all()


# --------------------------------------------------------------- R19 --
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_symmetric_scalar_hand_cases(bits):
    h = 1 << (bits - 1)
    qh = h - 1
    q = oracle.quantize_scalar_sym
    assert q(0.0, 1.0, bits) == h
    assert q(-0.0, 1.0, bits) == h
    assert q(0.5, 1.0, bits) == h                   # tie -> even (0)
    assert q(-0.5, 1.0, bits) == h
    assert q(0.75, 1.0, bits) == h + 1
    assert q(-0.75, 1.0, bits) == h - 1
    assert q(1e9, 1.0, bits) == h + qh              # clamps
    assert q(-1e9, 1.0, bits) == h - qh
    assert q(3.0, 0.0, bits) == h                   # zero scale: r = 0
    if bits >= 4:
        assert q(1.5, 1.0, bits) == h + 2           # tie -> even (2)
        assert q(2.5, 1.0, bits) == h + 2
        assert q(-2.5, 1.0, bits) == h - 2
        # one fp32 rounding of the product: 0.1f * 25.0f = 2.5 exactly in
        # fp32 (2.50000004 before rounding), then the tie goes to 2
        assert q(np.float32(0.1), np.float32(25.0), bits) == h + 2


@pytest.mark.parametrize("bits,g", [(2, 32), (4, 64), (4, 128), (8, 32), (8, 128)])
def test_symmetric_groups_are_absmax_grids(bits, g):
    d, qh, h = 128, (1 << (bits - 1)) - 1, 1 << (bits - 1)
    rng = np.random.default_rng(bits * 100 + g)
    x = rng.standard_normal((60, d)).astype(np.float32) * np.exp(rng.standard_normal((60, 1)))
    x[3] = 0.0                                      # an all-zero vector
    x[5, :] = x[5, 0]                                # constant input
    xb = bf16(x)
    st, codes, meta = oracle.quantize_vectors(xb, bits, g, 9, quant=oracle.QUANT_SYM)
    assert st == oracle.OK
    up = 2.0 ** oracle.meta_shift(d)
    for v in range(x.shape[0]):
        y = transformed(xb[v], 9)
        q = codes_of(codes[v], d, bits)
        sh, zh, sf, zf = meta_fields(meta[v], d, g)
        assert q.min() >= 1 and q.max() <= 2 * qh + 1
        for j in range(d // g):
            yg, qg = y[j * g:(j + 1) * g], q[j * g:(j + 1) * g] - h
            a = np.abs(yg).max()
            target = float(np.float32(np.float32(a) / np.float32(qh)))
            # the smallest fp16 grid value (x 2^k) at or above fl(a / qh)
            assert sf[j] >= target
            if sh[j] & 0x7FFF:
                below = f16(np.uint16(sh[j] - 1)) * up
                assert below < target
                assert zf[j] == -h * sf[j]
            else:
                assert a == 0 and zh[j] == 0 and (qg == 0).all()
                continue
            # every code a nearest grid point (ties either way)
            err = np.abs(yg - qg * sf[j])
            alt = np.abs(yg[:, None] - np.arange(-qh, qh + 1)[None, :] * sf[j]).min(axis=1)
            assert (err <= alt + 1e-6 * sf[j]).all()
            assert (err <= 0.5 * sf[j] * (1 + 1e-6)).all()


def test_symmetric_two_bit_is_ternary():
    rng = np.random.default_rng(2)
    xb = bf16(rng.standard_normal((30, 128)).astype(np.float32))
    st, codes, _ = oracle.quantize_vectors(xb, 2, 32, 0, quant=oracle.QUANT_SYM)
    assert st == oracle.OK
    q = np.concatenate([codes_of(c, 128, 2) for c in codes])
    assert set(np.unique(q)) <= {1, 2, 3} and {1, 3} <= set(np.unique(q))


@pytest.mark.parametrize("bits,g", [(4, 32), (8, 128), (2, 64)])
def test_symmetric_stream_decodes_to_the_grid(bits, g):
    desc, s, x, codes, meta = _raw_stream(bits, g, 2, 2, [50], quant=oracle.QUANT_SYM,
                                          kind="outlier_t")
    assert s[11] == 2                               # flags: quantizer 1
    st, xh = oracle.decode_values(s, desc)
    assert st == oracle.OK
    Hm, d, h = sylvester(128), 128, 1 << (bits - 1)
    D = signs_of(oracle.sign_words(11, d), d)
    for v in range(codes.shape[0]):
        q = codes_of(codes[v], d, bits) - h
        _, _, sf, _ = meta_fields(meta[v], d, g)
        want = q * np.repeat(sf, g)
        np.testing.assert_allclose(Hm @ (D * xh[v]), want, rtol=0,
                                   atol=1e-9 * max(abs(want).max(), 1e-30))
    asym = oracle.StreamDesc(bits, g, 128, 2, 2, [50], 11, 0, oracle.LOSSLESS_NONE)
    assert oracle.decompress(s, asym)[0] == oracle.CORRUPT


def test_symmetric_range_error():
    """The stored zero is -2^(b-1) x the scale, so it leaves the fp16 range
    (RANGE, reading R8) once 2^(b-1) * s_h > 65504: with y = +-479232 in
    every channel (one bf16 input channel), 4-bit needs s_h = RU16(479232 /
    7 / 8) = 8560 (zero -68480: RANGE), 8-bit s_h = 471.75 (zero -60384:
    fine); the asymmetric rule keeps both in range."""
    d = 128
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 479232.0                               # exact in bf16
    sym = oracle.QUANT_SYM
    assert oracle.quantize_vectors(bf16(x), 4, 128, 0, quant=sym)[0] == oracle.RANGE
    st, _, meta = oracle.quantize_vectors(bf16(x), 8, 128, 0, quant=sym)
    assert st == oracle.OK
    sh, zh, sf, zf = meta_fields(meta[0], d, 128)
    assert f16(sh)[0] == 471.75 and f16(zh)[0] == -60384.0
    assert oracle.quantize_vectors(bf16(x), 4, 128, 0)[0] == oracle.OK


# --------------------------------------------------------------- R21 --
def test_eight_bit_packing_and_layout():
    q = np.arange(128, dtype=np.uint8) * 2
    assert (oracle.pack_codes(q, 8) == q).all()
    lay = oracle.StreamDesc(8, 32, 128, 2, 2, [100]).layout()
    assert lay.code_bytes == 128 and lay.vec_per_code == 128 and lay.code_per_seg == 8
    lay = oracle.StreamDesc(8, 64, 64, 2, 2, [100]).layout()
    assert lay.code_bytes == 64 and lay.vec_per_code == 256 and lay.code_per_seg == 16
    for bad in (3, 6, 16):
        with pytest.raises(ValueError):
            oracle.StreamDesc(bad, 32, 128, 1, 1, [10]).layout()
    with pytest.raises(ValueError):
        oracle.StreamDesc(4, 32, 128, 1, 1, [10], quant=3).layout()
    with pytest.raises(ValueError):
        oracle.StreamDesc(4, 32, 128, 1, 1, [10], signs=2).layout()


@pytest.mark.parametrize("g", [32, 128])
def test_eight_bit_codes_are_nearest_grid_points(g):
    d = 128
    rng = np.random.default_rng(g)
    xb = bf16(rng.standard_normal((40, d)).astype(np.float32) * 3)
    st, codes, meta = oracle.quantize_vectors(xb, 8, g, 4)
    assert st == oracle.OK
    for v in range(xb.shape[0]):
        y = transformed(xb[v], 4)
        q = codes_of(codes[v], d, 8)
        _, _, sf, zf = meta_fields(meta[v], d, g)
        for j in range(d // g):
            yg, qg = y[j * g:(j + 1) * g], q[j * g:(j + 1) * g]
            assert zf[j] <= yg.min() and zf[j] + 255 * sf[j] >= yg.max()
            err = np.abs(yg - (zf[j] + qg * sf[j]))
            alt = np.abs(yg[:, None] - (zf[j] + np.arange(256)[None, :] * sf[j])).min(axis=1)
            assert (err <= alt + 1e-6 * sf[j]).all()


def test_eight_bit_stream_roundtrip_error_bound():
    desc, s, x, codes, meta = _raw_stream(8, 64, 2, 2, [70])
    st, xh = oracle.decode_values(s, desc)
    assert st == oracle.OK
    grid = _grid_values(codes, meta, 128, 8, 64)
    Hm = sylvester(128)
    D = signs_of(oracle.sign_words(11, 128), 128)
    for v in range(codes.shape[0]):
        np.testing.assert_allclose(Hm @ (D * xh[v]), grid[v], rtol=0,
                                   atol=1e-9 * abs(grid[v]).max())
        y = transformed(x[v], 11)
        _, _, sf, _ = meta_fields(meta[v], 128, 64)
        assert (np.abs(y - grid[v]) <= 0.5 * np.repeat(sf, 64) * (1 + 1e-6)).all()
    st, xb = oracle.decompress(s, desc)
    assert st == oracle.OK
    # bf16 decode: the unrounded decode rounded to nearest even
    back = synth.bf16_bits(torch.from_numpy(xh).to(torch.bfloat16))
    assert (back == xb).mean() > 0.999


def test_eight_bit_group_128_full_segment():
    """8-bit codes with group 128: a meta chunk covers 32 code chunks (the
    largest segment); 8400 vectors (1 layer x 2 x 2 heads x 2100 tokens)
    fill two segments and start a third. Round trip on the grid, in one and
    in several threads."""
    d, g = 128, 128
    desc, s, x, codes, meta = _raw_stream(8, g, 1, 2, [2100])
    lay = desc.layout()
    assert lay.code_per_seg == 32 and lay.n_code == 66 and lay.n_seg == 3
    st, xh = oracle.decode_values(s, desc)
    assert st == oracle.OK
    grid = _grid_values(codes, meta, d, 8, g)
    Hm = sylvester(d)
    D = signs_of(oracle.sign_words(11, d), d)
    for v in (0, 1, 4095, 4096, 8191, 8192, 8399):
        np.testing.assert_allclose(Hm @ (D * xh[v]), grid[v], rtol=0,
                                   atol=1e-9 * abs(grid[v]).max())
    st2, s2 = oracle.compress(desc, x, threads=3)
    assert st2 == oracle.OK and np.array_equal(s, s2)
    assert (oracle.decompress(s, desc, threads=3)[1] == oracle.decompress(s, desc)[1]).all()


# --------------------------------------------------------------- R22 --
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP e2m1 magnitudes (exponent bias 1)


def test_e2m1_table_and_nearest_even():
    assert [oracle.e2m1_to_f32(c) for c in range(8)] == E2M1
    assert [oracle.e2m1_to_f32(c | 8) for c in range(1, 8)] == [-v for v in E2M1[1:]]
    # every p on a fine grid (all midpoints included), against a scan written
    # here: nearest magnitude, ties to the even index, zero is code 0
    grid = np.concatenate([np.arange(-8, 8.0001, 1 / 64), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5,
                                                           5.0, -0.25, -5.0, 1e9, -1e9]])
    for p in grid.astype(np.float32):
        a = abs(float(p))
        d = [abs(a - v) for v in E2M1]
        best = min(d)
        i = min(j for j in range(8) if d[j] == best and (j % 2 == 0 or d.count(best) == 1))
        want = i | (8 if (i and p < 0) else 0)
        assert oracle.f32_to_e2m1_rne(p) == want, p
    assert oracle.f32_to_e2m1_rne(0.25) == 0 and oracle.f32_to_e2m1_rne(0.75) == 2
    assert oracle.f32_to_e2m1_rne(1.25) == 2 and oracle.f32_to_e2m1_rne(1.75) == 4
    assert oracle.f32_to_e2m1_rne(2.5) == 4 and oracle.f32_to_e2m1_rne(3.5) == 6
    assert oracle.f32_to_e2m1_rne(5.0) == 6 and oracle.f32_to_e2m1_rne(-0.1) == 0
    # magnitudes above 6 give 6 however large (a double scan alone would see
    # 1e30 - 4 and 1e30 - 6 as equal)
    for big in (6.0, 7.0, 1e9, 1e30, 3.4e38):
        assert oracle.f32_to_e2m1_rne(big) == 7 and oracle.f32_to_e2m1_rne(-big) == 15


def test_e4m3_against_torch_and_round_up():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    for b in range(256):
        got = oracle.e4m3_to_f32(b)
        assert (np.isnan(got) and np.isnan(ref[b])) or got == ref[b], b
    finite = sorted(set(float(v) for v in ref[:0x7F]))      # non-negative finite values
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(0, 450, 2000), np.exp(rng.uniform(-12, 6, 2000)), finite,
                         np.nextafter(np.array(finite, np.float32), np.float32(1e9))])
    for x in xs.astype(np.float32):
        b = oracle.f32_to_e4m3_ru(x)
        above = [v for v in finite if v >= float(x)]
        want = above[0] if above else 448.0
        assert oracle.e4m3_to_f32(b) == want, x


@pytest.mark.parametrize("g", [32, 64, 128])
def test_fp4_groups_are_dual_scale_e2m1_grids(g):
    d = 128
    rng = np.random.default_rng(g + 7)
    x = rng.standard_normal((50, d)).astype(np.float32) * np.exp(rng.standard_normal((50, 1)) * 2)
    x[4] = 0.0
    x[6, :8] *= 100.0                                   # one dominant half-group
    xb = bf16(x)
    st, codes, meta = oracle.quantize_vectors(xb, 4, g, 2, quant=oracle.QUANT_FP4)
    assert st == oracle.OK
    up = 2.0 ** oracle.meta_shift(d)
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for v in range(x.shape[0]):
        y = transformed(xb[v], 2)
        q = codes_of(codes[v], d, 4)
        m = meta[v].reshape(d // g, 4)
        for j in range(d // g):
            yg = y[j * g:(j + 1) * g]
            s2h = int(m[j, 0]) | (int(m[j, 1]) << 8)
            s2 = f16(s2h) * up
            a = np.abs(yg).max()
            target = float(np.float32(np.float32(a) / np.float32(2688.0)))
            assert s2 >= target and (s2h == 0 or f16(np.uint16(s2h - 1)) * up < target)
            for h in range(2):
                yh = yg[h * g // 2:(h + 1) * g // 2]
                qh = q[j * g + h * g // 2: j * g + (h + 1) * g // 2]
                s1 = e4[m[j, 2 + h]]
                assert 0 <= s1 <= 448
                S = s1 * s2
                if s2 == 0:
                    assert s1 == 0 and (qh == 0).all()
                    continue
                u = float(np.float32(np.float32(np.abs(yh).max()) / np.float32(6 * s2)))
                assert s1 == min(min(v2 for v2 in e4[:0x7F] if v2 >= u), 448.0)
                vals = np.array([E2M1[c & 7] * (-1 if c & 8 else 1) for c in qh]) * S
                # nearest point of the grid e2m1 x S (ties either way), and
                # within it: |y| <= 6 S up to the fp32 roundings of u and 1/S
                grid = np.array(E2M1 + [-v for v in E2M1[1:]]) * S
                err = np.abs(yh - vals)
                alt = np.abs(yh[:, None] - grid[None, :]).min(axis=1)
                assert (err <= alt + 1e-6 * S).all()
                assert np.abs(yh).max() <= 6 * S * (1 + 1e-6)


def test_fp4_stream_decodes_to_the_grid_and_flags():
    d, g = 128, 32
    desc, s, x, codes, meta = _raw_stream(4, g, 2, 2, [60], quant=oracle.QUANT_FP4,
                                          signs=oracle.SIGNS_PER_VECTOR, kind="outlier_t")
    assert s[11] == 4 | 8                                 # quantizer 2, per-vector signs
    st, xh = oracle.decode_values(s, desc)
    assert st == oracle.OK
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    up = 2.0 ** oracle.meta_shift(d)
    Hm = sylvester(d)
    T = 60
    for v in range(codes.shape[0]):
        q = codes_of(codes[v], d, 4)
        m = meta[v].reshape(d // g, 4)
        want = np.empty(d)
        for c in range(d):
            j, h = c // g, (c % g) // (g // 2)
            s2 = f16(int(m[j, 0]) | (int(m[j, 1]) << 8)) * up
            want[c] = E2M1[q[c] & 7] * (-1 if q[c] & 8 else 1) * e4[m[j, 2 + h]] * s2
        D = signs_of(oracle.sign_words_at(11, d, v // T), d)
        np.testing.assert_allclose(Hm @ (D * xh[v]), want, rtol=0, atol=1e-9 * abs(want).max())
    st, xb = oracle.decompress(s, desc)
    assert st == oracle.OK
    back = synth.bf16_bits(torch.from_numpy(xh).to(torch.bfloat16))
    assert (back == xb).mean() > 0.999
    other = oracle.StreamDesc(4, g, d, 2, 2, [60], 11, 0, oracle.LOSSLESS_NONE, oracle.QUANT_SYM,
                              oracle.SIGNS_PER_VECTOR)
    assert oracle.decompress(s, other)[0] == oracle.CORRUPT


def test_fp4_errors():
    d = 128
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 3.0e38                                    # y ~ 3e38: the fp16 scale overflows
    assert oracle.quantize_vectors(bf16(x), 4, 64, 0, quant=oracle.QUANT_FP4)[0] == oracle.RANGE
    x[0, 0] = np.inf
    assert oracle.quantize_vectors(bf16(x), 4, 64, 0, quant=oracle.QUANT_FP4)[0] == oracle.NONFINITE
    with pytest.raises(ValueError):                      # FP4 codes are 4-bit
        oracle.StreamDesc(2, 32, 128, 1, 1, [10], quant=oracle.QUANT_FP4).layout()
