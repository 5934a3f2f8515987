"""Pins of the oracle's per-vector quantizer and dequantizer.

The strongest pin is a closed-form construction: a bf16-exact input whose
transformed vector lies exactly on a known 2^b-level grid, so the expected
codes, meta and the exact round trip are known without running the oracle.
A dropped term, a wrong sign or index, a transposed operand or a wrong
rounding anywhere in sign -> FWHT -> min/max -> meta -> quantize -> pack ->
unpack -> dequantize -> inverse FWHT -> unsign fails it."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sylvester(d):
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def bf16_of(v: float) -> int:
    b = np.array([v], np.float32).view(np.uint32)[0]
    assert b & 0xFFFF == 0, "value not exactly representable in bf16"
    return int(b >> 16)


def f16_bits(v: float) -> int:
    h = np.float16(v)
    assert float(h) == v
    return int(h.view(np.uint16))


def sign_vector(seed, d):
    w = [int(x) for x in oracle.sign_words(seed, d)]
    return np.array([-1 if (w[c // 64] >> (c % 64)) & 1 else 1 for c in range(d)])


GRID_CASES = [  # (d, bits, group, columns, scale exponent, seed)
    (128, 4, 128, (1, 2, 4, 8), 0, 0),
    (128, 4, 64, (3, 5, 9, 17), -3, 11),
    (128, 4, 32, (1, 2, 4, 16), 4, 2),
    (128, 2, 32, (1, 2), 0, 5),
    (128, 2, 128, (6, 9), -6, 8),
    (64, 4, 64, (1, 2, 4, 8), 2, 3),
    (64, 2, 32, (5, 10), -1, 4),
    (256, 4, 128, (1, 2, 4, 8), 1, 6),
]


@pytest.mark.parametrize("d,bits,g,cols,e,seed", GRID_CASES)
def test_closed_form_grid_roundtrip(d, bits, g, cols, e, seed):
    """x = D * sum_m a_m e_{j_m} with a_m = 2^m * 2^e gives y = H D x =
    sum_m a_m H[:, j_m] (H e_j = H[:, j]). The columns' sign patterns are
    independent linear functionals over GF(2) with support below 32, so
    every group of >= 32 consecutive channels holds all 2^b sign
    combinations: y takes the odd multiples of 2^e in [-(2^b-1), 2^b-1]*2^e,
    min = -(2^b-1)2^e, max = +(2^b-1)2^e. Then z_h = -(2^b-1)2^e/2^k and
    s_h = 2*2^e/2^k exactly, q = (y/2^e + 2^b - 1)/2, and decoding returns x
    bit for bit."""
    k = {64: 3, 128: 3, 256: 4}[d]
    qmax = (1 << bits) - 1
    H = sylvester(d)
    s = sign_vector(seed, d)
    a = [2.0 ** (m + e) for m in range(len(cols))]
    xf = np.zeros(d)
    for am, j in zip(a, cols):
        xf[j] += s[j] * am
    x = np.array([[bf16_of(v) for v in xf]], np.uint16)
    y = sum(am * H[:, j] for am, j in zip(a, cols))            # exact, float64
    q_expect = ((y / 2.0 ** e + qmax) / 2).astype(np.int64)
    assert q_expect.min() == 0 and q_expect.max() == qmax
    z_expect = f16_bits(-qmax * 2.0 ** e / 2 ** k)
    s_expect = f16_bits(2 * 2.0 ** e / 2 ** k)

    st, codes, meta = oracle.quantize_vectors(x, bits, g, seed)
    assert st == oracle.OK
    assert np.array_equal(oracle.unpack_codes(codes[0], d, bits), q_expect)
    m = meta[0].reshape(-1, 4)
    assert np.all(m[:, 0].astype(int) | (m[:, 1].astype(int) << 8) == s_expect)
    assert np.all(m[:, 2].astype(int) | (m[:, 3].astype(int) << 8) == z_expect)

    xhat = oracle.dequantize_vectors(codes, meta, d, bits, g, seed)[0]
    nz = xf != 0
    assert np.array_equal(xhat[nz], x[0][nz])
    # a zero channel decodes to sign_c * (+0): -0 where the channel's sign is -1
    assert np.array_equal(xhat[~nz], np.where(s[~nz] < 0, 0x8000, 0).astype(np.uint16))


def test_pack_golden():
    with open(os.path.join(GOLDEN, "pack_codes.txt")) as f:
        rows = [l.split("#")[0].split() for l in f if l.split("#")[0].strip()]
    for r in rows:
        bits = int(r[0][4:])
        qi, bi = r.index("q"), r.index("bytes")
        q = np.array([int(v) for v in r[qi + 1:bi]], np.uint8)
        want = np.array([int(v, 16) for v in r[bi + 1:]], np.uint8)
        assert np.array_equal(oracle.pack_codes(q, bits), want)
        assert np.array_equal(oracle.unpack_codes(want, q.size, bits), q)


@pytest.mark.parametrize("bits", [2, 4])
def test_pack_bijection(bits):
    rng = np.random.default_rng(bits)
    for _ in range(20):
        q = rng.integers(0, 1 << bits, 128).astype(np.uint8)
        assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(q, bits), 128, bits), q)


def _bf16_random(rng, n, d, scale=1.0):
    x = (rng.standard_normal((n, d)) * scale).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)   # truncation: any bf16 will do


@pytest.mark.parametrize("d,bits,g", [(128, 4, 128), (128, 4, 64), (128, 2, 32),
                                      (64, 4, 32), (256, 2, 64)])
def test_quantizer_nearest_grid_and_meta_bounds(d, bits, g):
    """Brute force: with y from the (separately pinned) butterfly, the meta
    brackets each group (z_h <= min/2^k < next16(z_h); s_h the smallest fp16
    >= s32/2^k), and every code is the nearest grid point to y up to the
    roundings of t = y - zf, r = 1/sf and t * r (each at most half an fp32
    ulp; t * r < 16): |y - (zf + q sf)| <= sf * (1/2 + 2^-18)."""
    rng = np.random.default_rng(d + bits + g)
    seed = 99
    k = {64: 3, 128: 3, 256: 4}[d]
    qmax = (1 << bits) - 1
    s = sign_vector(seed, d)
    x = _bf16_random(rng, 40, d, scale=3.0)
    st, codes, meta = oracle.quantize_vectors(x, bits, g, seed)
    assert st == oracle.OK
    for v in range(x.shape[0]):
        xv = (x[v].astype(np.uint32) << 16).view(np.float32) * s
        y = oracle.fwht(xv.astype(np.float32)).astype(np.float64)
        q = oracle.unpack_codes(codes[v], d, bits).astype(np.float64)
        m = meta[v].reshape(-1, 4).astype(np.int64)
        for j in range(d // g):
            sh = np.uint16(m[j, 0] | (m[j, 1] << 8)).view(np.float16)
            zh = np.uint16(m[j, 2] | (m[j, 3] << 8)).view(np.float16)
            yg = y[j * g:(j + 1) * g]
            mn, mx = yg.min(), yg.max()
            assert float(zh) <= mn / 2 ** k < float(np.nextafter(zh, np.float16(np.inf)))
            zf, sf = float(zh) * 2 ** k, float(sh) * 2 ** k
            s32 = np.float32(np.float32(mx - zf) / np.float32(qmax))
            assert float(sh) >= float(s32) / 2 ** k
            assert float(np.nextafter(sh, np.float16(-np.inf))) < float(s32) / 2 ** k
            assert zf <= mn and zf + qmax * sf >= mx
            qg = q[j * g:(j + 1) * g]
            assert qg.min() >= 0 and qg.max() <= qmax
            err = np.abs(yg - (zf + qg * sf))
            assert np.all(err <= sf * (0.5 + 2.0 ** -18) + 1e-30)


def test_constant_and_zero_groups():
    d, g = 128, 32
    # all-zero vector: y = 0 -> z_h = +0, s_h = +0, codes 0, decode 0
    x = np.zeros((1, d), np.uint16)
    st, codes, meta = oracle.quantize_vectors(x, 4, g, 0)
    assert st == oracle.OK and not codes.any() and not meta.any()
    xhat = oracle.dequantize_vectors(codes, meta, d, 4, g, 0)[0]
    assert np.array_equal(xhat, np.where(sign_vector(0, d) < 0, 0x8000, 0).astype(np.uint16))
    # negative zeros: the canonical +0 rule makes the meta +0 as well
    x = np.full((1, d), 0x8000, np.uint16)
    st, codes, meta = oracle.quantize_vectors(x, 4, g, 0)
    assert st == oracle.OK and not codes.any() and not meta.any()
    # one-hot at channel 0 makes every group constant (+-1): s_h = 0, codes 0
    x = np.zeros((1, d), np.uint16)
    x[0, 0] = bf16_of(1.0)
    st, codes, meta = oracle.quantize_vectors(x, 2, g, 0)
    assert st == oracle.OK and not codes.any()
    m = meta[0].reshape(-1, 4)
    assert not m[:, :2].any()


def test_nonfinite_and_range_errors():
    d = 128
    for bad in (0x7F80, 0xFF80, 0x7FC0):                     # +inf, -inf, NaN
        x = np.zeros((1, d), np.uint16)
        x[0, 17] = bad
        assert oracle.quantize_vectors(x, 4, 128, 0)[0] == oracle.NONFINITE
    # finite input whose transform overflows fp32
    x = np.full((1, d), 0x7F7F, np.uint16)                   # bf16 max
    assert oracle.quantize_vectors(x, 4, 128, 0)[0] == oracle.NONFINITE
    # |min| / 8 beyond the fp16 range -> RANGE
    # one-hot at channel 0 gives the constant y = s_0 x_0; with y = -655360
    # (= -(2^19 + 2^17), bf16-exact) min/8 = -81920 < -65504 rounds down to
    # -inf in fp16 -> RANGE
    s0 = sign_vector(0, d)[0]
    x = np.zeros((1, d), np.uint16)
    x[0, 0] = bf16_of(-s0 * 655360.0)
    assert oracle.quantize_vectors(x, 4, 128, 0)[0] == oracle.RANGE
    # y = +655360: z_h = RD16(81920) = 65504 (finite), s_h = RU16(1094.4) = 1095
    x[0, 0] = bf16_of(s0 * 655360.0)
    st, codes, meta = oracle.quantize_vectors(x, 4, 128, 0)
    assert st == oracle.OK
    assert int(meta[0, 2]) | (int(meta[0, 3]) << 8) == f16_bits(65504.0)
    assert int(meta[0, 0]) | (int(meta[0, 1]) << 8) == f16_bits(1095.0)


def _nearest_even(fr):
    """Nearest integer to a Fraction, ties to even (exact)."""
    from fractions import Fraction
    n = fr.numerator // fr.denominator
    rem = fr - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def _f32_product(t, r):
    """The fp32 product, correctly rounded (IEEE binary32 multiply, round to
    nearest even), taken from numpy's float32 arithmetic as a library routine
    and checked here against exact rationals: it is the fp32 value nearest to
    the exact product."""
    from fractions import Fraction
    p = np.float32(t) * np.float32(r)
    exact = Fraction(float(t)) * Fraction(float(r))
    lo = Fraction(float(np.nextafter(p, np.float32(-np.inf))))
    hi = Fraction(float(np.nextafter(p, np.float32(np.inf))))
    here = Fraction(float(p))
    assert abs(exact - here) <= abs(exact - lo) and abs(exact - here) <= abs(exact - hi)
    return here


def test_quantizer_rounds_the_fp32_product():
    """Reading R5 (no fused multiply-add): the code is the nearest integer,
    ties to even, to p = fl32(t*r), the product rounded to fp32 on its own.
    Cases are built where the exact t*r lies within half an fp32 ulp of
    n + 1/2 but not on it, so p is the tie n + 1/2 and goes to the even
    integer, while the exact product would round the other way half of the
    time: a quantizer that fuses the product and the rounding (one FMA with
    a rounding constant) fails here in both directions."""
    from fractions import Fraction
    rng = np.random.default_rng(7)
    found = {"up": 0, "down": 0, "tie": 0}
    for _ in range(4000):
        sf = np.float32(np.float16(rng.uniform(0.01, 4.0))) * np.float32(8)
        r = np.float32(1) / sf
        qmax = 15
        n = int(rng.integers(0, qmax))
        t0 = np.float32((n + 0.5) / float(r))
        for t in (np.nextafter(t0, np.float32(-np.inf)), t0, np.nextafter(t0, np.float32(np.inf))):
            p = _f32_product(t, r)
            want = min(max(_nearest_even(p), 0), qmax)
            got = oracle.quantize_scalar(float(t), 0.0, float(r), qmax)
            assert got == want, (float(t), float(r), got, want)
            fused = min(max(_nearest_even(Fraction(float(t)) * Fraction(float(r))), 0), qmax)
            if p == Fraction(2 * n + 1, 2) and fused != want:
                found["up" if fused > want else "down"] += 1
            elif p == Fraction(2 * n + 1, 2):
                found["tie"] += 1
    # the fp32-product rule and the exact-product rule really were separated,
    # in both directions
    assert found["up"] > 0 and found["down"] > 0, found


def test_quantizer_scalar_clamps_and_subtracts_once():
    # t = fl(y - zf) is rounded before the product: y - zf = 1 + 2^-24 rounds to 1
    y, zf = float(np.float32(1.0)), float(np.float32(-2.0 ** -24))
    assert oracle.quantize_scalar(y, zf, 2.5, 15) == 2      # exact 2.5 -> even
    assert oracle.quantize_scalar(y, zf, 3.5, 15) == 4      # exact 3.5 -> even
    assert oracle.quantize_scalar(100.0, 0.0, 1.0, 15) == 15
    assert oracle.quantize_scalar(0.0, 1.0, 1.0, 15) == 0
