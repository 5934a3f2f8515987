"""Pins of the oracle's scalar building blocks against things other than itself:
published generator outputs, the Sylvester Hadamard matrix, hand-derived
rounding cases, x86 F16C hardware conversion, and numpy/torch conversions."""
import ctypes as C
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split("#")[0].strip() for l in f if l.split("#")[0].strip()]


def sylvester(d):
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


# --------------------------------------------------------------------------
# sign generator
# --------------------------------------------------------------------------
def test_splitmix64_published_outputs():
    want = [int(l, 16) for l in _golden_lines("splitmix64_seed0.txt")]
    assert oracle.splitmix64(0, len(want)) == want


def test_sign_words_are_generator_outputs():
    want = oracle.splitmix64(0, 2)
    assert [int(w) for w in oracle.sign_words(0, 128)] == want
    assert [int(w) for w in oracle.sign_words(0, 64)] == want[:1]


@pytest.mark.parametrize("d,seed", [(128, 0), (64, 7), (256, 12345)])
def test_channel_sign_mapping_through_quantizer(d, seed):
    """A one-hot input x = e_c gives y = s_c * H[:, c]; y_0 = s_c, and with
    group = d the codes are 0 or 15, so code 0 reveals s_c. Channel c must be
    negated iff bit (c mod 64) of sign word c // 64 is set."""
    words = [int(w) for w in oracle.sign_words(seed, d)]
    H = sylvester(d)
    for c in [1, 5, 63, 64, 77, 129, d - 1]:
        if c >= d:
            continue
        x = np.zeros((1, d), np.uint16)
        x[0, c] = 0x3F80  # bf16 1.0
        st, codes, meta = oracle.quantize_vectors(x, 4, min(d, 128), seed)
        assert st == oracle.OK
        q = oracle.unpack_codes(codes[0], d, 4)
        neg = (words[c // 64] >> (c % 64)) & 1
        sgn = -1 if neg else 1
        expect = np.where(sgn * H[:, c] > 0, 15, 0)
        assert np.array_equal(q, expect), (c, neg)
    # channel 0: H[:, 0] is constant, so the group is constant and the sign
    # shows in the zero point z_h = RD16(s_0 * 2^-k) = +-2^-k (k = 3, 3, 4
    # for d = 64, 128, 256), an exact fp16 power of two
    x = np.zeros((1, d), np.uint16)
    x[0, 0] = 0x3F80
    st, codes, meta = oracle.quantize_vectors(x, 4, min(d, 128), seed)
    zh = int(meta[0, 2]) | (int(meta[0, 3]) << 8)
    k = {64: 3, 128: 3, 256: 4}[d]
    mag = np.float16(2.0 ** -k).view(np.uint16)
    assert zh == (int(mag) | 0x8000 if words[0] & 1 else int(mag))


# --------------------------------------------------------------------------
# Hadamard butterfly
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [4, 16, 64, 128, 256])
def test_fwht_matches_sylvester_matrix_on_integers(d):
    """Integer inputs |x| <= 2^8 keep every partial sum exact in fp32, so the
    butterfly must equal the naive O(d^2) product H x exactly."""
    rng = np.random.default_rng(d)
    H = sylvester(d)
    for _ in range(20):
        x = rng.integers(-256, 257, size=d)
        y = oracle.fwht(x.astype(np.float32))
        assert np.array_equal(y.astype(np.int64), H @ x)


@pytest.mark.parametrize("d", [16, 128])
def test_fwht_columns_and_involution(d):
    H = sylvester(d)
    assert np.array_equal(H @ H.T, d * np.eye(d, dtype=np.int64))
    for c in range(d):
        e = np.zeros(d, np.float32)
        e[c] = 1.0
        assert np.array_equal(oracle.fwht(e), H[:, c].astype(np.float32))
    rng = np.random.default_rng(1)
    x = rng.integers(-64, 65, size=d).astype(np.float32)
    assert np.array_equal(oracle.fwht(oracle.fwht(x)), d * x)


def test_fwht_random_within_rounding_bound():
    """On random inputs the fp32 butterfly stays within log2(d) roundings of
    the exact product: |err| <= log2(d) * 2^-24 * sum|x| (each stage's
    rounding is at most half an ulp of a partial sum bounded by sum|x|)."""
    rng = np.random.default_rng(3)
    d = 128
    H = sylvester(d).astype(np.float64)
    for _ in range(50):
        x = rng.standard_normal(d).astype(np.float32)
        y = oracle.fwht(x).astype(np.float64)
        exact = H @ x.astype(np.float64)
        bound = 7 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum()
        assert np.all(np.abs(y - exact) <= bound)


def test_fwht_butterfly_order_golden():
    lines = _golden_lines("fwht_order_d4.txt")
    xin = np.array([float(v) for v in lines[0].split()[1:]], np.float32)
    want = np.array([float(v) for v in lines[1].split()[1:]], np.float32)
    assert np.array_equal(oracle.fwht(xin), want)


def test_meta_shift():
    assert [oracle.meta_shift(d) for d in (64, 128, 256)] == [3, 3, 4]


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def test_bf16_to_f32_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([oracle.bf16_to_f32(int(b)) for b in bits[::97]], np.float32)
    r = ref[::97]
    assert np.array_equal(np.isnan(got), np.isnan(r))
    m = ~np.isnan(r)
    assert np.array_equal(got[m].view(np.uint32), r[m].view(np.uint32))


def test_f32_to_bf16_rne_vs_torch(pins_lib):
    rng = np.random.default_rng(5)
    u = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    specials = np.array([0, 0x80000000, 0x7F800000, 0xFF800000, 0x7F7FFFFF,
                         0x3F808000, 0x3F818000, 0x3F80FFFF, 0x00000001,
                         0x807FFFFF, 0x3F7FFF80], np.uint32)
    u = np.concatenate([u, specials])
    x = u.view(np.float32)
    out = np.zeros(x.size, np.uint16)
    pins_lib.map_f32_to_bf16(x.ctypes.data, x.size, out.ctypes.data)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(out[~nan], ref[~nan])
    assert np.all((out[nan] & 0x7F80) == 0x7F80) and np.all((out[nan] & 0x7F) != 0)


def test_f16_to_f32_all_patterns(pins_lib):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    out = np.zeros(65536, np.float32)
    pins_lib.map_f16_to_f32(h.ctypes.data, h.size, out.ctypes.data)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert np.array_equal(out[~nan].view(np.uint32), ref[~nan].view(np.uint32))


THREADS = max(1, min(32, os.cpu_count() or 1))


@pytest.mark.parametrize("toward_neg", [1, 0], ids=["RD", "RU"])
def test_f32_to_f16_directed_band_exhaustive_vs_f16c(pins_lib, toward_neg):
    """Every fp32 bit pattern whose exponent field lies in [96, 150] (all
    magnitudes from below half the smallest fp16 subnormal to above the fp16
    overflow threshold), both signs, against the CPU's F16C conversion with
    the same explicit rounding mode; every 4099th pattern elsewhere."""
    first = C.c_uint32(0)
    for sign in (0, 0x80000000):
        lo, hi = sign | (96 << 23), sign | (151 << 23) - 1
        bad = pins_lib.pin_f16_directed_mt(lo, hi, toward_neg, THREADS, 1, C.byref(first))
        assert bad == 0, f"{bad} mismatches, first at 0x{first.value:08x}"
        for a, b in ((sign, lo - 1), (hi + 1, sign | 0x7FFFFFFF)):
            bad = pins_lib.pin_f16_directed_mt(a, b, toward_neg, THREADS, 4099,
                                               C.byref(first))
            assert bad == 0, f"{bad} mismatches, first at 0x{first.value:08x}"


@pytest.mark.slow
@pytest.mark.parametrize("toward_neg", [1, 0], ids=["RD", "RU"])
def test_f32_to_f16_directed_all_patterns_vs_f16c(pins_lib, toward_neg):
    """All 2^32 fp32 bit patterns (NaNs excluded)."""
    first = C.c_uint32(0)
    bad = pins_lib.pin_f16_directed_mt(0, 0xFFFFFFFF, toward_neg, THREADS, 1,
                                       C.byref(first))
    assert bad == 0, f"{bad} mismatches, first at 0x{first.value:08x}"


def test_f32_to_f16_directed_brackets():
    """RD(x) <= x <= RU(x), both on the fp16 grid, adjacent or equal."""
    rng = np.random.default_rng(9)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 5, 2000),
                         [0.0, -0.0, 65504.0, 65520.0, -65520.0, 1e-8, -1e-8]])
    for x in xs.astype(np.float32):
        lo = np.uint16(oracle.f32_to_f16_rd(x)).view(np.float16)
        hi = np.uint16(oracle.f32_to_f16_ru(x)).view(np.float16)
        assert float(lo) <= float(x) <= float(hi)
        if float(lo) != float(hi):
            assert np.nextafter(lo, np.float16(np.inf)) == hi
