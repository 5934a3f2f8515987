"""Pins of the oracle's lossless stage: bit-plane shuffle against an independent
numpy formulation and hand-placed single bits; zero-byte elimination against
hand-counted sizes, the tie rule and round trips."""
import numpy as np
import pytest

import oracle


def numpy_shuffle(chunk: np.ndarray) -> np.ndarray:
    """Independent statement of the shuffle: unpack the 4096 little-endian
    words into a [4096, 32] bit matrix (column p = bit p), transpose it to
    [32, 4096] and repack each row, bit j%8 of byte j/8 = row entry j."""
    words = chunk.view("<u4")
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).astype(np.uint8)
    return np.packbits(bits.T, axis=1, bitorder="little").reshape(-1)


def test_shuffle_matches_numpy_formulation():
    rng = np.random.default_rng(0)
    for density in (0.5, 0.05, 0.9):
        chunk = (rng.random(16384) < density).astype(np.uint8) * rng.integers(1, 256, 16384).astype(np.uint8)
        assert np.array_equal(oracle.bitplane_shuffle(chunk), numpy_shuffle(chunk))


@pytest.mark.parametrize("j,p", [(0, 0), (1, 0), (7, 31), (8, 5), (4095, 17), (1234, 9)])
def test_shuffle_single_bit_placement(j, p):
    chunk = np.zeros(16384, np.uint8)
    w = np.zeros(4096, "<u4")
    w[j] = np.uint32(1) << np.uint32(p)
    chunk[:] = w.view(np.uint8)
    out = oracle.bitplane_shuffle(chunk)
    want = np.zeros(16384, np.uint8)
    want[p * 512 + j // 8] = 1 << (j % 8)
    assert np.array_equal(out, want)


def test_shuffle_is_a_bijection():
    rng = np.random.default_rng(1)
    x = rng.integers(0, 256, 16384).astype(np.uint8)
    assert np.array_equal(oracle.bitplane_unshuffle(oracle.bitplane_shuffle(x)), x)
    assert np.array_equal(oracle.bitplane_shuffle(oracle.bitplane_unshuffle(x)), x)


def _chunk_with_shuffled_nonzeros(n, seed=0):
    """A chunk whose shuffled form has exactly n nonzero bytes."""
    rng = np.random.default_rng(seed)
    s = np.zeros(16384, np.uint8)
    idx = rng.choice(16384, n, replace=False)
    s[idx] = rng.integers(1, 256, n).astype(np.uint8)
    return oracle.bitplane_unshuffle(s), s


def test_zero_chunk_is_bitmap_only():
    enc = oracle.lossless_encode_chunk(np.zeros(16384, np.uint8))
    assert enc.size == 2048 and not enc.any()
    st, dec = oracle.lossless_decode_chunk(enc, 16384)
    assert st == oracle.OK and not dec.any()


def test_random_chunk_is_raw():
    x = np.random.default_rng(2).integers(0, 256, 16384).astype(np.uint8)
    enc = oracle.lossless_encode_chunk(x)
    assert enc.size == 16384 and np.array_equal(enc, x)


@pytest.mark.parametrize("n,size", [(14335, 16383), (14336, 16384), (0, 2048),
                                    (1, 2049), (7000, 9048)])
def test_zero_elimination_sizes_and_tie_rule(n, size):
    """Bitmap (2048 B) + nonzero bytes, used only if strictly shorter than
    16384: 14335 nonzeros -> 16383 (compressed); 14336 -> 16384 -> raw."""
    x, s = _chunk_with_shuffled_nonzeros(n, seed=n)
    enc = oracle.lossless_encode_chunk(x)
    assert enc.size == size
    if size < 16384:
        bitmap = np.unpackbits(enc[:2048], bitorder="little").astype(bool)
        assert np.array_equal(bitmap, s != 0)
        assert np.array_equal(enc[2048:], s[s != 0])
    else:
        assert np.array_equal(enc, x)
    st, dec = oracle.lossless_decode_chunk(enc, 16384)
    assert st == oracle.OK and np.array_equal(dec, x)


@pytest.mark.parametrize("length", [4, 16, 1000, 16368])
def test_short_chunk_is_raw(length):
    x = np.zeros(length, np.uint8)   # even all-zero short chunks stay raw
    enc = oracle.lossless_encode_chunk(x)
    assert enc.size == length
    st, dec = oracle.lossless_decode_chunk(enc, length)
    assert st == oracle.OK and np.array_equal(dec, x)


def test_corrupt_chunks_are_rejected():
    x, _ = _chunk_with_shuffled_nonzeros(100)
    enc = oracle.lossless_encode_chunk(x)
    assert enc.size == 2148
    bad = enc.copy()
    bad[0] ^= 0x80                                  # bitmap count != payload
    bad_bits = int(np.unpackbits(bad[:2048]).sum())
    assert bad_bits != 100
    assert oracle.lossless_decode_chunk(bad, 16384)[0] == oracle.CORRUPT
    assert oracle.lossless_decode_chunk(enc[:2000], 16384)[0] == oracle.CORRUPT
    assert oracle.lossless_decode_chunk(enc, 4096)[0] == oracle.CORRUPT
