"""The C ABI without a GPU: libkvc.so loads and exports every declared symbol,
host-pure sizing agrees with the oracle's independent layout arithmetic,
invalid arguments are refused before anything is enqueued, and the host
helpers (fast division, bit transpose, sign masks) are exact."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import kv_cache_compression_04_b200 as kvc
from kv_cache_compression_04_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return kvc.lib()


def test_exports_every_declared_symbol(L):
    import glob
    hdr = ""
    for path in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))):
        with open(path) as f:
            hdr += f.read()
    declared = set(re.findall(r"\b(kvc_[a-z0-9_]+)\s*\(", hdr))
    assert declared == set(kvc.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", kvc.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    for name in declared:
        assert re.search(rf"\bT {name}$", out, re.M), name


def test_status_strings(L):
    for i, name in enumerate(kvc.STATUS):
        assert kvc.kvc_status_string(i) == name
    assert kvc.kvc_status_string(99) == "KVC_ERR_UNKNOWN"


FAKE = 0x7F0000000000  # never dereferenced: validation happens on the host


def dense(L_, H, T, D, data=FAKE):
    d = kvc.kvc_kv_desc()
    d.kind, d.layers, d.kv_heads, d.head_dim = kvc.KVC_DENSE, L_, H, D
    d.data = data
    d.stride_token = D
    d.stride_head = T * D
    d.stride_kv = H * T * D
    d.stride_layer = 2 * H * T * D
    d.tokens = T
    return d


def paged(L_, H, D, seq, pt_stride=None, page_tokens=16):
    d = kvc.kvc_kv_desc()
    d.kind, d.layers, d.kv_heads, d.head_dim = kvc.KVC_PAGED, L_, H, D
    d.data = FAKE
    d.stride_slot = D
    d.stride_head = page_tokens * D
    d.stride_kv = H * page_tokens * D
    d.stride_page = 2 * H * page_tokens * D
    npages = sum((s + page_tokens - 1) // page_tokens for s in seq) + 1
    d.stride_layer = npages * d.stride_page
    d.page_tokens, d.n_requests, d.num_pages = page_tokens, len(seq), npages
    arr = (C.c_int32 * max(1, len(seq)))(*seq)
    d.seq_lens = C.cast(arr, C.POINTER(C.c_int32))
    d.page_table = FAKE
    d.page_table_stride = pt_stride if pt_stride is not None else max(
        [(s + page_tokens - 1) // page_tokens for s in seq] + [1])
    d._keep = (arr,)
    return d


SHAPES = [(1, 8, 64, 128, 4, 128), (32, 8, 4096, 128, 4, 128), (28, 4, 32768, 128, 2, 32),
          (2, 3, 1000, 128, 4, 64), (1, 1, 1, 64, 2, 64), (3, 2, 777, 64, 4, 32),
          (2, 8, 0, 128, 4, 128), (0, 8, 16, 128, 2, 32), (5, 1, 513, 128, 2, 128)]


@pytest.mark.parametrize("Ln,H,T,D,bits,g", SHAPES)
def test_max_bytes_matches_oracle_dense(L, Ln, H, T, D, bits, g):
    p = kvc.params(bits, g)
    od = oracle.StreamDesc(bits, g, D, Ln, H, [T])
    assert kvc.kvc_max_compressed_bytes(dense(Ln, H, T, D), p) == od.max_bytes()
    lay = od.layout()
    ws = kvc.kvc_workspace_bytes(dense(Ln, H, T, D), p)
    assert ws >= 8 * lay.n_code + 16384 * lay.n_meta


@pytest.mark.parametrize("seq,bits,g", [([20, 0, 33, 16], 4, 64), ([512, 8192, 3000], 2, 32),
                                        ([0], 4, 128), ([1] * 1024, 2, 64)])
def test_max_bytes_matches_oracle_paged(L, seq, bits, g):
    p = kvc.params(bits, g)
    od = oracle.StreamDesc(bits, g, 128, 3, 2, seq)
    assert kvc.kvc_max_compressed_bytes(paged(3, 2, 128, seq), p) == od.max_bytes()


def _compress(d, p, out=FAKE, cap=1 << 40, ws=FAKE, wsb=1 << 40):
    return kvc.kvc_compress(d, p, out, cap, None, ws, wsb, None)


def test_invalid_arguments_refused_on_host(L):
    p = kvc.params(4, 128)
    d = dense(2, 2, 64, 128)
    assert _compress(d, kvc.params(3, 128)) == kvc.KVC_ERR_UNSUPPORTED
    assert _compress(d, kvc.params(4, 48)) == kvc.KVC_ERR_UNSUPPORTED
    assert _compress(dense(2, 2, 64, 64), kvc.params(4, 128)) == kvc.KVC_ERR_UNSUPPORTED
    assert _compress(dense(2, 2, 64, 96), p) == kvc.KVC_ERR_UNSUPPORTED
    assert _compress(dense(2, 2, 64, 256), p) == kvc.KVC_ERR_UNSUPPORTED
    assert _compress(d, p, out=FAKE + 8) == kvc.KVC_ERR_INVALID_ARG
    assert _compress(d, p, ws=FAKE + 4) == kvc.KVC_ERR_INVALID_ARG
    assert _compress(d, p, out=None) == kvc.KVC_ERR_INVALID_ARG
    assert _compress(dense(2, 2, 64, 128, data=FAKE + 2), p) == kvc.KVC_ERR_INVALID_ARG
    need = kvc.kvc_max_compressed_bytes(d, p)
    assert _compress(d, p, cap=need - 1) == kvc.KVC_ERR_CAPACITY
    assert _compress(d, p, wsb=kvc.kvc_workspace_bytes(d, p) - 1) == kvc.KVC_ERR_CAPACITY
    bad = dense(2, 2, 64, 128)
    bad.stride_token = 132                               # 264 B: not 16-byte aligned
    assert _compress(bad, p) == kvc.KVC_ERR_INVALID_ARG
    bad = dense(2, 2, 64, 128)
    bad.kind = 7
    assert _compress(bad, p) == kvc.KVC_ERR_INVALID_ARG
    bad = dense(2, 2, 64, 128)
    bad.tokens = -1
    assert _compress(bad, p) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.lib().kvc_compress(None, C.byref(p), FAKE, 1 << 40, None, FAKE, 1 << 40,
                                  None) == kvc.KVC_ERR_INVALID_ARG
    # paged
    assert _compress(paged(2, 2, 128, [5] * 1025), p) == kvc.KVC_ERR_INVALID_ARG
    assert _compress(paged(2, 2, 128, [5, -1]), p) == kvc.KVC_ERR_INVALID_ARG
    assert _compress(paged(2, 2, 128, [40, 3], pt_stride=2), p) == kvc.KVC_ERR_INVALID_ARG
    pg = paged(2, 2, 128, [40, 3])
    pg.page_tokens = 0
    assert _compress(pg, p) == kvc.KVC_ERR_INVALID_ARG
    # too many vectors for 32-bit indexing
    assert _compress(dense(1 << 10, 8, 1 << 20, 128), p) == kvc.KVC_ERR_UNSUPPORTED
    assert kvc.kvc_max_compressed_bytes(dense(2, 2, 64, 96), p) == 0
    assert kvc.kvc_workspace_bytes(dense(2, 2, 64, 96), p) == 0


def test_decompress_refuses_bad_arguments_on_host(L):
    d = dense(2, 2, 64, 128)
    assert kvc.kvc_decompress(FAKE + 8, 100, d, FAKE, 256, None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_decompress(FAKE, 100, d, FAKE, 255, None) == kvc.KVC_ERR_CAPACITY
    assert kvc.kvc_decompress(FAKE, 100, dense(2, 2, 64, 96), FAKE, 256,
                              None) == kvc.KVC_ERR_UNSUPPORTED


# ------------------------------------------------------------ host helpers --
@pytest.fixture(scope="module")
def host_logic():
    out = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out, exist_ok=True)
    so = os.path.join(out, f"host_logic_{os.getpid()}.so")
    subprocess.run([build.nvcc(), *build.ARCH, "-std=c++17", "-O2", "-Xcompiler", "-fPIC", "-shared",
                    os.path.join(ROOT, "tests", "csrc", "host_logic.cu"), "-o", so], check=True)
    lib = C.CDLL(so)
    os.unlink(so)
    lib.hl_fdiv.restype = C.c_uint32
    lib.hl_fdiv.argtypes = [C.c_uint32, C.c_uint32]
    lib.hl_transpose32.argtypes = [C.c_void_p, C.c_void_p]
    lib.hl_transpose32_split.argtypes = [C.c_void_p, C.c_void_p]
    lib.hl_nz_nibble_mismatches.restype = C.c_uint64
    lib.hl_nz_nibble_mismatches.argtypes = [C.c_uint64, C.c_uint64]
    lib.hl_sign_masks.argtypes = [C.c_uint64, C.c_int, C.c_void_p]
    lib.hl_div_const_mismatches.restype = C.c_uint64
    lib.hl_div_const_mismatches.argtypes = [C.c_int, C.c_uint32, C.c_uint32]
    return lib


@pytest.mark.parametrize("q", [3, 7, 15, 127, 255])
def test_division_by_quantizer_constant_sampled(host_logic, q):
    """The encoder's x / q (Markstein's correction of x * RN(1/q), compiled
    for the host) is the correctly rounded quotient: every 9973rd fp32
    pattern, i.e. samples of every binade, subnormals included."""
    assert host_logic.hl_div_const_mismatches(q, 0, 9973) == 0
    assert host_logic.hl_div_const_mismatches(q, 1, 104729) == 0


@pytest.mark.slow
@pytest.mark.parametrize("q", [3, 7, 15, 127, 255])
def test_division_by_quantizer_constant_exhaustive(host_logic, q):
    """The same over every finite x >= 0."""
    assert host_logic.hl_div_const_mismatches(q, 0, 1) == 0


def test_fast_division_exact(host_logic):
    rng = np.random.default_rng(0)
    divisors = list(range(1, 300)) + [1000, 4096, 4352, 32768, 69632, 2 ** 20 + 7,
                                      2 ** 30 - 1, 2 ** 30, 2 ** 31 - 1]
    ns = [0, 1, 2 ** 31 - 1, 2 ** 31, 2 ** 32 - 1] + list(rng.integers(0, 2 ** 32, 300))
    for dv in divisors:
        for n in ns:
            assert host_logic.hl_fdiv(dv, int(n)) == int(n) // dv, (dv, n)


@pytest.mark.parametrize("fn", ["hl_transpose32", "hl_transpose32_split"])
def test_transpose32_is_bit_matrix_transpose(host_logic, fn):
    """Both the one-thread transpose and its two-thread split (the kernels'
    form) are the bit-matrix transpose: bit l of out[p] = bit p of in[l]."""
    rng = np.random.default_rng(1)
    cases = [rng.integers(0, 2 ** 32, 32, dtype=np.uint64).astype(np.uint32) for _ in range(20)]
    cases += [np.array([1 << ((3 * i) % 32) for i in range(32)], np.uint32),
              np.eye(32, dtype=np.uint32)[0] * 0xFFFFFFFF]
    for a in cases:
        out = np.zeros(32, np.uint32)
        getattr(host_logic, fn)(a.ctypes.data, out.ctypes.data)
        bits = (a[:, None] >> np.arange(32, dtype=np.uint32)) & 1       # [row l, bit p]
        want = (bits.T.astype(np.uint64) << np.arange(32, dtype=np.uint64)).sum(1)
        assert np.array_equal(out, want.astype(np.uint32))


@pytest.mark.parametrize("seed,d", [(0, 128), (12345, 64), (2 ** 63 + 5, 128)])
def test_sign_masks_match_oracle_sign_words(host_logic, seed, d):
    m = np.zeros(d // 2, np.uint32)
    host_logic.hl_sign_masks(seed, d, m.ctypes.data)
    w = [int(x) for x in oracle.sign_words(seed, d)]
    for j in range(d // 2):
        lo = (w[(2 * j) // 64] >> ((2 * j) % 64)) & 1
        hi = (w[(2 * j + 1) // 64] >> ((2 * j + 1) % 64)) & 1
        assert m[j] == (lo << 15) | (hi << 31)


def test_nonzero_byte_mask(host_logic):
    """The lossless stage's nonzero-byte mask (add-and-gather identity)
    against a byte-by-byte reference: every word in several 2^24 ranges that
    cover all byte patterns' boundaries, and all 2^32 words under -m slow."""
    for start in (0, 0x007F0000, 0x7F7F0000, 0x80800000, 0xFF000000, 0xFFFF0000 - (1 << 24)):
        assert host_logic.hl_nz_nibble_mismatches(start, 1 << 24) == 0, hex(start)


@pytest.mark.slow
def test_nonzero_byte_mask_exhaustive(host_logic):
    assert host_logic.hl_nz_nibble_mismatches(0, 1 << 32) == 0


def test_unfused_workspace_and_argument_checks(L):
    """The unfused baseline's workspace is the fused one (rounded to 256
    bytes) plus d fp32 per vector; it validates like kvc_compress, on the
    host, before anything runs."""
    p = kvc.params(4, 128, 0)
    for Ln, H, T, D in [(1, 8, 64, 128), (32, 8, 4096, 128), (2, 3, 333, 64)]:
        d = dense(Ln, H, T, D)
        pp = kvc.params(4, 64, 0) if D == 64 else p
        base = kvc.kvc_workspace_bytes(d, pp)
        V = Ln * 2 * H * T
        assert kvc.kvc_unfused_workspace_bytes(d, pp) == (base + 255) // 256 * 256 + V * D * 4
    d = dense(2, 2, 64, 128)
    cap = kvc.kvc_max_compressed_bytes(d, p)
    wsb = kvc.kvc_unfused_workspace_bytes(d, p)
    nb = FAKE
    assert kvc.kvc_compress_unfused(d, p, FAKE, cap, nb, FAKE, wsb - 1, None) == kvc.KVC_ERR_CAPACITY
    assert kvc.kvc_compress_unfused(d, p, FAKE, cap - 1, nb, FAKE, wsb, None) == kvc.KVC_ERR_CAPACITY
    assert kvc.kvc_compress_unfused(d, kvc.params(3, 128, 0), FAKE, cap, nb, FAKE, wsb,
                                    None) == kvc.KVC_ERR_UNSUPPORTED
    assert kvc.kvc_unfused_workspace_bytes(dense(2, 2, 64, 96), p) == 0


def test_timed_calls_refuse_bad_event_arrays(L):
    import ctypes as C
    d = dense(2, 2, 64, 128)
    p = kvc.params(4, 128)
    cap = kvc.kvc_max_compressed_bytes(d, p)
    wsb = kvc.kvc_workspace_bytes(d, p)
    four = (C.c_void_p * 4)(*([FAKE] * 4))
    five_null = (C.c_void_p * 5)(FAKE, FAKE, None, FAKE, FAKE)
    for arr, n in [(four, 4), (five_null, 5), (None, 5)]:
        assert L.kvc_compress_timed(C.byref(d), C.byref(p), FAKE, cap, None, FAKE, wsb, arr, n,
                                    None) == kvc.KVC_ERR_INVALID_ARG
        assert L.kvc_decompress_timed(FAKE, 4096, C.byref(d), FAKE, 1 << 20, arr, n,
                                      None) == kvc.KVC_ERR_INVALID_ARG


class _Ptr:
    def __init__(self, p):
        self.p = p

    def data_ptr(self):
        return self.p


def test_attend_refuses_bad_arguments_and_sizes_its_workspace(L):
    """kvc_attend / kvc_attend_workspace_bytes on the host side: shape and
    pointer checks, and the workspace size (status words, one 16 KB slot per
    meta chunk, one partial record of 4 + 128 floats per CTA and query head,
    the tensor-core path's 4 KB of query fragments and 256 bytes of sums per
    (layer, request, kv head) and one address per meta chunk)."""
    q, out = _Ptr(FAKE), _Ptr(FAKE)
    lens = [1000, 0, 513]
    ad = kvc.attn_desc(2, 8, 4, 4, 64, lens, q, out, 0.1)
    wsb = kvc.kvc_attend_workspace_bytes(ad)
    V = 2 * 2 * 8 * sum(lens)
    n_meta = -(-V * 8 // 16384)            # 2 groups of 4 bytes per vector
    splits = -(-1000 // 256)
    parts = 2 * 3 * 8 * splits * 4 * 132 * 4
    prep = 2 * 3 * 8 * (4096 + 256) + 64 + 8 * n_meta   # query fragments and sums per unit
    assert wsb >= n_meta * 16384 + parts + prep
    assert wsb <= n_meta * 16384 + parts + prep + 4096
    for bad, why in [(kvc.attn_desc(2, 8, 0, 4, 64, lens, q, out, 0.1), "q_per_kv 0"),
                     (kvc.attn_desc(2, 8, 9, 4, 64, lens, q, out, 0.1), "q_per_kv 9"),
                     (kvc.attn_desc(2, 8, 4, 3, 64, lens, q, out, 0.1), "bits 3"),
                     (kvc.attn_desc(2, 8, 4, 4, 48, lens, q, out, 0.1), "group 48"),
                     (kvc.attn_desc(2, 8, 4, 4, 64, lens, q, out, 0.1, head_dim=64), "d 64"),
                     (kvc.attn_desc(2, 8, 4, 4, 64, [], q, out, 0.1), "no requests")]:
        assert kvc.kvc_attend_workspace_bytes(bad) == 0, why
        assert kvc.kvc_attend(FAKE, 1 << 20, bad, FAKE, wsb, None) != kvc.KVC_OK, why
    assert kvc.kvc_attend(FAKE, 1 << 20, ad, FAKE, wsb - 1, None) == kvc.KVC_ERR_CAPACITY
    assert kvc.kvc_attend(FAKE + 8, 1 << 20, ad, FAKE, wsb, None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_attend(FAKE, 1 << 20, kvc.attn_desc(2, 8, 4, 4, 64, lens, _Ptr(FAKE + 1),
                                                       out, 0.1), FAKE, wsb,
                          None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_attend(FAKE, 1 << 20, kvc.attn_desc(2, 8, 4, 4, 64, lens, q, _Ptr(FAKE + 2),
                                                       0.1), FAKE, wsb,
                          None) == kvc.KVC_ERR_INVALID_ARG
    assert L.kvc_attend(FAKE, 1 << 20, None, FAKE, wsb, None) == kvc.KVC_ERR_INVALID_ARG
    four = (C.c_void_p * 4)(*([FAKE] * 4))
    assert L.kvc_attend_timed(FAKE, 1 << 20, C.byref(ad), FAKE, wsb, four, 4,
                              None) == kvc.KVC_ERR_INVALID_ARG
