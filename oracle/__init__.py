"""Plain CPU oracle of the FastKVComp-style KV-cache codec (ctypes wrapper).

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The product
path (``kv_cache_compression_04_b200``) never imports it and shares no code
with it; the two meet only through the seeded input generator, which holds
none of the method's arithmetic.

The arithmetic lives in ``kvc_oracle.c`` (plain C, fp32 with one rounding per
operation, built with ``-ffp-contract=off -fno-fast-math``). Functions below
only marshal numpy arrays.

Every oracle function is pinned by a ``-m "not gpu"`` test against something
other than itself (closed forms, hardware or library routines, hand-derived
golden values, brute force); see ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvc_oracle.c")
_HDR = os.path.join(_HERE, "kvc_oracle.h")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-pthread",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]

OK, INVALID_ARG, UNSUPPORTED, CAPACITY, NONFINITE, RANGE, CORRUPT = range(7)
CHUNK = 16384
BITMAP = 2048
HEADER = 64

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (the checker is built, not used)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_SO) or
             os.path.getmtime(_SO) < max(os.path.getmtime(_SRC),
                                         os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", *CFLAGS, "-shared", _SRC, "-o", tmp, "-lm"],
                       check=True)
        os.replace(tmp, _SO)
    return _SO


class Desc(C.Structure):
    _fields_ = [("bits", C.c_int32), ("group", C.c_int32),
                ("head_dim", C.c_int32), ("layers", C.c_int32),
                ("kv_heads", C.c_int32), ("origin", C.c_int32),
                ("n_requests", C.c_int32), ("sign_seed", C.c_uint64),
                ("token_lens", C.POINTER(C.c_uint32)), ("lossless", C.c_int32),
                ("quant", C.c_int32), ("signs", C.c_int32)]


# Lossless pipeline ids of a chunk and encoder modes (reading R17).
PIPE_ZE, PIPE_XOR_ZE, PIPE_ZE2, PIPE_XOR_ZE2 = range(4)
LOSSLESS_FIXED, LOSSLESS_SEARCH, LOSSLESS_NONE = range(3)
BITMAP2 = 256
# Quantizer (readings R5, R19) and sign diagonals (readings R3, R20).
QUANT_ASYM, QUANT_SYM, QUANT_FP4 = 0, 1, 2
SIGNS_GLOBAL, SIGNS_PER_VECTOR = 0, 1


class Layout(C.Structure):
    _fields_ = [("V", C.c_uint64), ("code_bytes", C.c_uint32),
                ("meta_bytes", C.c_uint32), ("vec_per_code", C.c_uint32),
                ("code_per_seg", C.c_uint32), ("n_code", C.c_uint64),
                ("n_meta", C.c_uint64), ("n_chunks", C.c_uint64),
                ("n_seg", C.c_uint64), ("data_base", C.c_uint64),
                ("max_bytes", C.c_uint64)]


def _p(a, ctype):
    return a.ctypes.data_as(C.POINTER(ctype))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            u8p, u16p, u32p, u64p = (C.POINTER(t) for t in
                                     (C.c_uint8, C.c_uint16, C.c_uint32,
                                      C.c_uint64))
            fp = C.POINTER(C.c_float)
            sig = {
                "orc_splitmix64_next": (C.c_uint64, [u64p]),
                "orc_sign_words": (None, [C.c_uint64, C.c_int, u64p]),
                "orc_fwht": (None, [fp, C.c_int]),
                "orc_meta_shift": (C.c_int, [C.c_int]),
                "orc_bf16_to_f32": (C.c_float, [C.c_uint16]),
                "orc_f32_to_bf16_rne": (C.c_uint16, [C.c_float]),
                "orc_f16_to_f32": (C.c_float, [C.c_uint16]),
                "orc_f32_to_f16_rd": (C.c_uint16, [C.c_float]),
                "orc_f32_to_f16_ru": (C.c_uint16, [C.c_float]),
                "orc_quantize_scalar": (C.c_int, [C.c_float, C.c_float, C.c_float, C.c_int]),
                "orc_quantize_scalar_sym": (C.c_int, [C.c_float, C.c_float, C.c_int]),
                "orc_quantize_vector_q": (C.c_int, [u16p, C.c_int, C.c_int, C.c_int,
                                                    C.c_int, u64p, u8p, u8p]),
                "orc_sign_words_at": (None, [C.c_uint64, C.c_int, C.c_uint64, u64p]),
                "orc_dequantize_vector_q": (None, [u8p, u8p, C.c_int, C.c_int, C.c_int,
                                                   C.c_int, u64p, u16p]),
                "orc_e2m1_to_f32": (C.c_float, [C.c_int]),
                "orc_f32_to_e2m1_rne": (C.c_int, [C.c_float]),
                "orc_e4m3_to_f32": (C.c_float, [C.c_int]),
                "orc_f32_to_e4m3_ru": (C.c_int, [C.c_float]),
                "orc_quantize_vector": (C.c_int, [u16p, C.c_int, C.c_int,
                                                  C.c_int, u64p, u8p, u8p]),
                "orc_dequantize_vector": (None, [u8p, u8p, C.c_int, C.c_int,
                                                 C.c_int, u64p, u16p]),
                "orc_pack_codes": (None, [u8p, C.c_int, C.c_int, u8p]),
                "orc_unpack_codes": (None, [u8p, C.c_int, C.c_int, u8p]),
                "orc_bitplane_shuffle": (None, [u8p, u8p]),
                "orc_bitplane_unshuffle": (None, [u8p, u8p]),
                "orc_lossless_encode_chunk": (C.c_uint32, [u8p, C.c_uint32,
                                                           u8p]),
                "orc_lossless_decode_chunk": (C.c_int, [u8p, C.c_uint32,
                                                        C.c_uint32, u8p]),
                "orc_layout_of": (C.c_int, [C.POINTER(Desc),
                                            C.POINTER(Layout)]),
                "orc_max_compressed_bytes": (C.c_uint64, [C.POINTER(Desc)]),
                "orc_code_chunk_index": (C.c_uint64, [C.POINTER(Layout),
                                                      C.c_uint64]),
                "orc_meta_chunk_index": (C.c_uint64, [C.POINTER(Layout),
                                                      C.c_uint64]),
                "orc_encode_segment": (C.c_int, [C.POINTER(Desc), C.c_uint64,
                                                 u16p, u8p, u32p, u8p, u32p]),
                "orc_decode_segment": (C.c_int, [C.POINTER(Desc), C.c_uint64,
                                                 u8p, u32p, u8p, u16p]),
                "orc_xor_words": (None, [u8p, C.c_uint32, C.c_int]),
                "orc_unxor_words": (None, [u8p, C.c_uint32, C.c_int]),
                "orc_ze2_encode": (C.c_uint32, [u8p, u8p]),
                "orc_ze2_decode": (C.c_int, [u8p, C.c_uint32, u8p]),
                "orc_chunk_encode_pipe": (C.c_uint32, [u8p, C.c_int, C.c_int, u8p]),
                "orc_chunk_decode_pipe": (C.c_int, [u8p, C.c_uint32, C.c_uint32,
                                                    C.c_int, C.c_int, u8p]),
                "orc_chunk_encode_select": (C.c_uint32, [u8p, C.c_uint32, C.c_int,
                                                         C.c_int, C.c_int, u8p,
                                                         C.POINTER(C.c_int)]),
                "orc_code_elim_pays": (C.c_int, [u32p, u32p, C.c_uint64]),
                "orc_compress": (C.c_int, [C.POINTER(Desc), u16p, u8p,
                                           C.c_uint64, u64p]),
                "orc_decompress": (C.c_int, [u8p, C.c_uint64,
                                             C.POINTER(Desc), u16p]),
                "orc_dequantize_vector_f64": (None, [u8p, u8p, C.c_int, C.c_int, C.c_int,
                                                     u64p, C.POINTER(C.c_double)]),
                "orc_decode_values_mt": (C.c_int, [u8p, C.c_uint64, C.POINTER(Desc),
                                                   C.POINTER(C.c_double), C.c_int]),
                "orc_attend": (C.c_int, [u8p, C.c_uint64, C.POINTER(Desc), u16p, C.c_int,
                                         C.c_double, C.POINTER(C.c_double), C.c_int]),
                "orc_compress_mt": (C.c_int, [C.POINTER(Desc), u16p, u8p,
                                              C.c_uint64, u64p, C.c_int]),
                "orc_decompress_mt": (C.c_int, [u8p, C.c_uint64,
                                                C.POINTER(Desc), u16p, C.c_int]),
                "orc_gather_dense": (None, [u16p, C.c_int, C.c_int, C.c_int64,
                                            C.c_int, C.c_int64, C.c_int64,
                                            C.c_int64, C.c_int64, C.c_uint64,
                                            C.c_uint64, u16p]),
                "orc_gather_paged": (None, [u16p, C.c_int, C.c_int, C.c_int,
                                            C.c_int64, C.c_int64, C.c_int64,
                                            C.c_int64, C.c_int64, C.c_int,
                                            C.c_int, u32p,
                                            C.POINTER(C.c_int32), C.c_int64,
                                            C.c_uint64, C.c_uint64, u16p]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------
def splitmix64(seed: int, n: int) -> list[int]:
    st = C.c_uint64(seed)
    return [lib().orc_splitmix64_next(C.byref(st)) for _ in range(n)]


def sign_words(seed: int, d: int) -> np.ndarray:
    w = np.zeros(4, np.uint64)
    lib().orc_sign_words(seed, d, _p(w, C.c_uint64))
    return w[: (d + 63) // 64]


def sign_words_at(seed: int, d: int, index: int) -> np.ndarray:
    """Sign words of the diagonal of (layer, kv, head) index `index` (R20)."""
    w = np.zeros(4, np.uint64)
    lib().orc_sign_words_at(seed, d, index, _p(w, C.c_uint64))
    return w[: (d + 63) // 64]


def fwht(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32).copy()
    lib().orc_fwht(_p(y, C.c_float), y.shape[-1])
    return y


def meta_shift(d: int) -> int:
    return lib().orc_meta_shift(d)


def f32_to_f16_rd(x: float) -> int:
    return lib().orc_f32_to_f16_rd(float(np.float32(x)))


def f32_to_f16_ru(x: float) -> int:
    return lib().orc_f32_to_f16_ru(float(np.float32(x)))


def f16_to_f32(h: int) -> float:
    return lib().orc_f16_to_f32(h)


def f32_to_bf16_rne(x: float) -> int:
    return lib().orc_f32_to_bf16_rne(float(np.float32(x)))


def bf16_to_f32(b: int) -> float:
    return lib().orc_bf16_to_f32(b)


# --------------------------------------------------------------------------
# vectors
# --------------------------------------------------------------------------
def quantize_scalar(y: float, zf: float, r: float, qmax: int) -> int:
    return lib().orc_quantize_scalar(y, zf, r, qmax)


def e2m1_to_f32(code: int) -> float:
    return lib().orc_e2m1_to_f32(code)


def f32_to_e2m1_rne(p: float) -> int:
    return lib().orc_f32_to_e2m1_rne(float(np.float32(p)))


def e4m3_to_f32(b: int) -> float:
    return lib().orc_e4m3_to_f32(b)


def f32_to_e4m3_ru(x: float) -> int:
    return lib().orc_f32_to_e4m3_ru(float(np.float32(x)))


def quantize_scalar_sym(y: float, r: float, bits: int) -> int:
    return lib().orc_quantize_scalar_sym(y, r, bits)


def quantize_vectors(x: np.ndarray, bits: int, group: int, seed: int, quant: int = QUANT_ASYM):
    """x: uint16 [V, d] bf16 bits -> (status, codes [V, d*b/8], meta [V, d/g*4])."""
    x = np.ascontiguousarray(x, np.uint16)
    V, d = x.shape
    sw = np.zeros(4, np.uint64)
    lib().orc_sign_words(seed, d, _p(sw, C.c_uint64))
    codes = np.zeros((V, d * bits // 8), np.uint8)
    meta = np.zeros((V, d // group * 4), np.uint8)
    status = OK
    for v in range(V):
        st = lib().orc_quantize_vector_q(_p(x[v], C.c_uint16), d, bits, group, quant,
                                         _p(sw, C.c_uint64), _p(codes[v], C.c_uint8),
                                         _p(meta[v], C.c_uint8))
        if st != OK and status == OK:
            status = st
    return status, codes, meta


def dequantize_vectors(codes: np.ndarray, meta: np.ndarray, d: int, bits: int,
                       group: int, seed: int, quant: int = QUANT_ASYM) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    meta = np.ascontiguousarray(meta, np.uint8)
    V = codes.shape[0]
    sw = np.zeros(4, np.uint64)
    lib().orc_sign_words(seed, d, _p(sw, C.c_uint64))
    out = np.zeros((V, d), np.uint16)
    for v in range(V):
        lib().orc_dequantize_vector_q(_p(codes[v], C.c_uint8), _p(meta[v], C.c_uint8),
                                      d, bits, group, quant, _p(sw, C.c_uint64),
                                      _p(out[v], C.c_uint16))
    return out


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    out = np.zeros(q.size * bits // 8, np.uint8)
    lib().orc_pack_codes(_p(q, C.c_uint8), q.size, bits, _p(out, C.c_uint8))
    return out


def unpack_codes(packed: np.ndarray, d: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    out = np.zeros(d, np.uint8)
    lib().orc_unpack_codes(_p(packed, C.c_uint8), d, bits, _p(out, C.c_uint8))
    return out


# --------------------------------------------------------------------------
# lossless stage
# --------------------------------------------------------------------------
def bitplane_shuffle(chunk: np.ndarray) -> np.ndarray:
    chunk = np.ascontiguousarray(chunk, np.uint8)
    assert chunk.size == CHUNK
    out = np.zeros(CHUNK, np.uint8)
    lib().orc_bitplane_shuffle(_p(chunk, C.c_uint8), _p(out, C.c_uint8))
    return out


def bitplane_unshuffle(planes: np.ndarray) -> np.ndarray:
    planes = np.ascontiguousarray(planes, np.uint8)
    assert planes.size == CHUNK
    out = np.zeros(CHUNK, np.uint8)
    lib().orc_bitplane_unshuffle(_p(planes, C.c_uint8), _p(out, C.c_uint8))
    return out


def lossless_encode_chunk(chunk: np.ndarray) -> np.ndarray:
    chunk = np.ascontiguousarray(chunk, np.uint8)
    out = np.zeros(CHUNK, np.uint8)
    n = lib().orc_lossless_encode_chunk(_p(chunk, C.c_uint8), chunk.size,
                                        _p(out, C.c_uint8))
    return out[:n].copy()


def code_elim_pays(sizes, lens) -> bool:
    """Reading R16: does zero-byte elimination in the code region pay for the
    shift of the code chunks after the first shrinking one?"""
    sizes = np.ascontiguousarray(sizes, np.uint32)
    lens = np.ascontiguousarray(lens, np.uint32)
    assert sizes.shape == lens.shape
    return bool(lib().orc_code_elim_pays(_p(sizes, C.c_uint32), _p(lens, C.c_uint32),
                                         sizes.size))


def lossless_decode_chunk(enc: np.ndarray, length: int):
    enc = np.ascontiguousarray(enc, np.uint8)
    out = np.zeros(max(length, 1), np.uint8)
    st = lib().orc_lossless_decode_chunk(_p(enc, C.c_uint8), enc.size, length,
                                         _p(out, C.c_uint8))
    return st, out[:length]


# --------------------------------------------------------------------------
# stream
# --------------------------------------------------------------------------
class StreamDesc:
    """Shape and parameters of one stream (the oracle's own description)."""

    def __init__(self, bits, group, head_dim, layers, kv_heads, token_lens,
                 sign_seed=0, origin=0, lossless=LOSSLESS_FIXED, quant=QUANT_ASYM,
                 signs=SIGNS_GLOBAL):
        self.token_lens = np.ascontiguousarray(np.asarray(token_lens, np.uint32))
        self.c = Desc(bits, group, head_dim, layers, kv_heads, origin,
                      len(self.token_lens), sign_seed,
                      _p(self.token_lens, C.c_uint32), lossless, quant, signs)

    @property
    def head_dim(self):
        return self.c.head_dim

    def layout(self) -> Layout:
        lay = Layout()
        st = lib().orc_layout_of(C.byref(self.c), C.byref(lay))
        if st != OK:
            raise ValueError(f"oracle: bad description (status {st})")
        return lay

    def max_bytes(self) -> int:
        return lib().orc_max_compressed_bytes(C.byref(self.c))


def code_chunk_index(lay: Layout, c: int) -> int:
    return lib().orc_code_chunk_index(C.byref(lay), c)


def meta_chunk_index(lay: Layout, s: int) -> int:
    return lib().orc_meta_chunk_index(C.byref(lay), s)


def compress(desc: StreamDesc, vectors: np.ndarray, threads: int = 1):
    """vectors: uint16 [V, d] in logical order -> (status, stream bytes).
    threads > 1 spreads the per-segment loop over POSIX threads (same bytes).
    The returned stream is a view of a buffer of the worst-case length."""
    vectors = np.ascontiguousarray(vectors, np.uint16)
    cap = desc.max_bytes()
    out = np.empty(cap, np.uint8)
    n = C.c_uint64(0)
    if threads > 1:
        st = lib().orc_compress_mt(C.byref(desc.c), _p(vectors, C.c_uint16),
                                   _p(out, C.c_uint8), cap, C.byref(n), int(threads))
    else:
        st = lib().orc_compress(C.byref(desc.c), _p(vectors, C.c_uint16),
                                _p(out, C.c_uint8), cap, C.byref(n))
    return st, out[: n.value]


def decompress(stream: np.ndarray, desc: StreamDesc, threads: int = 1):
    stream = np.ascontiguousarray(stream, np.uint8)
    lay = desc.layout()
    out = np.empty((lay.V, desc.head_dim), np.uint16)
    if threads > 1:
        st = lib().orc_decompress_mt(_p(stream, C.c_uint8), stream.size,
                                     C.byref(desc.c), _p(out, C.c_uint16), int(threads))
    else:
        st = lib().orc_decompress(_p(stream, C.c_uint8), stream.size,
                                  C.byref(desc.c), _p(out, C.c_uint16))
    return st, out


def encode_segment(desc: StreamDesc, s: int, vectors: np.ndarray):
    """-> (status, [chunk bytes ...], [pipeline ids]) for segment s (code
    chunks, then meta), each chunk as the encoder mode chooses it (the
    stream-wide code-region rule R16 is not applied here)."""
    vectors = np.ascontiguousarray(vectors, np.uint16)
    lay = desc.layout()
    buf = np.zeros((lay.code_per_seg + 1) * CHUNK, np.uint8)
    sizes = np.zeros(lay.code_per_seg + 1, np.uint32)
    pipes = np.zeros(lay.code_per_seg + 1, np.uint8)
    n = C.c_uint32(0)
    st = lib().orc_encode_segment(C.byref(desc.c), s, _p(vectors, C.c_uint16),
                                  _p(buf, C.c_uint8), _p(sizes, C.c_uint32),
                                  _p(pipes, C.c_uint8), C.byref(n))
    chunks, pos = [], 0
    for i in range(n.value):
        chunks.append(buf[pos:pos + sizes[i]].copy())
        pos += int(sizes[i])
    return st, chunks, [int(p) for p in pipes[:n.value]]


def decode_segment(desc: StreamDesc, s: int, chunks: list, nvec: int, pipes=None):
    lay = desc.layout()
    buf = np.concatenate(chunks).astype(np.uint8) if chunks else np.zeros(1, np.uint8)
    sizes = np.array([c.size for c in chunks], np.uint32)
    pp = np.zeros(max(len(chunks), 1), np.uint8)
    if pipes is not None:
        pp[:len(pipes)] = pipes
    out = np.zeros((nvec, desc.head_dim), np.uint16)
    st = lib().orc_decode_segment(C.byref(desc.c), s, _p(buf, C.c_uint8),
                                  _p(sizes, C.c_uint32), _p(pp, C.c_uint8),
                                  _p(out, C.c_uint16))
    return st, out


def xor_words(chunk: np.ndarray, run_words: int) -> np.ndarray:
    c = np.ascontiguousarray(chunk, np.uint8).copy()
    lib().orc_xor_words(_p(c, C.c_uint8), c.size // 4, run_words)
    return c


def unxor_words(chunk: np.ndarray, run_words: int) -> np.ndarray:
    c = np.ascontiguousarray(chunk, np.uint8).copy()
    lib().orc_unxor_words(_p(c, C.c_uint8), c.size // 4, run_words)
    return c


def ze2_encode(shuffled: np.ndarray) -> np.ndarray:
    sh = np.ascontiguousarray(shuffled, np.uint8)
    assert sh.size == CHUNK
    out = np.zeros(CHUNK + BITMAP2 + BITMAP, np.uint8)
    n = lib().orc_ze2_encode(_p(sh, C.c_uint8), _p(out, C.c_uint8))
    return out[:n].copy()


def ze2_decode(enc: np.ndarray):
    enc = np.ascontiguousarray(enc, np.uint8)
    out = np.zeros(CHUNK, np.uint8)
    st = lib().orc_ze2_decode(_p(enc, C.c_uint8), enc.size, _p(out, C.c_uint8))
    return st, out


def chunk_encode_pipe(chunk: np.ndarray, pipe: int, words_per_vector: int) -> np.ndarray:
    c = np.ascontiguousarray(chunk, np.uint8)
    assert c.size == CHUNK
    out = np.zeros(CHUNK + BITMAP2 + BITMAP, np.uint8)
    n = lib().orc_chunk_encode_pipe(_p(c, C.c_uint8), pipe, words_per_vector, _p(out, C.c_uint8))
    return out[:n].copy()


def chunk_decode_pipe(enc: np.ndarray, length: int, pipe: int, words_per_vector: int):
    enc = np.ascontiguousarray(enc, np.uint8)
    out = np.zeros(max(length, 1), np.uint8)
    st = lib().orc_chunk_decode_pipe(_p(enc, C.c_uint8), enc.size, length, pipe,
                                     words_per_vector, _p(out, C.c_uint8))
    return st, out[:length]


def chunk_encode_select(chunk: np.ndarray, is_meta: bool, words_per_vector: int, mode: int):
    """-> (encoded bytes, pipeline id) under reading R17."""
    c = np.ascontiguousarray(chunk, np.uint8)
    out = np.zeros(CHUNK + BITMAP2 + BITMAP, np.uint8)
    pipe = C.c_int(0)
    n = lib().orc_chunk_encode_select(_p(c, C.c_uint8), c.size, int(is_meta), words_per_vector,
                                      mode, _p(out, C.c_uint8), C.byref(pipe))
    return out[:n].copy(), pipe.value


def segment_vectors(lay: Layout, s: int) -> tuple[int, int]:
    vm = lay.vec_per_code * lay.code_per_seg
    return s * vm, min((s + 1) * vm, lay.V)


# --------------------------------------------------------------------------
# layouts
# --------------------------------------------------------------------------
def gather_dense(base: np.ndarray, layers, kv_heads, tokens, d, strides,
                 v_begin, v_end) -> np.ndarray:
    """base: uint16 flat buffer; strides in elements (layer, kv, head, token)."""
    base = np.ascontiguousarray(base, np.uint16)
    out = np.zeros((v_end - v_begin, d), np.uint16)
    lib().orc_gather_dense(_p(base, C.c_uint16), layers, kv_heads, tokens, d,
                           *[int(s) for s in strides], v_begin, v_end,
                           _p(out, C.c_uint16))
    return out


def gather_paged(pool: np.ndarray, layers, kv_heads, d, strides, page_tokens,
                 seq_lens, page_table, v_begin, v_end) -> np.ndarray:
    """strides in elements: (layer, page, kv, head, slot)."""
    pool = np.ascontiguousarray(pool, np.uint16)
    seq = np.ascontiguousarray(np.asarray(seq_lens, np.uint32))
    pt = np.ascontiguousarray(np.asarray(page_table, np.int32))
    out = np.zeros((v_end - v_begin, d), np.uint16)
    lib().orc_gather_paged(_p(pool, C.c_uint16), layers, kv_heads, d,
                           *[int(s) for s in strides], page_tokens, len(seq),
                           _p(seq, C.c_uint32), _p(pt, C.c_int32),
                           pt.shape[1] if pt.ndim == 2 else 0, v_begin, v_end,
                           _p(out, C.c_uint16))
    return out


# --------------------------------------------------------------------------
# attention over the compressed cache (reading R18)
# --------------------------------------------------------------------------
def decode_values(stream: np.ndarray, desc: StreamDesc, threads: int = 1):
    """-> (status, float64 [V, d]): decoded vectors without the bf16 rounding."""
    stream = np.ascontiguousarray(stream, np.uint8)
    lay = desc.layout()
    out = np.empty((lay.V, desc.head_dim), np.float64)
    st = lib().orc_decode_values_mt(_p(stream, C.c_uint8), stream.size, C.byref(desc.c),
                                    _p(out, C.c_double), int(max(1, threads)))
    return st, out


def attend(stream: np.ndarray, desc: StreamDesc, q: np.ndarray, q_per_kv: int,
           scale: float, threads: int = 1):
    """q: uint16 bf16 bits [layers, n_requests, kv_heads * q_per_kv, d] ->
    (status, float64 output of the same shape)."""
    stream = np.ascontiguousarray(stream, np.uint8)
    q = np.ascontiguousarray(q, np.uint16)
    out = np.zeros(q.shape, np.float64)
    st = lib().orc_attend(_p(stream, C.c_uint8), stream.size, C.byref(desc.c),
                          _p(q, C.c_uint16), int(q_per_kv), float(scale), _p(out, C.c_double),
                          int(max(1, threads)))
    return st, out
