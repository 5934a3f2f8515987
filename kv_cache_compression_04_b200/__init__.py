"""Python binding of libkvc.so, the B200 (sm_100a) KV-cache codec.

Argument marshalling only: every step of the codec runs in the library's CUDA
kernels; PyTorch supplies device memory and streams. The names mirror the C
ABI in ``include/kvc.h`` (``kvc_compress``, ``kvc_decompress``,
``kvc_max_compressed_bytes``, ``kvc_workspace_bytes``, ``kvc_stream_status``,
``kvc_status_string``). If ``libkvc.so`` has not been built, importing the
library raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkvc.so")

KVC_DENSE, KVC_PAGED = 0, 1
KVC_MAX_REQUESTS = 1024
KVC_NOALLOC_SCRATCH_BYTES = 16 << 20
STATUS = ["KVC_OK", "KVC_ERR_INVALID_ARG", "KVC_ERR_UNSUPPORTED", "KVC_ERR_CAPACITY",
          "KVC_ERR_NONFINITE", "KVC_ERR_RANGE", "KVC_ERR_CORRUPT", "KVC_ERR_TIMEOUT",
          "KVC_ERR_CUDA"]
(KVC_OK, KVC_ERR_INVALID_ARG, KVC_ERR_UNSUPPORTED, KVC_ERR_CAPACITY, KVC_ERR_NONFINITE,
 KVC_ERR_RANGE, KVC_ERR_CORRUPT, KVC_ERR_TIMEOUT, KVC_ERR_CUDA) = range(9)

# Every symbol include/kvc.h declares.
EXPORTS = ["kvc_max_compressed_bytes", "kvc_workspace_bytes", "kvc_compress",
           "kvc_decompress", "kvc_stream_status", "kvc_status_string", "kvc_compress_noalloc",
           "kvc_decompress_workspace_bytes", "kvc_unfused_workspace_bytes",
           "kvc_compress_unfused", "kvc_test_compress_stalled", "kvc_compress_timed",
           "kvc_decompress_timed", "kvc_attend_workspace_bytes", "kvc_attend",
           "kvc_attend_timed", "kvc_test_e2m1", "kvc_test_div_const",
           "kvc_test_rcp_scale"]


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS[status] if 0 <= status < len(STATUS) else status}")


class kvc_params(C.Structure):
    _fields_ = [("bits", C.c_int32), ("group_size", C.c_int32), ("sign_seed", C.c_uint64),
                ("lossless", C.c_int32), ("quant", C.c_int32), ("signs", C.c_int32),
                ("reserved", C.c_int32)]


# Quantizers (kvc_params.quant) and sign diagonals (kvc_params.signs).
KVC_QUANT_ASYM, KVC_QUANT_SYM, KVC_QUANT_FP4 = 0, 1, 2
KVC_SIGNS_GLOBAL, KVC_SIGNS_PER_VECTOR = 0, 1


# Lossless-stage modes (kvc_params.lossless) and pipeline ids of a chunk.
KVC_LOSSLESS_FIXED, KVC_LOSSLESS_SEARCH, KVC_LOSSLESS_NONE = range(3)


class kvc_attn_desc(C.Structure):
    _fields_ = [("layers", C.c_int32), ("kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("q_per_kv", C.c_int32), ("bits", C.c_int32), ("group_size", C.c_int32),
                ("quant", C.c_int32), ("kernel", C.c_int32), ("n_requests", C.c_int32),
                ("scale", C.c_float),
                ("seq_lens", C.POINTER(C.c_int32)), ("q", C.c_void_p), ("out", C.c_void_p)]


class kvc_kv_desc(C.Structure):
    _fields_ = [("kind", C.c_int32), ("layers", C.c_int32), ("kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("data", C.c_void_p),
                ("stride_layer", C.c_int64), ("stride_kv", C.c_int64),
                ("stride_head", C.c_int64), ("tokens", C.c_int64),
                ("stride_token", C.c_int64), ("page_tokens", C.c_int32),
                ("n_requests", C.c_int32), ("stride_page", C.c_int64),
                ("stride_slot", C.c_int64), ("num_pages", C.c_int64),
                ("seq_lens", C.POINTER(C.c_int32)), ("page_table", C.c_void_p),
                ("page_table_stride", C.c_int64)]


_lib = None


def lib() -> C.CDLL:
    """The loaded libkvc.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libkvc.so is not built ({LIB_PATH}); run "
                              "`python -m kv_cache_compression_04_b200.build`")
        L = C.CDLL(LIB_PATH)
        D, P = C.POINTER(kvc_kv_desc), C.POINTER(kvc_params)
        L.kvc_max_compressed_bytes.restype = C.c_size_t
        L.kvc_max_compressed_bytes.argtypes = [D, P]
        L.kvc_workspace_bytes.restype = C.c_size_t
        L.kvc_workspace_bytes.argtypes = [D, P]
        L.kvc_decompress_workspace_bytes.restype = C.c_size_t
        L.kvc_decompress_workspace_bytes.argtypes = [D]
        L.kvc_compress.restype = C.c_int
        L.kvc_compress.argtypes = [D, P, C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p,
                                   C.c_size_t, C.c_void_p]
        L.kvc_decompress.restype = C.c_int
        L.kvc_decompress.argtypes = [C.c_void_p, C.c_size_t, D, C.c_void_p, C.c_size_t,
                                     C.c_void_p]
        L.kvc_stream_status.restype = C.c_int
        L.kvc_stream_status.argtypes = [C.c_void_p, C.c_void_p]
        L.kvc_status_string.restype = C.c_char_p
        L.kvc_status_string.argtypes = [C.c_int]
        L.kvc_compress_noalloc.restype = C.c_int
        L.kvc_compress_noalloc.argtypes = [D, P, C.c_void_p, C.c_size_t, C.c_void_p,
                                           C.c_void_p, C.c_void_p]
        L.kvc_unfused_workspace_bytes.restype = C.c_size_t
        L.kvc_unfused_workspace_bytes.argtypes = [D, P]
        L.kvc_compress_unfused.restype = C.c_int
        L.kvc_compress_unfused.argtypes = [D, P, C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p,
                                           C.c_size_t, C.c_void_p]
        L.kvc_compress_timed.restype = C.c_int
        L.kvc_compress_timed.argtypes = [D, P, C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p,
                                         C.c_size_t, C.POINTER(C.c_void_p), C.c_int, C.c_void_p]
        L.kvc_decompress_timed.restype = C.c_int
        L.kvc_decompress_timed.argtypes = [C.c_void_p, C.c_size_t, D, C.c_void_p, C.c_size_t,
                                           C.POINTER(C.c_void_p), C.c_int, C.c_void_p]
        A = C.POINTER(kvc_attn_desc)
        L.kvc_attend_workspace_bytes.restype = C.c_size_t
        L.kvc_attend_workspace_bytes.argtypes = [A]
        L.kvc_attend.restype = C.c_int
        L.kvc_attend.argtypes = [C.c_void_p, C.c_size_t, A, C.c_void_p, C.c_size_t, C.c_void_p]
        L.kvc_attend_timed.restype = C.c_int
        L.kvc_attend_timed.argtypes = [C.c_void_p, C.c_size_t, A, C.c_void_p, C.c_size_t,
                                       C.POINTER(C.c_void_p), C.c_int, C.c_void_p]
        L.kvc_test_e2m1.restype = C.c_int
        L.kvc_test_e2m1.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_void_p]
        L.kvc_test_div_const.restype = C.c_int
        L.kvc_test_div_const.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_int, C.c_void_p]
        L.kvc_test_rcp_scale.restype = C.c_int
        L.kvc_test_rcp_scale.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_void_p]
        L.kvc_test_compress_stalled.restype = C.c_int
        L.kvc_test_compress_stalled.argtypes = [D, P, C.c_void_p, C.c_size_t, C.c_void_p,
                                                C.c_void_p, C.c_size_t, C.c_uint32, C.c_uint64,
                                                C.c_void_p]
        _lib = L
    return _lib


# ---------------------------------------------------------------- raw ABI --
def kvc_max_compressed_bytes(desc: kvc_kv_desc, params: kvc_params) -> int:
    return lib().kvc_max_compressed_bytes(C.byref(desc), C.byref(params))


def kvc_workspace_bytes(desc: kvc_kv_desc, params: kvc_params) -> int:
    return lib().kvc_workspace_bytes(C.byref(desc), C.byref(params))


def kvc_decompress_workspace_bytes(desc: kvc_kv_desc) -> int:
    return lib().kvc_decompress_workspace_bytes(C.byref(desc))


def kvc_compress(desc, params, out_ptr, out_capacity, out_bytes_dev_ptr, ws_ptr, ws_bytes,
                 stream) -> int:
    return lib().kvc_compress(C.byref(desc), C.byref(params), out_ptr, out_capacity,
                              out_bytes_dev_ptr, ws_ptr, ws_bytes, stream)


def kvc_unfused_workspace_bytes(desc: kvc_kv_desc, params: kvc_params) -> int:
    return lib().kvc_unfused_workspace_bytes(C.byref(desc), C.byref(params))


def kvc_compress_unfused(desc, params, out_ptr, out_capacity, out_bytes_dev_ptr, ws_ptr, ws_bytes,
                         stream) -> int:
    return lib().kvc_compress_unfused(C.byref(desc), C.byref(params), out_ptr, out_capacity,
                                      out_bytes_dev_ptr, ws_ptr, ws_bytes, stream)


def kvc_compress_noalloc(desc, params, out_ptr, out_capacity, out_bytes_dev_ptr, status_dev_ptr,
                         stream) -> int:
    return lib().kvc_compress_noalloc(C.byref(desc), C.byref(params), out_ptr, out_capacity,
                                      out_bytes_dev_ptr, status_dev_ptr, stream)


def kvc_test_compress_stalled(desc, params, out_ptr, out_capacity, out_bytes_dev_ptr, ws_ptr,
                              ws_bytes, skip_chunks, wait_ns, stream) -> int:
    """Test-only (include/kvc_test.h): kvc_compress whose compaction skips
    `skip_chunks` chunks and gives up its waits after `wait_ns`."""
    return lib().kvc_test_compress_stalled(C.byref(desc), C.byref(params), out_ptr, out_capacity,
                                           out_bytes_dev_ptr, ws_ptr, ws_bytes, skip_chunks,
                                           wait_ns, stream)


def _event_array(events):
    """torch.cuda.Event objects -> a C array of their cudaEvent_t handles."""
    return (C.c_void_p * len(events))(*[e.cuda_event for e in events])


def kvc_compress_timed(desc, params, out_ptr, out_capacity, out_bytes_dev_ptr, ws_ptr, ws_bytes,
                       events, stream) -> int:
    """kvc_compress recording `events` (5 torch.cuda.Event, created with
    enable_timing=True and already created on the device) around its kernels."""
    arr = _event_array(events)
    return lib().kvc_compress_timed(C.byref(desc), C.byref(params), out_ptr, out_capacity,
                                    out_bytes_dev_ptr, ws_ptr, ws_bytes, arr, len(events), stream)


def kvc_decompress_timed(in_ptr, in_bytes, desc, ws_ptr, ws_bytes, events, stream) -> int:
    arr = _event_array(events)
    return lib().kvc_decompress_timed(in_ptr, in_bytes, C.byref(desc), ws_ptr, ws_bytes, arr,
                                      len(events), stream)


def attn_desc(layers, kv_heads, q_per_kv, bits, group, seq_lens, q, out, scale,
              head_dim: int = 128, quant: int = 0, kernel: int = 0) -> kvc_attn_desc:
    """Descriptor of kvc_attend: q bf16 [layers, n_requests, kv_heads * q_per_kv,
    head_dim] and out fp32 of the same shape (device tensors)."""
    seq = (C.c_int32 * max(len(seq_lens), 1))(*[int(x) for x in seq_lens])
    d = kvc_attn_desc(layers, kv_heads, head_dim, q_per_kv, bits, group, quant, kernel,
                      len(seq_lens), float(scale), C.cast(seq, C.POINTER(C.c_int32)), q.data_ptr(),
                      out.data_ptr())
    d._keep = (seq, q, out)
    return d


def kvc_attend_workspace_bytes(attn: kvc_attn_desc) -> int:
    return lib().kvc_attend_workspace_bytes(C.byref(attn))


def kvc_attend(in_ptr, in_bytes, attn, ws_ptr, ws_bytes, stream) -> int:
    return lib().kvc_attend(in_ptr, in_bytes, C.byref(attn), ws_ptr, ws_bytes, stream)


def kvc_attend_timed(in_ptr, in_bytes, attn, ws_ptr, ws_bytes, events, stream) -> int:
    arr = _event_array(events)
    return lib().kvc_attend_timed(in_ptr, in_bytes, C.byref(attn), ws_ptr, ws_bytes, arr,
                                  len(events), stream)


def kvc_decompress(in_ptr, in_bytes, desc, ws_ptr, ws_bytes, stream) -> int:
    return lib().kvc_decompress(in_ptr, in_bytes, C.byref(desc), ws_ptr, ws_bytes, stream)


def kvc_stream_status(ws_ptr, stream) -> int:
    return lib().kvc_stream_status(ws_ptr, stream)


def kvc_status_string(status: int) -> str:
    return lib().kvc_status_string(status).decode()


# ------------------------------------------------------- descriptor helpers --
def params(bits: int, group: int, sign_seed: int = 0, lossless: int = KVC_LOSSLESS_FIXED,
           quant: int = KVC_QUANT_ASYM, signs: int = KVC_SIGNS_GLOBAL) -> kvc_params:
    return kvc_params(bits, group, sign_seed, lossless, quant, signs, 0)


def dense_desc(kv) -> kvc_kv_desc:
    """Descriptor of a bf16 tensor shaped [layers, 2, kv_heads, tokens, head_dim]
    (any strides with head_dim contiguous)."""
    L, two, H, T, D = kv.shape
    assert two == 2 and kv.stride(4) == 1, "expects [layers, 2, kv_heads, tokens, head_dim]"
    d = kvc_kv_desc()
    d.kind, d.layers, d.kv_heads, d.head_dim = KVC_DENSE, L, H, D
    d.data = kv.data_ptr() if kv.numel() else None
    d.stride_layer, d.stride_kv, d.stride_head = kv.stride(0), kv.stride(1), kv.stride(2)
    d.tokens, d.stride_token = T, kv.stride(3)
    d._keep = (kv,)
    return d


def paged_desc(pool, page_table, seq_lens, kv_heads: int | None = None) -> kvc_kv_desc:
    """Descriptor of a page pool shaped [layers, pages, 2, kv_heads, page_tokens,
    head_dim] with an int32 device page table [n_requests, max_pages] and a host
    list of per-request token counts."""
    L, P, two, H, PT, D = pool.shape
    assert two == 2 and pool.stride(5) == 1
    seq = (C.c_int32 * max(len(seq_lens), 1))(*[int(x) for x in seq_lens])
    d = kvc_kv_desc()
    d.kind, d.layers, d.kv_heads, d.head_dim = KVC_PAGED, L, H if kv_heads is None else kv_heads, D
    d.data = pool.data_ptr()
    d.stride_layer, d.stride_page, d.stride_kv = pool.stride(0), pool.stride(1), pool.stride(2)
    d.stride_head, d.stride_slot = pool.stride(3), pool.stride(4)
    d.page_tokens, d.n_requests, d.num_pages = PT, len(seq_lens), P
    d.seq_lens = C.cast(seq, C.POINTER(C.c_int32))
    d.page_table = page_table.data_ptr()
    d.page_table_stride = page_table.stride(0)
    d._keep = (pool, page_table, seq)
    return d


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != KVC_OK:
        raise KvcError(status, where)


# --------------------------------------------------------- convenience API --
class Codec:
    """Compresses / decompresses KV caches with caller-visible buffers.

    Buffers come from PyTorch's caching allocator (plumbing only); every
    compute step runs in libkvc's kernels. Errors raise KvcError."""

    def __init__(self, bits: int = 4, group: int = 128, sign_seed: int = 0,
                 lossless: int = KVC_LOSSLESS_FIXED, quant: int = KVC_QUANT_ASYM,
                 signs: int = KVC_SIGNS_GLOBAL):
        self.params = params(bits, group, sign_seed, lossless, quant, signs)

    def buffers(self, desc: kvc_kv_desc, device="cuda"):
        import torch
        cap = kvc_max_compressed_bytes(desc, self.params)
        wsb = kvc_workspace_bytes(desc, self.params)
        if cap == 0 or wsb == 0:
            raise KvcError(KVC_ERR_INVALID_ARG, "kvc_max_compressed_bytes")
        out = torch.empty(cap, dtype=torch.uint8, device=device)
        # one workspace serves both directions for this shape
        ws = torch.empty(max(wsb, kvc_decompress_workspace_bytes(desc)), dtype=torch.uint8,
                         device=device)
        nbytes = torch.zeros(1, dtype=torch.int64, device=device)
        return out, ws, nbytes

    def compress(self, desc: kvc_kv_desc, out=None, ws=None, nbytes=None, stream=None,
                 check: bool = True):
        """Enqueues compression; returns (out, workspace, device stream length)."""
        if out is None:
            out, ws, nbytes = self.buffers(desc)
        st = kvc_compress(desc, self.params, out.data_ptr(), out.numel(), nbytes.data_ptr(),
                          ws.data_ptr(), ws.numel(), _stream_ptr(stream))
        _check(st, "kvc_compress")
        if check:
            _check(kvc_stream_status(ws.data_ptr(), _stream_ptr(stream)), "kvc_compress (device)")
        return out, ws, nbytes

    @staticmethod
    def decompress(stream_buf, nbytes: int, desc: kvc_kv_desc, ws, stream=None,
                   check: bool = True):
        st = kvc_decompress(stream_buf.data_ptr(), int(nbytes), desc, ws.data_ptr(), ws.numel(),
                            _stream_ptr(stream))
        _check(st, "kvc_decompress")
        if check:
            _check(kvc_stream_status(ws.data_ptr(), _stream_ptr(stream)), "kvc_decompress (device)")
