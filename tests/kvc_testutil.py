"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and the
oracle on the same seeded bytes."""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_compression_04_b200 as kvc
import oracle
from kv_cache_compression_04_b200 import synth


def u16(t: torch.Tensor) -> np.ndarray:
    return synth.bf16_bits(t)


def gpu_compress(desc, bits, group, seed=0, slack: int = 0, lossless: int = 0, quant: int = 0,
                 signs: int = 0):
    """-> (status, stream uint8 numpy, device buffers)."""
    p = kvc.params(bits, group, seed, lossless, quant, signs)
    cap = kvc.kvc_max_compressed_bytes(desc, p)
    wsb = kvc.kvc_workspace_bytes(desc, p)
    assert cap > 0 and wsb > 0
    out = torch.full((cap + slack,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    nb = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = kvc.kvc_compress(desc, p, out.data_ptr(), cap, nb.data_ptr(), ws.data_ptr(), wsb,
                          kvc._stream_ptr(None))
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    st = kvc.kvc_stream_status(ws.data_ptr(), kvc._stream_ptr(None))
    n = int(nb.item())
    host = out[:n].cpu().numpy() if st == kvc.KVC_OK else None
    return st, host, out, n


def gpu_decompress(stream: np.ndarray | torch.Tensor, desc, nbytes: int | None = None):
    buf = stream if isinstance(stream, torch.Tensor) else torch.from_numpy(
        np.ascontiguousarray(stream)).cuda()
    n = buf.numel() if nbytes is None else nbytes
    ws = torch.empty(kvc.kvc_decompress_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    st = kvc.kvc_decompress(buf.data_ptr(), n, desc, ws.data_ptr(), ws.numel(),
                            kvc._stream_ptr(None))
    assert st == kvc.KVC_OK, kvc.STATUS[st]
    return kvc.kvc_stream_status(ws.data_ptr(), kvc._stream_ptr(None))


def oracle_desc(bits, group, d, layers, heads, token_lens, seed=0, origin=0, lossless=0, quant=0,
                signs=0):
    return oracle.StreamDesc(bits, group, d, layers, heads, token_lens, seed, origin, lossless,
                             quant, signs)


def first_diff(a: np.ndarray, b: np.ndarray, lay=None) -> str:
    if a.size != b.size:
        return f"sizes differ: {a.size} vs {b.size}"
    idx = np.flatnonzero(a != b)
    if idx.size == 0:
        return "equal"
    i = int(idx[0])
    msg = f"{idx.size} bytes differ, first at {i}: {a[i]:#x} vs {b[i]:#x}"
    if lay is not None and i >= lay.data_base:
        msg += f" (data offset {i - lay.data_base})"
    elif lay is not None and i >= 64:
        msg += f" (table entry {(i - 64) // 8})"
    return msg


def chunk_table(stream: np.ndarray, n_chunks: int):
    """-> (sizes, offsets) of the chunk table (pipeline ids in pipelines())."""
    e = stream[64:64 + 8 * n_chunks].view("<u8").astype(np.uint64)
    return (e & 0xFFFF).astype(np.int64), (((e >> 16) & 0xFFFFFFFFFFF) * 16).astype(np.int64)


def pipelines(stream: np.ndarray, n_chunks: int):
    e = stream[64:64 + 8 * n_chunks].view("<u8").astype(np.uint64)
    return (e >> 60).astype(np.int64)
