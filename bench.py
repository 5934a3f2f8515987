"""Throughput of the B200 KV-cache codec: one step = fused encode + fused decode
of one synthetic KV cache resident in HBM. The headline workload is the
largest single-GPU configuration, the paged ragged batch (80 layers x 2 x 8
heads x d128, 16 requests of 512..8192 tokens in 16-token pages placed by a
shuffled page table, 4-bit, group 64); Llama-3-8B- and Qwen-7B-shaped caches
and the message-size sweep are timed the same way under `per_config`.

Prints ONE JSON line (rank 0):
  value      raw bf16 bytes per second of encode + decode, all ranks (GB/s)
  e2e        the same metric through the C ABI with pinned host buffers:
             H2D KV, compress, D2H stream, H2D stream, decompress, D2H KV,
             in layer groups whose copies overlap in both directions
  roofline   the slower kernel: algorithmic bytes per launch / its CUDA-event
             duration against the measured HBM copy bandwidth
  cpu_baseline  the CPU oracle on a bounded sample of the same workload
Also: per-direction GB/s, compression ratio, break-even link speed, net wire
time saved at 100 and 400 Gbit/s, SM clocks sampled during the timed region.

Multi-GPU (torchrun): every rank compresses its own KV cache (weak scaling);
the only collectives are a barrier and a max over ranks of the timings.
`--impl reference` times the CPU oracle instead (rank 0 only).
`--sweep` runs the message-size sweep instead (1 GPU): Llama-3-8B-shaped KV
of 1 MiB .. 4 GiB, 4-bit g128 and 2-bit g32, one JSON line per point.
`--pipeline` times a layer-pipelined transfer of the llama8b cache over a
simulated 100 and 400 Gbit/s link instead (1 GPU), one JSON line per speed.
After the timed region (1 GPU), `per_config` also holds decode attention over
each compressed cache (kvc_attend against decompress + torch attention) and
the quantizer variants on the llama8b cache.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "encode/decode GB/s of raw bf16 KV on 1 B200 and % of HBM roofline; ratio"
FALLBACK_HBM_GBS = 6650.0


def traffic_file(workload: str) -> str:
    return os.path.join(ROOT, "profiles", f"dram_traffic_{workload}.txt")


def strip_c_comments(text: str) -> str:
    """C/C++ source without its comments and with runs of white space
    collapsed, so that a comment-only edit leaves the digest below unchanged
    (string literals are kept whole)."""
    import re
    tok = re.compile(r'"(?:\\.|[^"\\])*"|/\*.*?\*/|//[^\n]*', re.S)
    code = tok.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)
    return " ".join(code.split())


def kernel_source_sha() -> str:
    """Digest of the CUDA sources and the ABI headers without their comments
    (a recorded DRAM-traffic figure is stale once any code in them changed)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_compression_04_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")) +
                   glob.glob(os.path.join(csrc, "*.h"))) + sorted(
                       glob.glob(os.path.join(ROOT, "include", "*.h")))
    for f in files:
        with open(f, encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode() + b"\0" +
                     strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per compress / decompress call from the committed ncu
    summary, or None if it is missing, for another workload, or stale."""
    try:
        with open(traffic_file(workload)) as f:
            kv = dict(l.split(":", 1) for l in f.read().splitlines() if ":" in l and not l.startswith("#"))
        kv = {k.strip(): v.strip() for k, v in kv.items()}
        if kv.get("source_sha") != kernel_source_sha() or kv.get("workload") != workload:
            return None
        return {"encode_kernel": int(kv["encode_kernel_dram_bytes_per_launch"]),
                "decode_kernel": int(kv["decode_kernel_dram_bytes_per_launch"])}
    except Exception:
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while the timed
    region runs: NVML polled every millisecond from a thread (the region can
    be tens of milliseconds, shorter than nvidia-smi's sampling period);
    nvidia-smi in loop mode if NVML is unavailable. Reads only."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []          # (sm_mhz, max_mhz, set of reason names)
        self.mode = None
        self.stop = threading.Event()

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())

    def _poll(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

        def sample():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), {n for n, b in bits.items() if r & b}))
            except Exception:
                pass
        sample()  # at least one sample at each end of a very short region
        while not self.stop.is_set():
            time.sleep(0.001)
            sample()

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.mode = "nvml"
            self.thread.start()
            return self
        except Exception:
            pass
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            self.mode = "nvidia-smi"
        except Exception:
            self.mode = None
        return self

    def __exit__(self, *a):
        if self.mode == "nvml":
            self.stop.set()
            self.thread.join(timeout=5)
        elif self.mode == "nvidia-smi":
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.file.flush()
            self.file.seek(0)
            for line in self.file.read().splitlines():
                r = line.strip().split(", ")
                try:
                    self.samples.append((float(r[1]), float(r[2]),
                                         {n for n, v in zip(self.NAMES, r[5:9])
                                          if v.strip().lower() == "active"}))
                except Exception:
                    continue
            os.unlink(self.file.name)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["no samples" if self.mode else "no NVML / nvidia-smi"]}
        reasons = set().union(*(s[2] for s in self.samples))
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": self.mode}


# -------------------------------------------------------------- workloads --
def run_e2e(args, w, codec, keep, obuf, stream, dev, dist, world, raw):
    """End to end through the C ABI with pinned host buffers: every step
    uploads the KV cache, compresses it, downloads the stream, uploads it
    again, decompresses it and downloads the KV cache. The cache goes in
    layer groups (one kvc_compress / kvc_decompress call per group, each with
    its own stream, workspace and pinned buffers) on five CUDA streams (KV
    upload, compress, stream download, stream upload + decompress, KV
    download) ordered by events, so uploads and downloads of different groups
    overlap on the two copy directions."""
    import torch
    import kv_cache_compression_04_b200 as kvc
    src = keep.pool if w.paged else keep
    L = src.shape[0]
    G = max(1, min(args.e2e_groups, L))
    bounds = [(L * g // G, L * (g + 1) // G) for g in range(G)]

    def desc_of(t):
        return kvc.paged_desc(t, keep.page_table, w.seq_lens) if w.paged else kvc.dense_desc(t)

    h_in = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
    h_in.copy_(src)
    h_out = torch.empty(obuf.shape, dtype=obuf.dtype, pin_memory=True)
    groups = []
    for l0, l1 in bounds:
        sd, od = desc_of(src[l0:l1]), desc_of(obuf[l0:l1])
        out, ws, nb = codec.buffers(sd, dev)
        dws = torch.empty(kvc.kvc_decompress_workspace_bytes(od), dtype=torch.uint8, device=dev)
        groups.append(dict(l=(l0, l1), sd=sd, od=od, out=out, ws=ws, nb=nb, dws=dws,
                           hs=torch.empty(out.numel(), dtype=torch.uint8, pin_memory=True)))
    sk_in, s_enc, s_st_out, s_st_in, sk_out = (torch.cuda.Stream(dev) for _ in range(5))
    ptr = kvc._stream_ptr

    def compress(g, st):
        assert kvc.kvc_compress(g["sd"], codec.params, g["out"].data_ptr(), g["out"].numel(),
                                g["nb"].data_ptr(), g["ws"].data_ptr(), g["ws"].numel(),
                                ptr(st)) == kvc.KVC_OK

    def decompress(g, st):
        assert kvc.kvc_decompress(g["out"].data_ptr(), g["n"], g["od"], g["dws"].data_ptr(),
                                  g["dws"].numel(), ptr(st)) == kvc.KVC_OK

    for g in groups:  # stream sizes (fixed for a fixed input)
        compress(g, stream)
        g["n"] = int(g["nb"].item())
    n_total = sum(g["n"] for g in groups)
    before = obuf.view(torch.int16).sum(dtype=torch.int64)

    def e2e_step():
        go = torch.cuda.Event()
        go.record(stream)
        for s_ in (sk_in, s_enc, s_st_out, s_st_in, sk_out):
            s_.wait_event(go)
        ends = []
        for g in groups:
            (l0, l1), n = g["l"], g["n"]
            with torch.cuda.stream(sk_in):
                src[l0:l1].copy_(h_in[l0:l1], non_blocking=True)
            e = torch.cuda.Event(); e.record(sk_in); s_enc.wait_event(e)
            compress(g, s_enc)
            e = torch.cuda.Event(); e.record(s_enc); s_st_out.wait_event(e)
            with torch.cuda.stream(s_st_out):
                g["hs"][:n].copy_(g["out"][:n], non_blocking=True)
            e = torch.cuda.Event(); e.record(s_st_out); s_st_in.wait_event(e)
            with torch.cuda.stream(s_st_in):
                g["out"][:n].copy_(g["hs"][:n], non_blocking=True)
            decompress(g, s_st_in)
            e = torch.cuda.Event(); e.record(s_st_in); sk_out.wait_event(e)
            with torch.cuda.stream(sk_out):
                h_out[l0:l1].copy_(obuf[l0:l1], non_blocking=True)
        for s_ in (sk_in, s_enc, s_st_out, s_st_in, sk_out):
            e = torch.cuda.Event(); e.record(s_); stream.wait_event(e)

    e2e_step()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dist, dev)[0] / args.e2e_steps
    for g in groups:
        assert kvc.kvc_stream_status(g["ws"].data_ptr(), ptr(stream)) == kvc.KVC_OK
        assert kvc.kvc_stream_status(g["dws"].data_ptr(), ptr(stream)) == kvc.KVC_OK
    # the groups' decode equals the whole-cache decode left in obuf
    assert int(obuf.view(torch.int16).sum(dtype=torch.int64)) == int(before)
    inb = src.numel() * src.element_size()
    return {"value": round(job_gbs(raw, world, e2e_ms), 3), "unit": "GB/s",
            "h2d_bytes_per_step": inb + n_total, "d2h_bytes_per_step": n_total + inb,
            "ms_per_step": round(e2e_ms, 3), "layer_groups": G,
            "copies": "uploads and downloads of different layer groups overlap"}


def make_input(wname: str, device, rank: int):
    import torch
    from kv_cache_compression_04_b200 import synth
    import kv_cache_compression_04_b200 as kvc
    w = synth.workload(wname)
    w.seed += 1000 * rank
    if w.paged:
        pk = synth.paged_kv(w, device=device)
        desc = kvc.paged_desc(pk.pool, pk.page_table, w.seq_lens)

        def out_desc():
            pool2 = torch.empty_like(pk.pool)
            return kvc.paged_desc(pool2, pk.page_table, w.seq_lens), pool2
        return w, desc, out_desc, pk
    kv = synth.dense_kv(w, device=device)
    desc = kvc.dense_desc(kv)

    def out_desc():
        o = torch.empty_like(kv)
        return kvc.dense_desc(o), o
    return w, desc, out_desc, kv


def describe(w) -> str:
    if w.paged:
        return (f"{w.name}: {w.layers} layers x 2 x {w.kv_heads} heads x d{w.head_dim}, "
                f"{len(w.seq_lens)} requests, {w.total_tokens} tokens in 16-token pages, "
                f"{w.bits}-bit g{w.group}")
    return (f"{w.name}: [{w.layers}, 2, {w.kv_heads}, {w.tokens}, {w.head_dim}] bf16, "
            f"{w.bits}-bit g{w.group}")


# ------------------------------------------------------------ CPU oracle --
def host_cpu():
    """(logical CPUs, CPU model name) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def _sample_vectors(w, n, g):
    """n vectors drawn like the workload's keys (per-channel lognormal scales;
    Student-t values for the outlier workload), as bf16 bits."""
    import torch
    from kv_cache_compression_04_b200 import synth
    x = torch.randn(n, w.head_dim, generator=g)
    if w.kind == "lognormal":
        x = x * torch.exp(w.scale_sigma * torch.randn(1, w.head_dim, generator=g))
    return synth.bf16_bits(x.to(torch.bfloat16))


def oracle_sample(wname: str, budget_s: float, threads: int = 1, seed_offset: int = 0):
    """Round trips through the CPU oracle, as it stands, on vectors drawn like
    the workload's, until `budget_s` seconds are spent. One thread: whole
    segments one at a time (encode_segment + decode_segment). More threads:
    batches of `threads` x 4 segments through the oracle's thread pool
    (compress + decompress of a stream of that many segments). Returns (raw
    bytes processed, seconds, segments)."""
    import torch
    import oracle
    from kv_cache_compression_04_b200 import synth
    w = synth.workload(wname)
    od = oracle.StreamDesc(w.bits, w.group, w.head_dim, w.layers, w.kv_heads,
                           w.seq_lens if w.paged else [w.tokens])
    lay = od.layout()
    vm = lay.vec_per_code * lay.code_per_seg
    g = torch.Generator().manual_seed(w.seed + seed_offset)
    done_bytes, spent, segs = 0, 0.0, 0
    if threads <= 1:
        while spent < budget_s and segs < lay.n_seg:
            x = _sample_vectors(w, vm, g)
            t0 = time.perf_counter()
            st, chunks, pipes = oracle.encode_segment(od, segs, x)
            _, y = oracle.decode_segment(od, segs, chunks, vm, pipes)
            spent += time.perf_counter() - t0
            done_bytes += x.nbytes
            segs += 1
        return done_bytes, spent, segs
    nseg = 4 * threads
    # a stream of nseg whole segments: one layer, one head, K and V
    bd = oracle.StreamDesc(w.bits, w.group, w.head_dim, 1, 1, [nseg * vm // 2])
    assert bd.layout().n_seg == nseg
    x = _sample_vectors(w, nseg * vm, g)
    while spent < budget_s:
        t0 = time.perf_counter()
        st, stream = oracle.compress(bd, x, threads=threads)
        dst, y = oracle.decompress(stream, bd, threads=threads)
        spent += time.perf_counter() - t0
        assert st == oracle.OK and dst == oracle.OK
        done_bytes += x.nbytes
        segs += nseg
    return done_bytes, spent, segs


def cpu_baseline(wname: str, budget_s: float):
    """The oracle on this host: one thread, and every logical CPU."""
    n, model = host_cpu()
    b1, s1, n1 = oracle_sample(wname, budget_s / 2, threads=1)
    bn, sn, nn = oracle_sample(wname, budget_s / 2, threads=n) if n > 1 else (b1, s1, n1)
    return {"value": round(bn / sn / 1e9, 6), "unit": "GB/s", "cores": n, "kind": "oracle",
            "sample": f"{nn} whole segments ({bn} raw bytes) of vectors drawn like {wname}'s, "
                      f"encode + decode through the oracle's thread pool over segments, "
                      f"{n} threads",
            "single_thread": {"value": round(b1 / s1 / 1e9, 6), "unit": "GB/s", "cores": 1,
                              "sample": f"{n1} whole segments ({b1} raw bytes), one at a time"},
            "cpu_model": model, "host_logical_cpus": n}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    n, model = host_cpu()
    per_step = max(0.5, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(args.workload, per_step / 4, threads=n)
    tot_b, tot_s, segs = 0, 0.0, 0
    for _ in range(args.steps):
        b, s, k = oracle_sample(args.workload, per_step, threads=n)
        tot_b += b
        tot_s += s
        segs += k
    from kv_cache_compression_04_b200 import synth
    w = synth.workload(args.workload)
    v = tot_b / tot_s / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": describe(w), "sample": f"{segs} segments"},
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": n,
                             "kind": "oracle", "cpu_model": model,
                             "sample": f"{segs} whole segments of vectors drawn like "
                                       f"{args.workload}'s, encode + decode through the "
                                       f"oracle's thread pool, {n} threads"},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------- kernel events --
def new_events(n, stream):
    """n timing events, each recorded once so that its CUDA event exists
    before its handle goes through the C ABI."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:
        e.record(stream)
    return ev


def kernel_means(calls):
    """Mean duration (ms) of each of a timed call's four kernels."""
    k = len(calls)
    return [sum(c[i].elapsed_time(c[i + 1]) for c in calls) / k for i in range(4)]


def payload_bytes(w) -> int:
    """The quantized payload: packed codes and fp16 scale/zero of every vector."""
    return w.vectors * (w.head_dim * w.bits // 8 + (w.head_dim // w.group) * 4)


# ------------------------------------------------------ multi-rank timing --
def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (every rank gets the result).
    Each rank times its own work on the device; the job's time is the
    slowest rank's."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_gbs(raw_bytes_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the raw bytes all ranks processed / the time."""
    return raw_bytes_per_rank * world / (ms * 1e-3) / 1e9


# ------------------------------------------------------------------ main --
def time_config(wname: str, dev, steps: int, warmup: int, hbm: float, flush=None,
                brief: bool = False, variant: dict | None = None):
    """kvc_compress and kvc_decompress of one workload resident in HBM, timed
    like the headline step (CUDA events on the launching stream around each
    call, after `warmup` untimed steps; with `flush`, a write of it before
    every step so small inputs are not served from L2). Returns the per-call
    times, GB/s of raw input, roofline fractions (algorithmic bytes = raw
    bytes + stream bytes, against `hbm` GB/s), ratio and break-even."""
    import torch
    import kv_cache_compression_04_b200 as kvc
    w, desc, out_desc_fn, keep = make_input(wname, dev, 0)
    v = variant or {}
    w.bits, w.group = v.get("bits", w.bits), v.get("group", w.group)
    codec = kvc.Codec(w.bits, w.group, w.sign_seed, quant=v.get("quant", 0),
                      signs=v.get("signs", 0))
    out, ws, nb = codec.buffers(desc, dev)
    odesc, obuf = out_desc_fn()
    dws = torch.empty(kvc.kvc_decompress_workspace_bytes(odesc), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = kvc._stream_ptr(stream)

    def enc():
        assert kvc.kvc_compress(desc, codec.params, out.data_ptr(), out.numel(), nb.data_ptr(),
                                ws.data_ptr(), ws.numel(), sp) == kvc.KVC_OK

    enc()
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    n = int(nb.item())

    def dec():
        assert kvc.kvc_decompress(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(),
                                  sp) == kvc.KVC_OK

    dec()
    assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK
    # ordinary calls for the call-level times (dependent launches overlap the
    # kernels' tails), then timed calls for the per-kernel times
    te = []
    evs = [new_events(3, stream) for _ in range(warmup + steps)]
    cevs = [new_events(5, stream) for _ in range(warmup + steps)]
    devs = [new_events(5, stream) for _ in range(warmup + steps)]
    torch.cuda.synchronize(dev)
    for it in range(warmup + steps):
        if flush is not None:
            flush.zero_()
        e = evs[it]
        e[0].record(stream)
        enc()
        e[1].record(stream)
        dec()
        e[2].record(stream)
        if it >= warmup:
            te.append(e)
    ce, de = [], []
    for it in range(warmup + steps):
        if flush is not None:
            flush.zero_()
        c, d = cevs[it], devs[it]
        assert kvc.kvc_compress_timed(desc, codec.params, out.data_ptr(), out.numel(),
                                      nb.data_ptr(), ws.data_ptr(), ws.numel(), c,
                                      sp) == kvc.KVC_OK
        assert kvc.kvc_decompress_timed(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(), d,
                                        sp) == kvc.KVC_OK
        if it >= warmup:
            ce.append(c)
            de.append(d)
    torch.cuda.synchronize(dev)
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK
    enc_ms = statistics.median(e[0].elapsed_time(e[1]) for e in te)
    dec_ms = statistics.median(e[1].elapsed_time(e[2]) for e in te)
    enc_k = statistics.median(c[1].elapsed_time(c[2]) for c in ce)
    dec_k = statistics.median(d[3].elapsed_time(d[4]) for d in de)
    raw = w.raw_bytes
    alg = raw + n
    kalg = raw + payload_bytes(w)
    saved_bits = 8 * (raw - n)
    t_codec = (enc_ms + dec_ms) * 1e-3
    r = {"workload": describe(w), "raw_bytes": raw, "stream_bytes": n,
         "encode_ms": round(enc_ms, 4), "decode_ms": round(dec_ms, 4),
         "encode_GBps": round(raw / (enc_ms * 1e-3) / 1e9, 1),
         "decode_GBps": round(raw / (dec_ms * 1e-3) / 1e9, 1),
         "roundtrip_GBps": round(raw / t_codec / 1e9, 1),
         "encode_frac": round(alg / (enc_ms * 1e-3) / 1e9 / hbm, 4),
         "decode_frac": round(alg / (dec_ms * 1e-3) / 1e9 / hbm, 4),
         "encode_kernel_ms": round(enc_k, 4), "decode_kernel_ms": round(dec_k, 4),
         "encode_kernel_frac": round(kalg / (enc_k * 1e-3) / 1e9 / hbm, 4),
         "decode_kernel_frac": round(kalg / (dec_k * 1e-3) / 1e9 / hbm, 4),
         "ratio": round(raw / n, 4),
         "break_even_gbit_s": round(saved_bits / t_codec / 1e9, 1),
         "net_gain_ms": {"100Gbit": round((saved_bits / 100e9 - t_codec) * 1e3, 4),
                         "400Gbit": round((saved_bits / 400e9 - t_codec) * 1e3, 4)},
         "steps": steps, "timing": "median of steps",
         "l2": "flushed before every step" if flush is not None else "inputs larger than L2"}
    if brief:
        for k in ("workload", "steps", "timing", "l2", "raw_bytes"):
            r.pop(k)
        r["name"] = wname
    del keep, out, ws, nb, obuf, dws
    torch.cuda.empty_cache()
    return r


# Quantizer variants timed on the Llama-3-8B-shaped cache (same call, same
# timing as the per-config lines).
VARIANTS = {"symmetric_4bit_g128": {"quant": 1},
            "fp4_e2m1_g128": {"quant": 2},
            "8bit_g128": {"bits": 8},
            "per_vector_signs_4bit_g128": {"signs": 1}}


# query heads per kv head of the model each workload is shaped after
ATTN_QPK = {"llama8b": 4, "qwen7b": 7, "paged": 8}


def time_attend(wname: str, dev, steps: int, warmup: int, hbm: float, qpk: int | None = None):
    """One decode step of grouped-query attention over the compressed cache
    of a workload (kvc_attend: every layer, request and query head), timed
    like time_config, against (dense workloads) decompress-to-bf16 followed
    by torch's scaled_dot_product_attention, and the same attention on the
    uncompressed bf16 cache. Algorithmic bytes of the attention kernel: the
    packed codes and scale/zero of every key and value it scores (the
    payload), the bf16 queries and the fp32 outputs."""
    import torch
    import kv_cache_compression_04_b200 as kvc
    qpk = qpk or ATTN_QPK.get(wname.split("-")[0], 4)
    w, desc, out_desc_fn, keep = make_input(wname, dev, 0)
    codec = kvc.Codec(w.bits, w.group, w.sign_seed)
    out, ws, nb = codec.buffers(desc, dev)
    stream = torch.cuda.current_stream(dev)
    sp = kvc._stream_ptr(stream)
    assert kvc.kvc_compress(desc, codec.params, out.data_ptr(), out.numel(), nb.data_ptr(),
                            ws.data_ptr(), ws.numel(), sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    n = int(nb.item())
    lens = list(w.seq_lens) if w.paged else [w.tokens]
    L, H, d = w.layers, w.kv_heads, w.head_dim
    g = torch.Generator(device=dev).manual_seed(7)
    q = torch.randn(L, len(lens), H * qpk, d, generator=g, device=dev).to(torch.bfloat16)
    o = torch.empty(L, len(lens), H * qpk, d, device=dev)
    scale = d ** -0.5
    ad = kvc.attn_desc(L, H, qpk, w.bits, w.group, lens, q, o, scale)
    aws = torch.empty(kvc.kvc_attend_workspace_bytes(ad), dtype=torch.uint8, device=dev)

    def att():
        assert kvc.kvc_attend(out.data_ptr(), n, ad, aws.data_ptr(), aws.numel(),
                              sp) == kvc.KVC_OK

    att()
    assert kvc.kvc_stream_status(aws.data_ptr(), sp) == kvc.KVC_OK
    evs = [new_events(2, stream) for _ in range(warmup + steps)]
    tev = [new_events(5, stream) for _ in range(warmup + steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        e[0].record(stream)
        att()
        e[1].record(stream)
    for e in tev:
        assert kvc.kvc_attend_timed(out.data_ptr(), n, ad, aws.data_ptr(), aws.numel(), e,
                                    sp) == kvc.KVC_OK
    torch.cuda.synchronize(dev)
    assert kvc.kvc_stream_status(aws.data_ptr(), sp) == kvc.KVC_OK
    call_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs[warmup:])
    kt = [statistics.median(e[i].elapsed_time(e[i + 1]) for e in tev[warmup:]) for i in range(4)]
    alg = payload_bytes(w) + q.numel() * 2 + o.numel() * 4
    r = {"workload": describe(w), "q_per_kv": qpk, "query_heads": H * qpk,
         "requests": len(lens), "call_ms": round(call_ms, 4),
         "kernel_ms": {"clear": round(kt[0], 4), "meta_expand": round(kt[1], 4),
                       "attend": round(kt[2], 4), "combine": round(kt[3], 4)},
         "attend_kernel": {"bound": "hbm", "algorithmic_bytes": alg,
                           "achieved": round(alg / (kt[2] * 1e-3) / 1e9, 1), "peak": hbm,
                           "unit": "GB/s", "frac": round(alg / (kt[2] * 1e-3) / 1e9 / hbm, 4)},
         "kv_positions_per_s": round(L * H * w.total_tokens / (call_ms * 1e-3), 1),
         "steps": steps, "timing": "median of steps", "l2": "inputs larger than L2"}
    if not w.paged:
        # decompress to bf16, then torch's attention (flash or memory-efficient)
        odesc, obuf = out_desc_fn()
        dws = torch.empty(kvc.kvc_decompress_workspace_bytes(odesc), dtype=torch.uint8,
                          device=dev)
        qs = q.view(L, H * qpk, 1, d)
        k4, v4 = obuf[:, 0], obuf[:, 1]
        from torch.nn.attention import SDPBackend, sdpa_kernel
        F = torch.nn.functional

        def sdpa():
            with sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION,
                              SDPBackend.CUDNN_ATTENTION]):
                return F.scaled_dot_product_attention(qs, k4, v4, scale=scale, enable_gqa=True)

        def unfused():
            assert kvc.kvc_decompress(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(),
                                      sp) == kvc.KVC_OK
            return sdpa()

        try:
            unfused()
            ref = sdpa().float().view_as(o)
            torch.cuda.synchronize(dev)
            ue = [new_events(3, stream) for _ in range(warmup + steps)]
            se = [new_events(2, stream) for _ in range(warmup + steps)]
            for e in ue:
                e[0].record(stream)
                assert kvc.kvc_decompress(out.data_ptr(), n, odesc, dws.data_ptr(),
                                          dws.numel(), sp) == kvc.KVC_OK
                e[1].record(stream)
                sdpa()
                e[2].record(stream)
            for e in se:
                e[0].record(stream)
                sdpa()
                e[1].record(stream)
            torch.cuda.synchronize(dev)
            dms = statistics.median(e[0].elapsed_time(e[1]) for e in ue[warmup:])
            ams = statistics.median(e[1].elapsed_time(e[2]) for e in ue[warmup:])
            bms = statistics.median(e[0].elapsed_time(e[1]) for e in se[warmup:])
            rel = float((o - ref).abs().max() / ref.abs().max())
            r["unfused"] = {"decompress_ms": round(dms, 4), "sdpa_ms": round(ams, 4),
                            "total_ms": round(dms + ams, 4),
                            "fused_speedup": round((dms + ams) / call_ms, 3),
                            "what": "kvc_decompress to bf16, then torch "
                                    "scaled_dot_product_attention (GQA)"}
            r["uncompressed_sdpa_ms"] = round(bms, 4)
            r["vs_uncompressed_sdpa"] = round(bms / call_ms, 3)
            r["max_rel_diff_vs_bf16_sdpa"] = round(rel, 6)
        except RuntimeError as exc:  # no fused torch attention for this shape
            r["unfused"] = {"unavailable": str(exc).splitlines()[0][:200]}
        del obuf, dws
    del keep, out, ws, nb, aws, q, o
    torch.cuda.empty_cache()
    return r


def run_sweep(args):
    """Message-size sweep: [32, 2, 8, T, 128] with T = 8 * 2^i tokens (1 MiB ..
    4 GiB), 4-bit g128 and 2-bit g32. Each step times one compress and one
    decompress with CUDA events after flushing L2 (a 256 MiB write outside the
    events), so small sizes are not served from cache."""
    import torch
    import kv_cache_compression_04_b200 as kvc
    from kv_cache_compression_04_b200 import build, synth
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = kvc._stream_ptr(stream)
    for bits in (4, 2):
        for i in range(13):
            w = synth.workload(f"sweep-{i}-{bits}")
            kv = synth.dense_kv(w, device=dev)
            desc = kvc.dense_desc(kv)
            codec = kvc.Codec(w.bits, w.group, w.sign_seed)
            out, ws, nb = codec.buffers(desc, dev)
            o = torch.empty_like(kv)
            odesc = kvc.dense_desc(o)
            dws = torch.empty(kvc.kvc_decompress_workspace_bytes(odesc), dtype=torch.uint8,
                              device=dev)

            def enc():
                assert kvc.kvc_compress(desc, codec.params, out.data_ptr(), out.numel(),
                                        nb.data_ptr(), ws.data_ptr(), ws.numel(), sp) == kvc.KVC_OK

            enc()
            assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
            n = int(nb.item())

            def dec():
                assert kvc.kvc_decompress(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(),
                                          sp) == kvc.KVC_OK

            dec()
            assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK
            steps = max(5, min(100, int(4e9 / w.raw_bytes)))
            te, td = [], []
            for it in range(args.warmup + steps):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                e[0].record(stream)
                enc()
                e[1].record(stream)
                dec()
                e[2].record(stream)
                torch.cuda.synchronize(dev)
                if it >= args.warmup:
                    te.append(e[0].elapsed_time(e[1]))
                    td.append(e[1].elapsed_time(e[2]))
            assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
            enc_ms, dec_ms = statistics.median(te), statistics.median(td)
            raw = w.raw_bytes
            saved_bits = 8 * (raw - n)
            t_codec = (enc_ms + dec_ms) * 1e-3
            print(json.dumps({
                "sweep": w.name, "bits": w.bits, "group": w.group, "raw_bytes": raw,
                "stream_bytes": n, "ratio": round(raw / n, 4), "steps": steps,
                "encode_us": round(enc_ms * 1e3, 2), "decode_us": round(dec_ms * 1e3, 2),
                "encode_GBps": round(raw / (enc_ms * 1e-3) / 1e9, 1),
                "decode_GBps": round(raw / (dec_ms * 1e-3) / 1e9, 1),
                "roundtrip_GBps": round(raw / t_codec / 1e9, 1),
                "break_even_gbit_s": round(saved_bits / t_codec / 1e9, 1),
                "net_gain_ms": {"100Gbit": round((saved_bits / 100e9 - t_codec) * 1e3, 4),
                                "400Gbit": round((saved_bits / 400e9 - t_codec) * 1e3, 4)},
                "l2": "flushed before every step (256 MiB write)", "timing": "median of steps"}),
                flush=True)
            del kv, out, ws, nb, o, dws
            torch.cuda.empty_cache()
    return 0


class LayerPipeline:
    """Layer-pipelined transfer of a dense KV cache: layer l is compressed on
    one stream, held on a 'wire' stream for its stream bytes / link speed (a
    spin of that many SM cycles at the given clock), then decompressed on a
    third stream into the receiver's cache, so compression, transfer and
    decompression of different layers overlap. One kvc_compress and one
    kvc_decompress call per layer, each with its own buffers."""

    def __init__(self, kv, rx, codec, dev):
        import torch
        import kv_cache_compression_04_b200 as kvc
        self.kvc, self.torch, self.dev, self.codec = kvc, torch, dev, codec
        self.L = kv.shape[0]
        self.descs = [kvc.dense_desc(kv[l:l + 1]) for l in range(self.L)]
        self.odescs = [kvc.dense_desc(rx[l:l + 1]) for l in range(self.L)]
        self.bufs = [codec.buffers(d, dev) for d in self.descs]
        self.dws = [torch.empty(kvc.kvc_decompress_workspace_bytes(d), dtype=torch.uint8,
                                device=dev) for d in self.odescs]
        self.se, self.sw, self.sd = (torch.cuda.Stream(dev) for _ in range(3))
        self.pe, self.pd = kvc._stream_ptr(self.se), kvc._stream_ptr(self.sd)
        for l in range(self.L):
            self.enc(l)
        torch.cuda.synchronize(dev)
        self.n = [int(b[2].item()) for b in self.bufs]

    def enc(self, l):
        out, ws, nb = self.bufs[l]
        assert self.kvc.kvc_compress(self.descs[l], self.codec.params, out.data_ptr(),
                                     out.numel(), nb.data_ptr(), ws.data_ptr(), ws.numel(),
                                     self.pe) == self.kvc.KVC_OK

    def dec(self, l):
        out = self.bufs[l][0]
        assert self.kvc.kvc_decompress(out.data_ptr(), self.n[l], self.odescs[l],
                                       self.dws[l].data_ptr(), self.dws[l].numel(),
                                       self.pd) == self.kvc.KVC_OK

    def transfer(self, link_bytes_per_s: float, sm_hz: float) -> float:
        """One pipelined transfer; returns its CUDA-event time in ms."""
        torch = self.torch
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(self.se)
        for l in range(self.L):
            self.enc(l)
            e1 = torch.cuda.Event()
            e1.record(self.se)
            self.sw.wait_event(e1)
            with torch.cuda.stream(self.sw):
                torch.cuda._sleep(int(self.n[l] / link_bytes_per_s * sm_hz))
            e2 = torch.cuda.Event()
            e2.record(self.sw)
            self.sd.wait_event(e2)
            self.dec(l)
        t1.record(self.sd)
        torch.cuda.synchronize(self.dev)
        return t0.elapsed_time(t1)

    def statuses_ok(self) -> bool:
        return all(self.kvc.kvc_stream_status(d.data_ptr(), self.pd) == self.kvc.KVC_OK
                   for d in self.dws)


def run_pipeline(args):
    """Layer-pipelined transfer of the llama8b cache over a simulated 100 and
    400 Gbit/s link (LayerPipeline), compared with sending the raw bf16 cache
    over the same link. The receiver's cache is checked against a whole-cache
    round trip (decoding is per vector, so the chunking does not change it)."""
    import torch
    import kv_cache_compression_04_b200 as kvc
    from kv_cache_compression_04_b200 import build, synth
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.workload("llama8b")
    kv = synth.dense_kv(w, device=dev)
    rx = torch.empty_like(kv)
    codec = kvc.Codec(w.bits, w.group, w.sign_seed)
    L = w.layers
    pipe = LayerPipeline(kv, rx, codec, dev)
    n = pipe.n
    # whole-cache reference for the receiver's check
    ref = torch.empty_like(kv)
    se = pipe.se
    with torch.cuda.stream(se):
        cout, cws, cnb = codec.buffers(kvc.dense_desc(kv), dev)
        sp = kvc._stream_ptr(se)
        assert kvc.kvc_compress(kvc.dense_desc(kv), codec.params, cout.data_ptr(), cout.numel(),
                                cnb.data_ptr(), cws.data_ptr(), cws.numel(), sp) == kvc.KVC_OK
        rdesc = kvc.dense_desc(ref)
        rws = torch.empty(kvc.kvc_decompress_workspace_bytes(rdesc), dtype=torch.uint8,
                          device=dev)
        torch.cuda.synchronize(dev)
        assert kvc.kvc_decompress(cout.data_ptr(), int(cnb.item()), rdesc, rws.data_ptr(),
                                  rws.numel(), sp) == kvc.KVC_OK
    torch.cuda.synchronize(dev)
    try:
        import pynvml
        pynvml.nvmlInit()
        sm_hz = pynvml.nvmlDeviceGetMaxClockInfo(pynvml.nvmlDeviceGetHandleByIndex(0),
                                                 pynvml.NVML_CLOCK_SM) * 1e6
    except Exception:
        sm_hz = 1.965e9
    raw_l = w.raw_bytes // L
    # per-layer compress and decompress times, each stage alone (for the
    # two-GPU model: sender and receiver are different GPUs)
    te = [torch.cuda.Event(enable_timing=True) for _ in range(L + 1)]
    td = [torch.cuda.Event(enable_timing=True) for _ in range(L + 1)]
    enc_ms, dec_ms = [0.0] * L, [0.0] * L
    for rep in range(args.warmup + 3):
        te[0].record(se)
        for l in range(L):
            pipe.enc(l)
            te[l + 1].record(se)
        torch.cuda.synchronize(dev)
        td[0].record(pipe.sd)
        for l in range(L):
            pipe.dec(l)
            td[l + 1].record(pipe.sd)
        torch.cuda.synchronize(dev)
        if rep >= args.warmup:
            for l in range(L):
                enc_ms[l] += te[l].elapsed_time(te[l + 1]) / 3
                dec_ms[l] += td[l].elapsed_time(td[l + 1]) / 3
    for gbit in (100, 400):
        link = gbit * 1e9 / 8  # bytes per second
        times = []
        for rep in range(args.warmup + 3):
            rx.zero_()
            torch.cuda.synchronize(dev)
            ms = pipe.transfer(link, sm_hz)
            if rep >= args.warmup:
                times.append(ms)
        assert pipe.statuses_ok()
        assert torch.equal(rx.view(torch.int16), ref.view(torch.int16))
        pipe_ms = statistics.median(times)
        raw_ms = w.raw_bytes / link * 1e3
        e_t = w_t = d_t = 0.0  # three-stage pipeline, sender and receiver on two GPUs
        for l in range(L):
            e_t += enc_ms[l]
            w_t = max(e_t, w_t) + n[l] / link * 1e3
            d_t = max(w_t, d_t) + dec_ms[l]
        print(json.dumps({
            "pipeline": "llama8b cache, one batch per layer (32), compress -> simulated link -> "
                        "decompress on three streams",
            "link_gbit_s": gbit, "raw_bytes": w.raw_bytes, "stream_bytes": sum(n),
            "raw_transfer_ms": round(raw_ms, 3),
            "compressed_transfer_only_ms": round(sum(n) / link * 1e3, 3),
            "pipelined_one_gpu_ms": round(pipe_ms, 3),
            "speedup_vs_raw_one_gpu": round(raw_ms / pipe_ms, 3),
            "pipelined_two_gpu_model_ms": round(d_t, 3),
            "speedup_vs_raw_two_gpu_model": round(raw_ms / d_t, 3),
            "per_layer_compress_us": round(sum(enc_ms) / L * 1e3, 2),
            "per_layer_decompress_us": round(sum(dec_ms) / L * 1e3, 2),
            "per_layer_raw_bytes": raw_l, "link_model": "spin of stream bytes / link seconds "
                                                        "at the max SM clock",
            "receiver_check": "equal to a whole-cache round trip"}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="paged",
                    help="the headline workload (the largest single-GPU configuration)")
    ap.add_argument("--per-config", default="llama8b,qwen7b",
                    help="other workloads timed after the headline one ('' for none)")
    ap.add_argument("--config-steps", type=int, default=20)
    ap.add_argument("--sweep-points", type=int, default=1,
                    help="1: also time every message-size sweep point into per_config")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-groups", type=int, default=8,
                    help="layer groups of the end-to-end timing (one call pair each)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--unfused-steps", type=int, default=20)
    ap.add_argument("--attend", type=int, default=1,
                    help="1: also time decode attention over each compressed cache")
    ap.add_argument("--variants", type=int, default=1,
                    help="1: also time the quantizer variants on the llama8b cache")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--pipeline", action="store_true")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep(args)
    if args.pipeline:
        return run_pipeline(args)
    if args.impl == "reference":
        return run_reference(args)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import torch
    import kv_cache_compression_04_b200 as kvc
    from kv_cache_compression_04_b200 import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    build.build()
    dev = torch.device("cuda", local)

    w, desc, out_desc_fn, keep = make_input(args.workload, dev, rank)
    codec = kvc.Codec(w.bits, w.group, w.sign_seed)
    out, ws, nb = codec.buffers(desc, dev)
    odesc, obuf = out_desc_fn()
    dws = torch.empty(kvc.kvc_decompress_workspace_bytes(odesc), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = kvc._stream_ptr(stream)
    raw = w.raw_bytes

    def enc():
        st = kvc.kvc_compress(desc, codec.params, out.data_ptr(), out.numel(), nb.data_ptr(),
                              ws.data_ptr(), ws.numel(), sp)
        assert st == kvc.KVC_OK, kvc.STATUS[st]

    def dec(n):
        st = kvc.kvc_decompress(out.data_ptr(), n, odesc, dws.data_ptr(), dws.numel(), sp)
        assert st == kvc.KVC_OK, kvc.STATUS[st]

    # correctness gate + stream size
    enc()
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    nbytes = int(nb.item())
    dec(nbytes)
    assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK

    for _ in range(args.warmup):
        enc()
        dec(nbytes)
    K = args.steps
    # Each step's calls record five events each around their kernels
    # (kvc_compress_timed / kvc_decompress_timed), so the dominant kernels
    # are timed on the launching stream inside the timed region itself.
    ce = [new_events(5, stream) for _ in range(K)]
    de = [new_events(5, stream) for _ in range(K)]
    start, stop = new_events(2, stream)

    def enc_timed(e):
        st = kvc.kvc_compress_timed(desc, codec.params, out.data_ptr(), out.numel(),
                                    nb.data_ptr(), ws.data_ptr(), ws.numel(), e, sp)
        assert st == kvc.KVC_OK, kvc.STATUS[st]

    def dec_timed(e):
        st = kvc.kvc_decompress_timed(out.data_ptr(), nbytes, odesc, dws.data_ptr(), dws.numel(),
                                      e, sp)
        assert st == kvc.KVC_OK, kvc.STATUS[st]

    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(K):
            enc_timed(ce[i])
            dec_timed(de[i])
        stop.record(stream)
        # poll instead of blocking so the clock sampler thread keeps running
        while not stop.query():
            time.sleep(0.0002)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    total_ms = start.elapsed_time(stop)
    kc = kernel_means(ce)     # clear, encode, finish, compaction
    kd = kernel_means(de)     # clear, meta expansion, eliminated-chunk decode, decode
    enc_call = sum(e[0].elapsed_time(e[4]) for e in ce) / K
    dec_call = sum(e[0].elapsed_time(e[4]) for e in de) / K
    total_ms, enc_avg, dec_avg, enc_k, dec_k = max_over_ranks(
        [total_ms, enc_call, dec_call, kc[1], kd[3]], dist, dev)
    assert kvc.kvc_stream_status(ws.data_ptr(), sp) == kvc.KVC_OK
    assert kvc.kvc_stream_status(dws.data_ptr(), sp) == kvc.KVC_OK

    # ------------------------------------------------ end to end via host --
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, w, codec, keep, obuf, stream, dev, dist, world, raw)

    # ------------------------------------- unfused baseline (fusion gain) --
    # The same compress call as two kernels with the fp32 transformed tensor
    # in HBM between them (kvc_compress_unfused; identical stream), timed the
    # same way, outside the timed region above.
    unfused = None
    if args.unfused_steps > 0:
        uws = torch.empty(kvc.kvc_unfused_workspace_bytes(desc, codec.params), dtype=torch.uint8,
                          device=dev)

        def enc_unfused():
            st = kvc.kvc_compress_unfused(desc, codec.params, out.data_ptr(), out.numel(),
                                          nb.data_ptr(), uws.data_ptr(), uws.numel(), sp)
            assert st == kvc.KVC_OK, kvc.STATUS[st]

        for _ in range(3):
            enc_unfused()
        u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        u0.record(stream)
        for _ in range(args.unfused_steps):
            enc_unfused()
        u1.record(stream)
        torch.cuda.synchronize(dev)
        assert kvc.kvc_stream_status(uws.data_ptr(), sp) == kvc.KVC_OK
        assert int(nb.item()) == nbytes
        u_ms = max_over_ranks([u0.elapsed_time(u1) / args.unfused_steps], dist, dev)[0]
        unfused = {"encode_ms": round(u_ms, 4), "fusion_speedup": round(u_ms / enc_avg, 3),
                   "intermediate_bytes": int(w.vectors) * w.head_dim * 4,
                   "what": "kvc_compress_unfused: transform kernel -> fp32 tensor in HBM -> "
                           "quantize kernel, same finishing kernels, same stream"}
        del uws

    # -------------------------- the other workloads, timed the same way --
    # (after the timed region, with the headline workload's buffers freed)
    per_config = None
    if world == 1 and (args.per_config or args.attend or args.variants or args.sweep_points):
        del out, ws, nb, obuf, dws, keep
        torch.cuda.empty_cache()
        hbm_, _ = peaks()
        per_config = {}
        for wname in [x for x in args.per_config.split(",") if x and x != args.workload]:
            per_config[wname] = time_config(wname, dev, args.config_steps, args.warmup, hbm_)
            if args.attend:
                per_config[wname]["attend"] = time_attend(wname, dev, args.config_steps,
                                                          args.warmup, hbm_)
        if args.attend:
            per_config["attend_" + args.workload] = time_attend(args.workload, dev,
                                                                args.config_steps, args.warmup,
                                                                hbm_)
        if args.variants:
            per_config["variants_llama8b"] = {
                name: time_config("llama8b", dev, args.config_steps, args.warmup, hbm_,
                                  brief=True, variant=v) for name, v in VARIANTS.items()}
        if args.sweep_points:
            flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
            per_config["sweep"] = [time_config(f"sweep-{i}-{b}", dev, args.config_steps,
                                               args.warmup, hbm_, flush=flush, brief=True)
                                   for b in (4, 2) for i in range(13)]
            del flush
            torch.cuda.empty_cache()

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    hbm, peak_kind = peaks()
    traffic = recorded_traffic(args.workload)
    step_ms = total_ms / K
    value = job_gbs(raw, world, step_ms)
    # algorithmic bytes: a call reads the KV cache and writes the stream (or
    # the reverse); the fused encode kernel reads the KV cache and writes the
    # quantized payload (codes in place, raw meta to the workspace), the
    # decode kernel the reverse (2 bytes per raw element, bits/8 per code,
    # 4 bytes of scale and zero per group)
    pay = payload_bytes(w)
    enc_gbs = (raw + nbytes) / (enc_avg * 1e-3) / 1e9
    dec_gbs = (raw + nbytes) / (dec_avg * 1e-3) / 1e9
    enc_k_gbs = (raw + pay) / (enc_k * 1e-3) / 1e9
    dec_k_gbs = (raw + pay) / (dec_k * 1e-3) / 1e9
    dom = "encode_kernel" if enc_k >= dec_k else "decode_kernel"
    achieved = enc_k_gbs if dom == "encode_kernel" else dec_k_gbs
    ratio = raw / nbytes
    saved_bits = 8 * (raw - nbytes)
    t_codec = (enc_avg + dec_avg) * 1e-3
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; shapes and distributions of the named workload)",
        "config": {"workload": describe(w), "raw_bytes_per_step_per_gpu": raw,
                   "stream_bytes": nbytes, "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"weak x{world}, no data-path collective"},
        "encode_GBps": round(raw / (enc_avg * 1e-3) / 1e9, 3),
        "decode_GBps": round(raw / (dec_avg * 1e-3) / 1e9, 3),
        "encode_ms": round(enc_avg, 4), "decode_ms": round(dec_avg, 4),
        "ratio": round(ratio, 4),
        "break_even_gbit_s": round(saved_bits / t_codec / 1e9, 1),
        "net_gain_ms": {"100Gbit": round((saved_bits / 100e9 - t_codec) * 1e3, 3),
                        "400Gbit": round((saved_bits / 400e9 - t_codec) * 1e3, 3)},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_kind": peak_kind, "traffic": traffic.get(dom) if traffic else None,
                     "algorithmic_bytes_per_launch": raw + pay,
                     "encode_kernel_ms": round(enc_k, 4), "decode_kernel_ms": round(dec_k, 4),
                     "encode_kernel_frac": round(enc_k_gbs / hbm, 4),
                     "decode_kernel_frac": round(dec_k_gbs / hbm, 4),
                     "compress_call_frac": round(enc_gbs / hbm, 4),
                     "decompress_call_frac": round(dec_gbs / hbm, 4)},
        "kernel_ms": {"compress": {"clear": round(kc[0], 4), "encode": round(kc[1], 4),
                                   "finish": round(kc[2], 4), "compaction": round(kc[3], 4)},
                      "decompress": {"clear": round(kd[0], 4), "meta_expand": round(kd[1], 4),
                                     "elim_decode": round(kd[2], 4),
                                     "decode": round(kd[3], 4)}},
        "gpu_launches": (9 if w.paged else 8) * K,  # per step: workspace clear, load plans
        # (paged pools), encode, finish, compaction
        # (returns at once unless code chunks are stored eliminated); status clear, meta
        # expansion, eliminated-chunk decode (returns at once unless the header flags such
        # chunks), decode
        "clocks": clk.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if unfused:
        line["unfused_baseline"] = unfused
    if per_config:
        line["per_config"] = per_config
    if world == 1 and args.cpu_budget > 0:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_budget)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
