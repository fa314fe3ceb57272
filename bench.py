#!/usr/bin/env python3
"""Benchmark: NVFP4 paged decode step (quantize-append + paged attention).

Workload: the Qwen3-0.6B-shaped decode batch (16 q / 8 kv heads, head_size
128, block_size 16, 32 sequences with 512-4096 keys, N(0,1) K/V with 2% of
(head, channel) pairs x20, random block tables). One step is one launch of
the fused decode step: it quantizes and appends each sequence's new token (32
tokens) and runs decode attention over every sequence's keys (FP8 output +
bf16 dequant).

Timed region: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and torch.cuda.synchronize(); device time from CUDA
events on the launching stream, max over ranks. Inputs are rotated over
enough independent copies (cache, tables, queries) to exceed 4x the 126 MB L2,
so every step reads its KV from HBM.

value = algorithmic NVFP4 KV bytes read per step (sum over sequences of
seq_len * kv_heads * 2 * full_dim, no block padding) / step time, summed over
ranks (each rank runs its own replica: the path has no exchange step).

Also reported: roofline of the attention kernel (its own CUDA-event time per
launch), the quantize-append sweep (8192 tokens into a 65536 x 16 cache) in
Mtok/s, the long-context decode batch (64 x 32768 keys, 2.4 GB of KV) in KV
GB/s, the mixed chunked-prefill batch (8 x 2048 causal queries over 10240
keys plus 56 decode sequences, head_size 256, GQA 8) as the whole call and as
its prefill (TFLOP/s against the sustained bf16 tensor peak) and decode
sub-batches, the end-to-end number through host buffers, the CPU oracle
baseline and SM clocks sampled during each timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 paged decode attn KV GB/s (% of HBM peak); append Mtok/s"
WORKLOAD = "qwen3_0p6b_decode"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--profile", choices=["attention", "append", "step", "activation", "prefill",
                                          "prefill_qfp4"],
                   default=None,
                   help="kernel-only mode for profilers: set up, then launch the chosen "
                        "kernel --steps times (no timing, no JSON)")
    p.add_argument("--workload", default=WORKLOAD, help="workload for --profile attention")
    p.add_argument("--time-workloads", default=None,
                   help="comma-separated workload names (e.g. long_decode,mixed_prefill_decode):"
                        " time one attention call per workload, L2 flushed before each, and"
                        " print one JSON line each instead of the benchmark line")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peaks():
    """(burst, sustained) dense bf16 TFLOP/s and their kind."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            "measured"
    return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


# ------------------------------------------------------------------ distributed
def dist_init(n):
    import torch
    import torch.distributed as dist
    if n <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    from datetime import timedelta
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, dist.get_world_size(), dist


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(x, dist):
    """The largest x over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return x
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ms_local, steps, bytes_per_step, dist, world):
    """(ms per step, whole-job GB/s): every rank processes bytes_per_step per
    step (replicas, weak scaling) and the job takes its slowest rank's time."""
    ms_step = max_over_ranks(ms_local, dist) / steps
    return ms_step, world * bytes_per_step / (ms_step * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi SM clock + throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, region=0):
        """Clocks over the region between marks 2*region and 2*region + 1."""
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        if len(self.marks) >= 2 * region + 2:
            t0, t1 = self.marks[2 * region], self.marks[2 * region + 1]
        else:
            t0, t1 = 0, time.time()
        rows = [s for t, s in self.samples if t0 - 0.15 <= t <= t1 + 0.15] or \
               [s for _, s in self.samples[-5:]]
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------ our arm
KERNEL_SOURCES = {
    "decode_attention_kernel<128,16>": ["attention_decode.cu", "nvfp4kv_device.cuh",
                                        "nvfp4kv_launch.h"],
    "quantize_append_pair_kernel<128>": ["writer.cu", "nvfp4kv_device.cuh", "nvfp4kv_launch.h"],
}


def kernel_source_sha(kernel):
    """Hash of the source files that define a kernel (stale-profile check)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_quantized_paged_append_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes (read + write) per launch from the committed ncu summary
    (profiles/traffic.json), if it was taken on the current kernel sources;
    else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class DecodeState:
    """One independent copy of the step's device state. The step's host inputs
    (q, new k/v, slots, seq_lens, block table) live in one device staging
    buffer, so the end-to-end loop moves them with a single host-to-device
    copy per step."""

    def __init__(self, w, scales, hist_cache, device):
        import torch
        import nvfp4_quantized_paged_append_b200 as nk
        from nvfp4_quantized_paged_append_b200 import workloads as wl
        self.cache = hist_cache.clone()
        B, H, D = w.num_seqs, w.num_kv_heads, w.head_size
        # the new token of each sequence = its last position
        ks, vs = [], []
        for b in range(B):
            k, v = wl.seq_kv(w, b, device, start=int(w.seq_lens[b]) - 1)
            ks.append(k)
            vs.append(v)
        slots = torch.from_numpy(np.array(
            [w.slots_for_seq(b, int(w.seq_lens[b]) - 1)[0] for b in range(B)], np.int64))
        parts = [("q", wl.queries(w, device)), ("k_new", torch.cat(ks)), ("v_new", torch.cat(vs)),
                 ("slots", slots), ("sl", torch.from_numpy(w.seq_lens)),
                 ("bt", torch.from_numpy(w.block_table))]
        offs, total = [], 0
        for _, t in parts:
            offs.append(total)
            total += -(-t.numel() * t.element_size() // 256) * 256
        self.stage = torch.zeros(total, dtype=torch.uint8, device=device)
        for (name, t), off in zip(parts, offs):
            n = t.numel() * t.element_size()
            view = self.stage[off:off + n].view(t.dtype).view(t.shape)
            view.copy_(t)
            setattr(self, name, view)
        self.kvs = torch.tensor([scales[0], scales[1]], dtype=torch.float32, device=device)
        self.ks = self.kvs[0:1]
        self.vs = self.kvs[1:2]
        self.osc = torch.tensor([scales[2]], dtype=torch.float32, device=device)
        self.o8 = torch.empty((B, w.num_q_heads, D), dtype=torch.uint8, device=device)
        self.o16 = torch.empty((B, w.num_q_heads, D), dtype=torch.bfloat16, device=device)
        self.ws = nk.alloc_workspace(B, w.num_q_heads, H, D, device)

    def append(self, nk, stream=None):
        nk.quantize_append_paged(self.k_new, self.v_new, self.cache, self.slots, self.ks, self.vs,
                                 stream=stream)

    def attend(self, nk, stream=None, metadata_ready=False):
        nk.paged_attention(self.q, self.cache, self.bt, self.sl, self.kvs, self.o8, self.osc,
                           self.ws, o_bf16=self.o16, stream=stream, metadata_ready=metadata_ready)

    def step(self, nk, stream=None, metadata_ready=False, history_ready=False):
        """One decode step in one launch: append the new rows, attend."""
        nk.paged_decode_append(self.q, self.k_new, self.v_new, self.cache, self.bt, self.sl,
                               self.kvs, self.o8, self.osc, self.ws, o_bf16=self.o16,
                               stream=stream, metadata_ready=metadata_ready,
                               history_ready=history_ready)


def cudart():
    """The CUDA runtime library the process's torch uses (for per-step copies
    and events without Python tensor overhead)."""
    import ctypes
    import glob
    import torch
    cands = glob.glob(os.path.join(os.path.dirname(torch.__file__), "lib", "libcudart.so*"))
    try:
        import nvidia.cuda_runtime as ncr
        for d in ncr.__path__:
            cands += glob.glob(os.path.join(d, "lib", "libcudart.so*"))
    except ImportError:
        pass
    if not cands:
        raise RuntimeError("libcudart not found next to torch")
    return ctypes.CDLL(sorted(cands)[0])


def build_cache(w, scales, dev):
    """The workload's whole cache, written by the library's writer."""
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    cache = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
    ks = torch.tensor([scales[0]], dtype=torch.float32, device=dev)
    vs = torch.tensor([scales[1]], dtype=torch.float32, device=dev)
    for b in range(w.num_seqs):
        k, v = wl.seq_kv(w, b, dev)
        nk.quantize_append_paged(k, v, cache, torch.from_numpy(w.slots_for_seq(b)).to(dev), ks, vs)
    return cache


class AttentionCall:
    """Device inputs/outputs of one attention call over a workload (or a
    sub-batch of one, sharing its cache)."""

    def __init__(self, w, cache, q, scales, dev):
        import torch
        import nvfp4_quantized_paged_append_b200 as nk
        self.nk, self.w, self.cache, self.q = nk, w, cache, q
        self.bt = torch.from_numpy(w.block_table).to(dev)
        self.sl = torch.from_numpy(w.seq_lens).to(dev)
        self.qo = None if w.is_decode else torch.from_numpy(w.qo_indptr).to(dev)
        self.kvs = torch.tensor([scales[0], scales[1]], dtype=torch.float32, device=dev)
        self.osc = torch.tensor([scales[2]], dtype=torch.float32, device=dev)
        shape = (w.num_q_tokens, w.num_q_heads, w.head_size)
        self.o8 = torch.empty(shape, dtype=torch.uint8, device=dev)
        self.o16 = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, dev)

    q_fp4 = False  # prefill rows on the block-scaled path with NVFP4 queries

    def __call__(self, stream):
        self.nk.paged_attention(self.q, self.cache, self.bt, self.sl, self.kvs, self.o8, self.osc,
                                self.ws, qo_indptr=self.qo, max_q_len=self.w.max_q_len,
                                o_bf16=self.o16, stream=stream, q_fp4=self.q_fp4)


def time_calls(fn, n, stream, warm=3):
    """Mean milliseconds per call of n back-to-back calls on `stream`
    (CUDA events on that stream), after `warm` untimed calls."""
    import torch
    for _ in range(warm):
        fn(stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    e0.record(stream)
    for _ in range(n):
        fn(stream)
    e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / n


def long_decode_record(stream, clocks, region, n_calls=20):
    """Long-context decode (64 sequences x 32768 keys, 32 q / 8 kv heads,
    head_size 128, block_size 32; 2.4 GB of NVFP4 KV, far above L2): n
    back-to-back attention calls."""
    import torch
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    w = wl.make_workload("long_decode")
    scales = wl.global_scales(w, dev)
    cache = build_cache(w, scales, dev)
    call = AttentionCall(w, cache, wl.queries(w, dev), scales, dev)
    time_calls(call, 3, stream, warm=2)
    clocks.mark()
    ms = time_calls(call, n_calls, stream)
    clocks.mark()
    peak, kind = peaks()
    gbs = w.kv_bytes() / (ms * 1e-3) / 1e9
    rec = {"workload": "long_decode", "kernel": "decode_attention_kernel<128,32>",
           "calls": n_calls, "kernel_ms": round(ms, 5), "kv_bytes": w.kv_bytes(),
           "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "peak": peak,
           "peak_kind": f"{kind} HBM copy", "frac_of_8TBps": round(gbs / 8000.0, 4),
           "l2": "2.4 GB of KV per call (> 19x L2)", "clocks": clocks.summary(region)}
    del cache, call
    torch.cuda.empty_cache()
    return rec


def mixed_record(stream, clocks, region, n_prefill=5, n_decode=20):
    """Mixed chunked prefill + decode (64 q / 8 kv heads, head_size 256,
    block_size 16; 8 sequences prefilling 2048 causal queries over 8192 cached
    keys, 56 decode sequences of 1024-16384 keys). Timed as the whole mixed
    call, and as its prefill and decode sub-batches alone (same cache)."""
    import torch
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    w = wl.make_workload("mixed_prefill_decode")
    scales = wl.global_scales(w, dev)
    cache = build_cache(w, scales, dev)
    q = wl.queries(w, dev)
    pre_seqs = [b for b in range(w.num_seqs) if w.q_lens[b] > 1]
    dec_seqs = [b for b in range(w.num_seqs) if w.q_lens[b] == 1]
    wp, tp = w.subset(pre_seqs)
    wd, td = w.subset(dec_seqs)
    full = AttentionCall(w, cache, q, scales, dev)
    pre = AttentionCall(wp, cache, q[torch.from_numpy(tp).to(dev)].contiguous(), scales, dev)
    dec = AttentionCall(wd, cache, q[torch.from_numpy(td).to(dev)].contiguous(), scales, dev)
    time_calls(full, 1, stream, warm=1)
    clocks.mark()
    ms_full = time_calls(full, n_prefill, stream)
    ms_pre = time_calls(pre, n_prefill, stream)
    ms_dec = time_calls(dec, n_decode, stream)
    pre.q_fp4 = True  # the same prefill with NVFP4 queries (block-scaled QK^T)
    ms_pre4 = time_calls(pre, n_prefill, stream)
    pre.q_fp4 = False
    clocks.mark()
    burst, sustained, tkind = tensor_peaks()
    peak, kind = peaks()
    flops = w.prefill_flops()
    tf = flops / (ms_pre * 1e-3) / 1e12
    dgbs = wd.kv_bytes() / (ms_dec * 1e-3) / 1e9
    rec = {"workload": "mixed_prefill_decode",
           "call_ms": round(ms_full, 4),
           "call_tflops_prefill_over_call": round(flops / (ms_full * 1e-3) / 1e12, 1),
           "prefill": {"kernel": "prefill attention (8 seqs x 2048 causal queries over 10240 keys)",
                       "ms": round(ms_pre, 4), "flops": flops, "tflops": round(tf, 1),
                       "peak": sustained, "unit": "TFLOP/s",
                       "peak_kind": f"{tkind} dense bf16, sustained (seconds-long loop)",
                       "frac": round(tf / sustained, 4),
                       "frac_of_burst": round(tf / burst, 4),
                       "prefill_kv_bytes": wp.kv_bytes()},
           "prefill_qfp4": {"kernel": "the same prefill with NVFP4 queries (NVFP4_ATTN_QFP4: "
                                      "q K^T on tcgen05 kind::mxf4nvf4; changes the results)",
                            "ms": round(ms_pre4, 4),
                            "tflops": round(flops / (ms_pre4 * 1e-3) / 1e12, 1),
                            "frac": round(flops / (ms_pre4 * 1e-3) / 1e12 / sustained, 4)},
           "decode": {"kernel": "decode_attention_kernel<256,16>", "ms": round(ms_dec, 5),
                      "kv_bytes": wd.kv_bytes(), "gbs": round(dgbs, 1),
                      "frac": round(dgbs / peak, 4), "peak": peak,
                      "peak_kind": f"{kind} HBM copy"},
           "timing": f"back-to-back calls: {n_prefill} mixed, {n_prefill} prefill-only, "
                     f"{n_decode} decode-only, {n_prefill} prefill-only with NVFP4 queries "
                     f"(CUDA events on the launching stream)",
           "clocks": clocks.summary(region)}
    del cache, full, pre, dec
    torch.cuda.empty_cache()
    return rec


def fp8_kv_record(stream, clocks, region, nvfp4_attn_ms, n_calls=500):
    """The same decode batch (qwen3_0p6b_decode) over an FP8-E4M3 KV cache:
    the pages' comparison format (NVFP4 vs FP8 KV TPOT). Decode attention
    calls back to back over rotated cache copies (> 4x L2)."""
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    w = wl.make_workload(WORKLOAD)
    scales = wl.global_scales(w, dev)
    cache = nk.alloc_fp8_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
    ks = torch.tensor([scales[0]], dtype=torch.float32, device=dev)
    vs = torch.tensor([scales[1]], dtype=torch.float32, device=dev)
    for b in range(w.num_seqs):
        k, v = wl.seq_kv(w, b, dev)
        nk.quantize_append_paged(k, v, cache, torch.from_numpy(w.slots_for_seq(b)).to(dev), ks, vs,
                                 fp8=True)
    copies = max(2, -(-4 * L2_BYTES // cache.numel()) + 1)
    caches = [cache] + [cache.clone() for _ in range(copies - 1)]
    q = wl.queries(w, dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    kvs = torch.tensor([scales[0], scales[1]], dtype=torch.float32, device=dev)
    osc = torch.tensor([scales[2]], dtype=torch.float32, device=dev)
    o8 = torch.empty((w.num_seqs, w.num_q_heads, w.head_size), dtype=torch.uint8, device=dev)
    o16 = torch.empty_like(o8, dtype=torch.bfloat16)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, dev)
    it = [0]

    def once(s):
        nk.paged_attention(q, caches[it[0] % copies], bt, sl, kvs, o8, osc, ws, o_bf16=o16,
                           stream=s, fp8=True)
        it[0] += 1

    time_calls(once, 3, stream, warm=5)
    clocks.mark()
    ms = time_calls(once, n_calls, stream)
    clocks.mark()
    kvb = int(w.seq_lens.astype(np.int64).sum()) * w.num_kv_heads * 2 * w.head_size
    peak, kind = peaks()
    gbs = kvb / (ms * 1e-3) / 1e9
    rec = {"workload": f"{WORKLOAD} over an FP8-E4M3 KV cache",
           "kernel": "decode_attention_kernel<128,16,fp8>", "calls": n_calls,
           "kernel_ms": round(ms, 5), "kv_bytes": kvb, "gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": f"{kind} HBM copy",
           "nvfp4_kernel_ms": round(nvfp4_attn_ms, 5),
           "fp8_over_nvfp4_time": round(ms / nvfp4_attn_ms, 3),
           "l2": f"rotated over {copies} cache copies", "clocks": clocks.summary(region)}
    del caches, cache
    torch.cuda.empty_cache()
    return rec


def activation_record(stream, clocks, region, n_calls=200):
    """Activation NVFP4 quantizer with swizzled scales on an 8192 x 4096 bf16
    activation (a Qwen3-8B-sized hidden state for 8192 tokens), N(0,1) with 2%
    of channels x20; inputs rotated over 4 copies (256 MiB > L2)."""
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    dev = torch.device("cuda", torch.cuda.current_device())
    rows, cols = 8192, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(8)
    x = torch.randn((rows, cols), generator=g, device=dev, dtype=torch.float32)
    x[:, torch.randperm(cols, generator=g, device=dev)[: cols // 50]] *= 20.0
    x = x.to(torch.bfloat16)
    inv = torch.tensor([6.0 * 448.0 / float(x.float().abs().amax())], dtype=torch.float32,
                       device=dev)
    xs = [x.clone() for _ in range(4)]
    fp4 = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    sf = torch.empty(nk.activation_sf_bytes(rows, cols, True), dtype=torch.uint8, device=dev)
    it = [0]

    def once(s):
        nk.quantize_activation(xs[it[0] % 4], inv, True, fp4, sf, stream=s)
        it[0] += 1

    time_calls(once, 3, stream, warm=3)
    clocks.mark()
    ms = time_calls(once, n_calls, stream)
    clocks.mark()
    nbytes = rows * cols * 2 + rows * cols // 2 + sf.numel()
    peak, kind = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    rec = {"workload": "activation 8192 x 4096 bf16 -> NVFP4, swizzled scales",
           "kernel": "quantize_activation_kernel<true>", "calls": n_calls,
           "kernel_ms": round(ms, 5), "bytes": nbytes,
           "mtok_s": round(rows / (ms * 1e-3) / 1e6, 1), "gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": f"{kind} HBM copy",
           "clocks": clocks.summary(region)}
    del xs, x, fp4, sf
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world, dist):
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.cuda.set_device(dev)
    nk.lib()

    w = wl.make_workload(WORKLOAD)
    scales = wl.global_scales(w, dev)
    kv_bytes = w.kv_bytes()
    # history: every token but the last, written once by the library's writer
    hist = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
    ksd = torch.tensor([scales[0]], dtype=torch.float32, device=dev)
    vsd = torch.tensor([scales[1]], dtype=torch.float32, device=dev)
    for b in range(w.num_seqs):
        L = int(w.seq_lens[b])
        k, v = wl.seq_kv(w, b, dev, stop=L - 1)
        nk.quantize_append_paged(k, v, hist, torch.from_numpy(w.slots_for_seq(b, 0, L - 1)).to(dev),
                                 ksd, vsd)
    cache_bytes = hist.numel()
    copies = max(2, -(-4 * L2_BYTES // cache_bytes) + 1)
    states = [DecodeState(w, scales, hist, dev) for _ in range(copies)]
    del hist
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    for st in states:  # eager run of every copy before capture (first calls are eager)
        st.step(nk, stream)
        st.append(nk, stream)
        st.attend(nk, stream)
    stream.synchronize()
    # Per buffer copy: one CUDA graph for the step (the fused append + decode
    # attention kernel, launched as a programmatic dependent of the previous
    # step's kernel; its block tables and lengths are step inputs no kernel
    # writes, so it reads them while that kernel finishes), one for the same
    # step as two kernels (writer, then attention) and one for the attention
    # kernel alone.
    g_step, g_two, g_att = [], [], []
    # one round of steps (one per buffer copy) in one graph: each step's kernel is
    # a programmatic dependent of the one before, which writes neither its
    # metadata nor its cache (another copy's), so it reads its metadata and
    # starts its first page copies while that kernel finishes (q only after
    # that kernel has completed), as after the projection kernel of a model
    g_round = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_round, stream=stream):
        for st in states:
            st.step(nk, stream, history_ready=True)
    for st in states:
        ga = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ga, stream=stream):
            st.step(nk, stream, metadata_ready=True)
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            st.append(nk, stream)
            st.attend(nk, stream, metadata_ready=True)
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb, stream=stream):
            st.attend(nk, stream)
        g_step.append(ga)
        g_two.append(g2)
        g_att.append(gb)

    def run_steps(n):
        for _ in range(n // copies):
            g_round.replay()
        for j in range(n % copies):
            g_step[j].replay()

    def run_graphs(graphs, n):
        for j in range(n):
            graphs[j % copies].replay()

    def run_attention(n):
        run_graphs(g_att, n)

    run_steps(max(3, args.warmup))
    stream.synchronize()

    clocks = ClockSampler(dev.index)
    clocks.start()
    # keep the GPU under the same load ~1.5 s before the timed region so the
    # sampled clocks are the loaded ones (extra warm-up, not timed)
    t_end = time.time() + 1.5
    while time.time() < t_end:
        run_steps(200)
        stream.synchronize()
    barrier(dist)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clocks.mark()
    e0.record(stream)
    run_steps(args.steps)
    e1.record(stream)
    stream.synchronize()
    clocks.mark()
    torch.cuda.synchronize()
    barrier(dist)
    ms_local = e0.elapsed_time(e1)
    ms_step, value = job_throughput(ms_local, args.steps, kv_bytes, dist, world)
    # the attention kernel's own average duration: the same number of
    # attention-only launches back to back on the launching stream
    run_attention(max(3, args.warmup))
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    run_attention(args.steps)
    a1.record(stream)
    stream.synchronize()
    attn_ms = a0.elapsed_time(a1) / args.steps
    # one graph per step (no overlap between consecutive steps), for comparison
    run_graphs(g_step, max(3, args.warmup))
    a0.record(stream)
    run_graphs(g_step, args.steps)
    a1.record(stream)
    stream.synchronize()
    single_ms = a0.elapsed_time(a1) / args.steps
    # the same step as two kernels (writer, then attention), for comparison
    run_graphs(g_two, max(3, args.warmup))
    a0.record(stream)
    run_graphs(g_two, args.steps)
    a1.record(stream)
    stream.synchronize()
    two_ms = a0.elapsed_time(a1) / args.steps

    # ---- quantize-append sweep (8192 tokens) for Mtok/s
    app = wl.make_append()
    ka, va = app.kv(dev)
    gka, gva = app.scales(ka, va)
    slots = torch.from_numpy(app.slot_mapping()).to(dev)
    acache = nk.alloc_kv_cache(app.num_blocks, app.block_size, app.num_kv_heads, app.head_size, dev)
    ksa = torch.tensor([gka], dtype=torch.float32, device=dev)
    vsa = torch.tensor([gva], dtype=torch.float32, device=dev)
    # rotate input copies so reads come from HBM (each copy ~32 MB of bf16)
    acopies = max(2, -(-4 * L2_BYTES // (ka.numel() * 4)) + 1)
    kas = [ka.clone() for _ in range(acopies)]
    vas = [va.clone() for _ in range(acopies)]
    nrep = 400
    it = [0]

    def append_once(s):
        i = it[0]
        it[0] += 1
        nk.quantize_append_paged(kas[i % acopies], vas[i % acopies], acache, slots, ksa, vsa,
                                 stream=s)

    # launched one call at a time from Python (host-bound near 12 us per call)
    app_calls_ms = time_calls(append_once, nrep, stream, warm=20)
    # the kernel back to back: one graph launches the writer once per input copy
    g_app = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app, stream=stream):
        for i in range(acopies):
            nk.quantize_append_paged(kas[i], vas[i], acache, slots, ksa, vsa, stream=stream)
    for _ in range(3):
        g_app.replay()
    app_reps = max(1, nrep // acopies)
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    b0.record(stream)
    for _ in range(app_reps):
        g_app.replay()
    b1.record(stream)
    stream.synchronize()
    app_ms = b0.elapsed_time(b1) / (app_reps * acopies)
    app_bytes = app.algorithmic_bytes()
    del g_app, kas, vas, acache
    torch.cuda.empty_cache()

    # ---- end to end through host buffers (pinned), every step: one H2D copy
    # of the packed step inputs (q, new k/v, slots, seq_lens, block table),
    # the fused step through the C ABI, and a D2H copy of the bf16 output. The
    # H2D copies run on one stream, the steps on the compute stream and the
    # D2H copies on a third, chained by events per buffer copy, so the copies
    # of one step overlap the compute of its neighbours.
    import ctypes
    host_stage = states[0].stage.cpu().pin_memory()
    host_outs = [torch.empty_like(st.o16, device="cpu").pin_memory() for st in states]
    h2d = host_stage.numel()
    d2h = host_outs[0].numel() * host_outs[0].element_size()
    up_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    lib = nk.lib()

    def p(t):
        return ctypes.c_void_p(t.data_ptr())

    cargs = []
    for st in states:
        B, H, D = w.num_seqs, w.num_kv_heads, w.head_size
        cargs.append((p(st.q), st.q.stride(0), w.num_q_heads, p(st.k_new), p(st.v_new),
                     st.k_new.stride(0), st.v_new.stride(0), p(st.cache), w.num_blocks,
                     w.block_size, H, D, p(st.bt), w.max_blocks_per_seq, p(st.sl), B,
                     p(st.kvs), ctypes.c_float(0.0), p(st.o8), p(st.osc), p(st.o16), None,
                     p(st.ws), st.ws.numel(),
                     nk.NVFP4_ATTN_METADATA_READY | nk.NVFP4_ATTN_HISTORY_READY,
                     ctypes.c_void_p(stream.cuda_stream)))
    # the per-step copies and stream/event plumbing go straight to the CUDA
    # runtime (a Python tensor copy or event costs more host time than the step)
    rt = cudart()
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    rt.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
    rt.cudaEventRecord.argtypes = [vp, vp]
    rt.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
    rt.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
    rt.cudaEventDestroy.argtypes = [vp]

    def new_event():
        ev = vp()
        if rt.cudaEventCreateWithFlags(ctypes.byref(ev), 2) != 0:  # timing disabled
            raise RuntimeError("cudaEventCreateWithFlags failed")
        return ev

    h2d_done = [new_event() for _ in states]
    step_done = [new_event() for _ in states]
    d2h_done = [new_event() for _ in states]
    s_up, s_down, s_main = (vp(x.cuda_stream) for x in (up_stream, down_stream, stream))
    h_stage = vp(host_stage.data_ptr())
    d_stage = [vp(st.stage.data_ptr()) for st in states]
    h_out = [vp(t.data_ptr()) for t in host_outs]
    d_out = [vp(st.o16.data_ptr()) for st in states]
    e2e_steps = max(50, min(500, args.steps))
    stream.synchronize()
    for it_ in range(e2e_steps + 10):
        if it_ == 10:
            torch.cuda.synchronize()
            barrier(dist)
            x0 = torch.cuda.Event(enable_timing=True)
            x0.record(stream)
        j = it_ % copies
        if it_ >= copies:  # the copy's previous result has left the device
            rt.cudaStreamWaitEvent(s_up, d2h_done[j], 0)
        rt.cudaMemcpyAsync(d_stage[j], h_stage, h2d, 1, s_up)
        rt.cudaEventRecord(h2d_done[j], s_up)
        rt.cudaStreamWaitEvent(s_main, h2d_done[j], 0)
        st_ = lib.nvfp4_paged_decode_append(*cargs[j])
        if st_ != 0:
            raise RuntimeError(f"nvfp4_paged_decode_append: {st_}")
        rt.cudaEventRecord(step_done[j], s_main)
        rt.cudaStreamWaitEvent(s_down, step_done[j], 0)
        rt.cudaMemcpyAsync(h_out[j], d_out[j], d2h, 2, s_down)
        rt.cudaEventRecord(d2h_done[j], s_down)
    stream.wait_stream(down_stream)
    x1 = torch.cuda.Event(enable_timing=True)
    x1.record(stream)
    stream.synchronize()
    for ev in h2d_done + step_done + d2h_done:
        rt.cudaEventDestroy(ev)
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / e2e_steps, dist)
    del g_round, g_step, g_two, g_att, states
    torch.cuda.empty_cache()

    # ---- the other configurations' kernels: long-context decode and the
    # mixed chunked-prefill batch
    long_rec = long_decode_record(stream, clocks, 1)
    mixed_rec = mixed_record(stream, clocks, 2)
    act_rec = activation_record(stream, clocks, 3)
    fp8_rec = fp8_kv_record(stream, clocks, 4, attn_ms)
    clocks.stop()

    peak, peak_kind = peaks()
    # the step is one kernel (fused append + decode attention): its duration is
    # the step time; algorithmic bytes = the KV rows read + the new bf16 rows
    # read + the new NVFP4 rows written
    new_rows = w.num_seqs * w.num_kv_heads * 2 * (2 * w.head_size + w.full_dim)
    step_bytes = kv_bytes + new_rows
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    traffic = profiled_traffic("decode_attention_kernel<128,16>", WORKLOAD)
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1+e4m3) kv, bf16 q, f16 mma, fp32 accum, e4m3 out",
        "data": "synthetic (seeded N(0,1) K/V/Q, 2% outlier channels x20)",
        "config": {
            "workload": WORKLOAD, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_size": w.head_size,
            "block_size": w.block_size, "ctx_lens": "uniform 512-4096 (seeded)",
            "kv_bytes_per_step": kv_bytes, "new_tokens_per_step": w.num_seqs,
            "l2": f"inputs rotated over {copies} copies ({copies * cache_bytes / 2**20:.0f} MiB of cache) > 4x L2",
            "parallelism": f"replicas x{world} (independent shards, no collective)",
            "step": "one launch: quantize-append of the 32 new tokens fused into decode "
                    "attention (nvfp4_paged_decode_append); graphs of one step per buffer "
                    "copy, each launch a programmatic dependent of the previous",
        },
        "roofline": {
            "bound": "hbm", "kernel": "decode_attention_kernel<128,16> (fused append)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} HBM copy",
            "traffic": traffic, "algorithmic_bytes_per_launch": step_bytes,
            "kernel_ms": round(ms_step, 6),
            "frac_of_8TBps": round(achieved / 8000.0, 4),
            "attention_only_ms": round(attn_ms, 6),
            "attention_only_frac": round(kv_bytes / (attn_ms * 1e-3) / 1e9 / peak, 4),
            "two_kernel_step_ms": round(two_ms, 6),
            "one_graph_per_step_ms": round(single_ms, 6),
        },
        "append": {
            "workload": "append_sweep", "tokens": app.num_tokens, "live_tokens": app.live_tokens(),
            "timing": f"graphs of {acopies} back-to-back launches over rotated input copies",
            "ms": round(app_ms, 5), "mtok_s": round(app.num_tokens / (app_ms * 1e-3) / 1e6, 1),
            "host_launched_ms": round(app_calls_ms, 5),
            "gbs": round(app_bytes / (app_ms * 1e-3) / 1e9, 1),
            "frac": round(app_bytes / (app_ms * 1e-3) / 1e9 / peak, 4),
            "algorithmic_bytes": app_bytes,
            "traffic": profiled_traffic("quantize_append_pair_kernel<128>", "append_sweep"),
        },
        "long_decode": long_rec,
        "mixed_prefill_decode": mixed_rec,
        "activation_quant": act_rec,
        "fp8_kv_decode": fp8_rec,
        "e2e": {
            "value": round(world * kv_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(e2e_ms, 5),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "copies_per_step": "1 H2D (packed inputs) + 1 D2H, on their own streams, "
                               "overlapping neighbouring steps",
        },
        # timed region: one fused append + decode attention launch per step
        "gpu_launches": args.steps,
        "clocks": clocks.summary(0),
    }
    return result


# ------------------------------------------------------------------ CPU oracle
def oracle_sample_gbs(w, seqs, scales, budget_s=15.0):
    """Time the CPU oracle on a bounded sample of the workload; KV GB/s."""
    import torch
    import oracle
    from nvfp4_quantized_paged_append_b200 import workloads as wl

    def u16(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    q = u16(wl.queries(w, "cpu"))
    blocks = {}
    for b in seqs:
        for x in w.block_table[b, : -(-int(w.seq_lens[b]) // w.block_size)]:
            blocks.setdefault(int(x), len(blocks))
    cache = np.zeros((len(blocks), 2, w.num_kv_heads, w.block_size, w.full_dim), np.uint8)
    bt = np.zeros((len(seqs), w.max_blocks_per_seq), np.int32)
    for i, b in enumerate(seqs):
        L = int(w.seq_lens[b])
        k, v = wl.seq_kv(w, b, "cpu")
        n = np.arange(L)
        loc = np.array([blocks[int(x)] for x in w.block_table[b, n // w.block_size]], np.int64)
        oracle.quantize_append_paged(u16(k), u16(v), cache, loc * w.block_size + n % w.block_size,
                                     scales[0], scales[1], w.block_size)
        nblk = -(-L // w.block_size)
        bt[i, :nblk] = [blocks[int(x)] for x in w.block_table[b, :nblk]]
    sl = np.array([w.seq_lens[b] for b in seqs], np.int32)
    qs = np.ascontiguousarray(q[list(seqs)])
    kvb = int(sl.astype(np.int64).sum()) * w.num_kv_heads * 2 * w.full_dim
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.paged_attention(qs, cache, bt, sl, None, scales[0], scales[1], 0.0, scales[2])
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 50:
            break
    dt = (time.perf_counter() - t0) / reps
    return kvb / dt / 1e9, dt, kvb


def cpu_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else os.cpu_count()


def run_reference(args, rank, world):
    """The oracle (CPU, as it stands) on the same workload and metric: exactly
    --steps timed steps after --warmup untimed ones, each step the oracle's
    attention over a bounded sample of the workload's sequences, sized so the
    whole run stays within a few minutes."""
    if rank != 0:
        return None
    import oracle
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    oracle.build()
    w = wl.make_workload(WORKLOAD)
    scales = wl.global_scales(w, "cpu")
    seqs = [0, 1]
    _, dt0, _ = oracle_sample_gbs(w, seqs, scales, budget_s=0.0)  # sizing probe, untimed
    if dt0 * args.steps > 180.0:
        seqs = [0]
    sample = f"oracle attention on sequences {seqs} of {w.num_seqs} per step"
    t_warm = time.perf_counter()
    for _ in range(args.warmup):
        oracle_sample_gbs(w, seqs, scales, budget_s=0.0)
        if time.perf_counter() - t_warm > 20.0:
            break
    total_t, total_b = 0.0, 0
    for _ in range(args.steps):
        _, dt, kvb = oracle_sample_gbs(w, seqs, scales, budget_s=0.0)
        total_t += dt
        total_b += kvb
    value = total_b / total_t / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_workload_times(args):
    """One attention call per named workload (its own cache, filled by the
    writer), after a 256 MiB write that evicts L2; median of 10 event-timed
    calls after 2 warm-ups. KV GB/s counts the K+V rows the call must read;
    for multi-token query ranges the causal prefill FLOPs are reported too
    (the call's time covers both the decode and the prefill kernel)."""
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    peak, peak_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for name in args.time_workloads.split(","):
        w = wl.make_workload(name.strip())
        scales = wl.global_scales(w, dev)
        cache = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
        ks = torch.tensor([scales[0]], device=dev)
        vs = torch.tensor([scales[1]], device=dev)
        for b in range(w.num_seqs):
            k, v = wl.seq_kv(w, b, dev)
            nk.quantize_append_paged(k, v, cache, torch.from_numpy(w.slots_for_seq(b)).to(dev),
                                     ks, vs)
        q = wl.queries(w, dev)
        o8 = torch.empty((w.num_q_tokens, w.num_q_heads, w.head_size), dtype=torch.uint8,
                         device=dev)
        ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, dev)
        bt = torch.from_numpy(w.block_table).to(dev)
        sl = torch.from_numpy(w.seq_lens).to(dev)
        qo = None if w.is_decode else torch.from_numpy(w.qo_indptr).to(dev)
        kvs = torch.tensor([scales[0], scales[1]], device=dev)
        osc = torch.tensor([scales[2]], device=dev)
        times = []
        for i in range(12):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            nk.paged_attention(q, cache, bt, sl, kvs, o8, osc, ws, qo_indptr=qo,
                               max_q_len=w.max_q_len)
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                times.append(e0.elapsed_time(e1) * 1e3)
        us = statistics.median(times)
        gbs = w.kv_bytes() / (us * 1e-6) / 1e9
        line = {"workload": name.strip(), "call_us": round(us, 2), "kv_bytes": w.kv_bytes(),
                "kv_gbs": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peak, 4),
                "frac_of_8TBps": round(gbs / 8000.0, 4), "peak_kind": peak_kind,
                "timing": "median of 10 single calls, L2 evicted before each"}
        flops = w.prefill_flops()
        if flops:
            line["prefill_flops"] = flops
            line["prefill_tflops_over_call"] = round(flops / (us * 1e-6) / 1e12, 1)
        print(json.dumps(line), flush=True)
        del cache, ws
        torch.cuda.empty_cache()


def run_profile(args):
    """Set up one workload and launch one kernel --steps times (for ncu)."""
    import torch
    import nvfp4_quantized_paged_append_b200 as nk
    from nvfp4_quantized_paged_append_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    if args.profile == "step":
        w = wl.make_workload(WORKLOAD)
        scales = wl.global_scales(w, dev)
        hist = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
        ks = torch.tensor([scales[0]], device=dev)
        vs = torch.tensor([scales[1]], device=dev)
        for b in range(w.num_seqs):
            L = int(w.seq_lens[b])
            k, v = wl.seq_kv(w, b, dev, stop=L - 1)
            nk.quantize_append_paged(k, v, hist,
                                     torch.from_numpy(w.slots_for_seq(b, 0, L - 1)).to(dev), ks, vs)
        st = DecodeState(w, scales, hist, dev)
        for _ in range(args.steps):
            st.step(nk)
        torch.cuda.synchronize()
        print(f"profile mode: step x{args.steps} done", flush=True)
        return
    if args.profile == "activation":
        rows, cols = 8192, 4096
        x = torch.randn((rows, cols), device=dev).to(torch.bfloat16)
        inv = torch.tensor([6.0 * 448.0 / float(x.float().abs().amax())], device=dev)
        for _ in range(args.steps):
            nk.quantize_activation(x, inv, True)
        torch.cuda.synchronize()
        print(f"profile mode: activation x{args.steps} done", flush=True)
        return
    if args.profile == "append":
        app = wl.make_append()
        k, v = app.kv(dev)
        gk, gv = app.scales(k, v)
        slots = torch.from_numpy(app.slot_mapping()).to(dev)
        cache = nk.alloc_kv_cache(app.num_blocks, app.block_size, app.num_kv_heads,
                                  app.head_size, dev)
        ks = torch.tensor([gk], device=dev)
        vs = torch.tensor([gv], device=dev)
        for _ in range(args.steps):
            nk.quantize_append_paged(k, v, cache, slots, ks, vs)
    else:
        if args.profile in ("prefill", "prefill_qfp4"):
            # a small chunked-prefill batch with the mixed batch's shapes: 2
            # sequences of 512 causal queries over 2560 keys, 64 q / 8 kv heads,
            # head size 256, block size 16 (512 CTAs)
            w = wl.custom_workload("prefill_small", 11, 64, 8, 256, 16, [2560, 2560],
                                   [512, 512], outliers="x20")
        else:
            w = wl.make_workload(args.workload)
        scales = wl.global_scales(w, dev)
        cache = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, dev)
        ks = torch.tensor([scales[0]], device=dev)
        vs = torch.tensor([scales[1]], device=dev)
        for b in range(w.num_seqs):
            k, v = wl.seq_kv(w, b, dev)
            nk.quantize_append_paged(k, v, cache, torch.from_numpy(w.slots_for_seq(b)).to(dev),
                                     ks, vs)
        q = wl.queries(w, dev)
        o8 = torch.empty((w.num_q_tokens, w.num_q_heads, w.head_size), dtype=torch.uint8,
                         device=dev)
        ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, dev)
        bt = torch.from_numpy(w.block_table).to(dev)
        sl = torch.from_numpy(w.seq_lens).to(dev)
        qo = None if w.is_decode else torch.from_numpy(w.qo_indptr).to(dev)
        kvs = torch.tensor([scales[0], scales[1]], device=dev)
        osc = torch.tensor([scales[2]], device=dev)
        for _ in range(args.steps):
            nk.paged_attention(q, cache, bt, sl, kvs, o8, osc, ws, qo_indptr=qo,
                               max_q_len=w.max_q_len, q_fp4=args.profile == "prefill_qfp4")
    torch.cuda.synchronize()
    print(f"profile mode: {args.profile} x{args.steps} done", flush=True)


def main():
    args = parse()
    if args.profile:
        run_profile(args)
        return
    if args.time_workloads:
        run_workload_times(args)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, dist = dist_init(args.gpus)
    res = run_ours(args, rank, world, dist)
    if rank == 0 and not args.no_cpu_baseline:
        # bounded CPU oracle sample (rank 0, 1 GPU only)
        if world == 1:
            from nvfp4_quantized_paged_append_b200 import workloads as wl
            import oracle
            oracle.build()
            w = wl.make_workload(WORKLOAD)
            scales = wl.global_scales(w, "cpu")
            gbs, dt, kvb = oracle_sample_gbs(w, [0, 1], scales, budget_s=10.0)
            res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_threads(),
                                   "kind": "oracle",
                                   "sample": f"oracle attention, sequences 0-1 of {w.num_seqs} "
                                             f"({kvb} KV bytes), repeated for ~10 s"}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
