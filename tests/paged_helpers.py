"""Shared test helpers: build NVFP4 caches for a workload on both sides.

GPU side: the library's writer fills a device cache. Oracle side: the C
oracle's writer fills a host cache holding only the sequences under test (a
compact block numbering), so sampled checks of the largest workloads stay
small. Both sides draw K/V/Q from the seeded generators in
``nvfp4_quantized_paged_append_b200.workloads``.
"""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_scalar(x: float, device="cuda") -> torch.Tensor:
    return torch.tensor([x], dtype=torch.float32, device=device)


def build_gpu_cache(w: wl.PagedWorkload, scales, device="cuda", sentinel: int | None = None,
                    fp8: bool = False):
    """Device HND cache written by the library's writer, token by sequence
    (fp8: an FP8-E4M3 cache)."""
    k_scale, v_scale, _ = scales
    alloc = nk.alloc_fp8_kv_cache if fp8 else nk.alloc_kv_cache
    cache = alloc(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, device)
    if sentinel is not None:
        cache.fill_(sentinel)
    ks, vs = dev_scalar(k_scale, device), dev_scalar(v_scale, device)
    for b in range(w.num_seqs):
        k, v = wl.seq_kv(w, b, device)
        slots = torch.from_numpy(w.slots_for_seq(b)).to(device)
        nk.quantize_append_paged(k, v, cache, slots, ks, vs, fp8=fp8)
    return cache


def oracle_case(w: wl.PagedWorkload, seqs, scales, device="cuda", rows=None, fp8=False):
    """Oracle inputs for the listed sequences: compact cache + block table.

    rows: optional {b: [query row indices]} for prefill sequences; each listed
    row becomes a one-query sequence ending at its absolute position (the
    same causal window), so single rows of long prefills can be checked.
    Returns dict with cache, block_table, seq_lens, qo_indptr, q (uint16), and
    out_index (list of (q token index in the full problem) per oracle row).
    """
    k_scale, v_scale, _ = scales
    qfull = u16(wl.queries(w, device))
    indptr = w.qo_indptr
    blocks = []
    for b in seqs:
        blocks += [int(x) for x in w.block_table[b, : -(-int(w.seq_lens[b]) // w.block_size)]]
    remap = {blk: i for i, blk in enumerate(dict.fromkeys(blocks))}
    nb = len(remap)
    row_bytes = w.head_size if fp8 else w.full_dim
    cache = np.zeros((nb, 2, w.num_kv_heads, w.block_size, row_bytes), np.uint8)
    writer = oracle.fp8kv_quantize_append_paged if fp8 else oracle.quantize_append_paged
    for b in seqs:
        k, v = wl.seq_kv(w, b, device)
        L = int(w.seq_lens[b])
        n = np.arange(L)
        loc = np.array([remap[int(x)] for x in w.block_table[b, n // w.block_size]], np.int64)
        slots = loc * w.block_size + n % w.block_size
        writer(u16(k), u16(v), cache, slots.astype(np.int64), k_scale, v_scale, w.block_size)
    tables, lens, qrows, out_index = [], [], [], []
    for b in seqs:
        L = int(w.seq_lens[b])
        qlen = int(w.q_lens[b])
        nblk = -(-L // w.block_size)
        t = [remap[int(x)] for x in w.block_table[b, :nblk]]
        sel = range(qlen) if rows is None or b not in rows else rows[b]
        for r in sel:
            pos = L - qlen + r
            tables.append(t)
            lens.append(pos + 1)
            tok = int(indptr[b]) + r
            qrows.append(qfull[tok])
            out_index.append(tok)
    width = max(len(t) for t in tables)
    bt = np.zeros((len(tables), width), np.int32)
    for i, t in enumerate(tables):
        bt[i, : len(t)] = t
    return dict(cache=cache, block_table=bt, seq_lens=np.array(lens, np.int32),
                q=np.ascontiguousarray(np.stack(qrows)), out_index=out_index, fp8=fp8)


def run_oracle(case, scales):
    k_scale, v_scale, o_scale = scales
    return oracle.paged_attention(case["q"], case["cache"], case["block_table"], case["seq_lens"],
                                  None, k_scale, v_scale, 0.0, o_scale,
                                  kv_format=oracle.KV_FP8 if case.get("fp8") else oracle.KV_NVFP4)


def run_gpu_attention(w: wl.PagedWorkload, cache, scales, device="cuda", q=None, fp8=False):
    k_scale, v_scale, o_scale = scales
    q = wl.queries(w, device) if q is None else q
    tq = q.shape[0]
    o8 = torch.empty((tq, w.num_q_heads, w.head_size), dtype=torch.uint8, device=device)
    o16 = torch.empty((tq, w.num_q_heads, w.head_size), dtype=torch.bfloat16, device=device)
    o32 = torch.empty((tq, w.num_q_heads, w.head_size), dtype=torch.float32, device=device)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, device)
    bt = torch.from_numpy(w.block_table).to(device)
    sl = torch.from_numpy(w.seq_lens).to(device)
    qo = None if w.is_decode else torch.from_numpy(w.qo_indptr).to(device)
    kvs = torch.tensor([k_scale, v_scale], dtype=torch.float32, device=device)
    nk.paged_attention(q, cache, bt, sl, kvs, o8, dev_scalar(o_scale, device), ws, qo_indptr=qo,
                       max_q_len=w.max_q_len, o_bf16=o16, o_f32=o32, fp8=fp8)
    torch.cuda.synchronize()
    return o8, o16, o32, ws


# ----------------------------------------------------------------- tolerances
REL_TOL = 2e-3  # per output row: max |o - o_ref| <= REL_TOL * max |o_ref|


def e4m3_ordinal(codes: np.ndarray) -> np.ndarray:
    """Signed position of an E4M3 code on the value ladder (+-0 -> 0)."""
    c = codes.astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def check_rows(o32_gpu: np.ndarray, o_ref: np.ndarray, tol=REL_TOL):
    """o arrays [rows][D]; asserts the per-row relative bound; returns worst ratio."""
    err = np.abs(o32_gpu.astype(np.float64) - o_ref).max(axis=-1)
    scale = np.abs(o_ref).max(axis=-1)
    scale = np.where(scale > 0, scale, 1.0)
    ratio = err / scale
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > tol:
        i = int(ratio.argmax())
        j = int(np.abs(o32_gpu[i].astype(np.float64) - o_ref[i]).argmax())
        bad = int((ratio > tol).sum())
        raise AssertionError(
            f"max per-row relative error {worst:.3e} > {tol} at row {i} (d={j}: gpu "
            f"{float(o32_gpu[i, j]):.6g} ref {float(o_ref[i, j]):.6g}, row max {scale[i]:.4g}); "
            f"{bad} of {ratio.size} rows over")
    return worst


def check_fp8(o8_gpu: np.ndarray, o8_ref: np.ndarray):
    d = np.abs(e4m3_ordinal(o8_gpu) - e4m3_ordinal(o8_ref))
    assert int(d.max()) <= 1, f"E4M3 outputs differ by {int(d.max())} steps"
    return int(d.max())


def check_bf16_from_fp8(o16_gpu: np.ndarray, o8_ref: np.ndarray, o_scale: float):
    """o_bf16 must be bf16(fl32(E4M3 * o_scale)) of a code within 1 step of the oracle's."""
    ok = np.zeros(o8_ref.shape, bool)
    ords = e4m3_ordinal(o8_ref)
    for delta in (-1, 0, 1):
        o = ords + delta
        for zero_sign in (0x00, 0x80):          # ordinal 0 is both +0 and -0
            code = np.where(o < 0, 0x80 | (-o), np.where(o == 0, zero_sign, o)).clip(0, 255)
            code = code.astype(np.uint8)
            code = np.where((code & 0x7F) == 0x7F, code - 1, code).astype(np.uint8)  # no NaN codes
            val = (torch.from_numpy(code).view(torch.float8_e4m3fn).float()
                   * torch.tensor(o_scale, dtype=torch.float32))
            ok |= u16(val.to(torch.bfloat16)) == o16_gpu
    assert ok.all(), f"{int((~ok).sum())} bf16 outputs are not the dequantized FP8 value"
