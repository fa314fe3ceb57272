"""NVFP4 queries in the chunked prefill (NVFP4_ATTN_QFP4): the rows of
sequences with more than one query compute q K^T on the block-scaled tensor
cores (tcgen05 kind::mxf4nvf4), each query row quantized to NVFP4 by the KV row
codec under its own power-of-two global scale and K read as the cache's own
codes and block scales; decode rows are unchanged.

Bar: the same tolerance as the other attention paths (2e-3 per row before the
FP8 cast, one E4M3 step after), against the fp64 oracle over the quantized
queries. The oracle's NVFP4-query attention equals plain attention over the
queries round-tripped through the row codec (tests/test_oracle_pins.py), so
the quantized queries are formed here with the oracle's codec and the plain
oracle runs on them; that keeps single rows of long prefills checkable."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import (build_gpu_cache, check_bf16_from_fp8, check_fp8, check_rows, dev_scalar,
                           oracle_case, run_oracle, u16)

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _qhat_row(row):
    """NVFP4 round trip of one query row (bf16 bits uint16[D]) -> bf16 bits."""
    d = row.shape[0]
    g = oracle.q_row_global(row)
    q = oracle.quantize_row(np.ascontiguousarray(row), g)
    codes = np.empty(d, np.uint8)
    codes[0::2] = q[: d // 2] & 0xF
    codes[1::2] = q[: d // 2] >> 4
    sc = torch.from_numpy(q[d // 2:].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals = GRID[codes & 7] * np.where(codes & 8, -1.0, 1.0) * np.repeat(sc, 16) * g
    bits = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    return bits.view(np.uint16)


def _run(w, scales, cache):
    k_scale, v_scale, o_scale = scales
    q = wl.queries(w, DEV)
    shape = (q.shape[0], w.num_q_heads, w.head_size)
    o8 = torch.empty(shape, dtype=torch.uint8, device=DEV)
    o16 = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
    o32 = torch.empty(shape, dtype=torch.float32, device=DEV)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
    nk.paged_attention(q, cache, torch.from_numpy(w.block_table).to(DEV),
                       torch.from_numpy(w.seq_lens).to(DEV),
                       torch.tensor([k_scale, v_scale], dtype=torch.float32, device=DEV), o8,
                       dev_scalar(o_scale), ws, qo_indptr=torch.from_numpy(w.qo_indptr).to(DEV),
                       max_q_len=w.max_q_len, o_bf16=o16, o_f32=o32, q_fp4=True)
    torch.cuda.synchronize()
    assert nk.read_device_status(ws) == (nk.NVFP4_OK, 0)
    return o8.cpu(), o16.cpu(), o32.cpu()


def _check(w, scales, out, seqs, rows=None):
    case = oracle_case(w, seqs, scales, DEV, rows=rows)
    prefill_tok = set()
    for b in range(w.num_seqs):
        if int(w.q_lens[b]) > 1:
            prefill_tok.update(range(int(w.qo_indptr[b]), int(w.qo_indptr[b + 1])))
    qh = case["q"].copy()
    for i, tok in enumerate(case["out_index"]):
        if tok in prefill_tok:
            for h in range(w.num_q_heads):
                qh[i, h] = _qhat_row(case["q"][i, h])
    case["q"] = qh
    o64, r8, _ = run_oracle(case, scales)
    o8, o16, o32 = out
    idx = case["out_index"]
    d = w.head_size
    worst = check_rows(o32.numpy()[idx].reshape(-1, d), o64.reshape(-1, d))
    check_fp8(o8.numpy()[idx], r8)
    check_bf16_from_fp8(o16.contiguous().view(torch.int16).numpy().view(np.uint16)[idx], r8,
                        scales[2])
    return worst


QFP4_EDGE = [
    # (bs, Hq, Hkv, seq_lens, q_lens)
    (16, 64, 8, [333, 20], [90, 7]),           # G = 8 (16 tokens per tile); a partial chunk
    (32, 16, 8, [700, 129], [300, 129]),       # G = 2 (64 tokens per tile), bs 32, q_len == L
    (16, 16, 2, [3000, 1, 65], [700, 1, 64]),  # many chunks, a decode row, chunk edge
    (16, 40, 8, [200, 64], [130, 64]),         # G = 5 (125 rows per tile)
    (16, 16, 8, [5], [9]),                     # q_len > L: early rows see nothing
]


@pytest.mark.parametrize("bs,hq,hkv,lens,qlens", QFP4_EDGE)
def test_qfp4_prefill_edges(bs, hq, hkv, lens, qlens):
    w = wl.custom_workload("qfp4", 400 + bs + len(lens), hq, hkv, 256, bs, lens, qlens,
                           outliers="x20", spare_blocks=3)
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = _run(w, scales, cache)
    _check(w, scales, out, range(w.num_seqs))


def test_qfp4_mixed_prefill_decode_sampled():
    """The mixed batch's shapes (G = 8, D = 256, 2048-query prefills over 10240
    keys, 56 decode rows): sampled prefill rows and decode rows."""
    w = wl.make_workload("mixed_prefill_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = _run(w, scales, cache)
    rows = {0: [0, 1, 15, 16, 1023, 2047], 7: [5, 1500, 2046]}
    _check(w, scales, out, [0, 7, 8, 63], rows=rows)


def test_qfp4_rejected_off_head_size_256():
    w = wl.custom_workload("qfp4_d128", 3, 16, 8, 128, 16, [100], [20])
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    with pytest.raises(nk.Nvfp4Error):
        _run(w, scales, cache)
