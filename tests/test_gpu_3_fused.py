"""The fused decode step (nvfp4_paged_decode_append): one launch writes every
sequence's newest K/V row into the NVFP4 cache and attends over all keys.

Bar: the cache bytes equal the oracle writer's bit for bit (the new rows
included, nothing else touched); the outputs equal those of the unfused path
(the library's writer, then nvfp4_paged_attention) bit for bit, and are within
the attention tolerance of the fp64 oracle ("FlashInfer backend adds
end-to-end NVFP4 KV cache support", key source snippets: the forward pass
writes with reshape_and_cache_flash, then runs the attention kernel)."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import check_bf16_from_fp8, check_fp8, check_rows, dev_scalar, oracle_case, \
    run_oracle, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _history_cache(w, scales, sentinel=0x5A):
    """Device cache holding every token but each sequence's last (library
    writer), over a sentinel fill; and the oracle's cache of all tokens."""
    k_scale, v_scale, _ = scales
    cache = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, DEV)
    cache.fill_(sentinel)
    ref = np.full(tuple(cache.shape), sentinel, np.uint8)
    ks, vs = dev_scalar(k_scale), dev_scalar(v_scale)
    k_new, v_new = [], []
    for b in range(w.num_seqs):
        L = int(w.seq_lens[b])
        k, v = wl.seq_kv(w, b, DEV)
        if L > 1:
            nk.quantize_append_paged(k[:L - 1], v[:L - 1], cache,
                                     torch.from_numpy(w.slots_for_seq(b, 0, L - 1)).to(DEV), ks, vs)
        oracle.quantize_append_paged(u16(k), u16(v), ref, w.slots_for_seq(b), k_scale, v_scale,
                                     w.block_size)
        k_new.append(k[L - 1:])
        v_new.append(v[L - 1:])
    return cache, ref, torch.cat(k_new).contiguous(), torch.cat(v_new).contiguous()


def _outputs(w):
    shape = (w.num_seqs, w.num_q_heads, w.head_size)
    return (torch.empty(shape, dtype=torch.uint8, device=DEV),
            torch.empty(shape, dtype=torch.bfloat16, device=DEV),
            torch.empty(shape, dtype=torch.float32, device=DEV))


def _run_case(w):
    scales = wl.global_scales(w, DEV)
    k_scale, v_scale, o_scale = scales
    hist, ref_cache, k_new, v_new = _history_cache(w, scales)
    q = wl.queries(w, DEV)
    bt = torch.from_numpy(w.block_table).to(DEV)
    sl = torch.from_numpy(w.seq_lens).to(DEV)
    kvs = torch.tensor([k_scale, v_scale], dtype=torch.float32, device=DEV)
    osc = dev_scalar(o_scale)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)

    # fused
    cache_f = hist.clone()
    f8, f16, f32 = _outputs(w)
    nk.paged_decode_append(q, k_new, v_new, cache_f, bt, sl, kvs, f8, osc, ws, o_bf16=f16,
                           o_f32=f32)
    assert nk.read_device_status(ws) == (nk.NVFP4_OK, 0)
    # unfused: the writer, then attention
    cache_u = hist.clone()
    slots = torch.from_numpy(np.array([w.slots_for_seq(b, int(w.seq_lens[b]) - 1)[0]
                                       for b in range(w.num_seqs)], np.int64)).to(DEV)
    nk.quantize_append_paged(k_new, v_new, cache_u, slots, kvs[0:1], kvs[1:2])
    u8, u16_, u32 = _outputs(w)
    nk.paged_attention(q, cache_u, bt, sl, kvs, u8, osc, ws, o_bf16=u16_, o_f32=u32)
    torch.cuda.synchronize()

    assert np.array_equal(cache_f.cpu().numpy(), ref_cache), "fused cache differs from the oracle writer"
    assert torch.equal(cache_f, cache_u)
    assert torch.equal(f8, u8) and torch.equal(f16, u16_) and torch.equal(f32, u32)
    case = oracle_case(w, range(w.num_seqs), scales, DEV)
    o64, r8, _ = run_oracle(case, scales)
    d = w.head_size
    check_rows(f32.cpu().numpy().reshape(-1, d), o64.reshape(-1, d))
    check_fp8(f8.cpu().numpy(), r8)
    check_bf16_from_fp8(f16.contiguous().view(torch.int16).cpu().numpy().view(np.uint16), r8,
                        o_scale)


def test_fused_decode_append_qwen3_0p6b_decode():
    _run_case(wl.make_workload("qwen3_0p6b_decode"))


FUSED_EDGE = [
    # (D, bs, Hq, Hkv, seq_lens)
    (128, 16, 16, 8, [1, 17, 33, 16, 500]),       # first token; new token opens a page; page end
    (256, 16, 64, 8, [129, 1000, 2]),             # G = 8, D 256 (separate lo fragments)
    (256, 32, 16, 2, [65, 32, 4000]),             # bs 32, one page per unit
    (64, 16, 12, 2, [97, 1300, 1]),               # D 64: rows 4-byte aligned, G = 6
    (64, 32, 4, 4, [33, 64, 700]),                # G = 1, bs 32
    (128, 16, 12, 4, [100, 2500]),                # G = 3
]


@pytest.mark.parametrize("D,bs,hq,hkv,lens", FUSED_EDGE)
def test_fused_decode_append_edges(D, bs, hq, hkv, lens):
    _run_case(wl.custom_workload("fused", 300 + D + bs + len(lens), hq, hkv, D, bs, lens,
                                 outliers="x20", spare_blocks=5))


def test_fused_decode_append_bad_block_flagged():
    """A new token whose block id is out of range is neither written nor
    attended to; the status reads back NVFP4_ERR_DEVICE_BOUNDS."""
    w = wl.custom_workload("fused_bad", 9, 8, 2, 128, 16, [40, 70])
    scales = wl.global_scales(w, DEV)
    hist, _, k_new, v_new = _history_cache(w, scales)
    w.block_table[1, (70 - 1) // 16] = w.num_blocks + 5
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
    f8, f16, f32 = _outputs(w)
    cache = hist.clone()
    nk.paged_decode_append(wl.queries(w, DEV), k_new, v_new, cache,
                           torch.from_numpy(w.block_table).to(DEV),
                           torch.from_numpy(w.seq_lens).to(DEV),
                           torch.tensor([scales[0], scales[1]], device=DEV), f8,
                           dev_scalar(scales[2]), ws, o_f32=f32)
    st, bits = nk.read_device_status(ws)
    assert st == nk.NVFP4_ERR_DEVICE_BOUNDS and bits & nk.DEV_BAD_BLOCK
    assert torch.isfinite(f32).all()
    # sequence 0's new row was written; nothing else of sequence 1's changed
    diff = (cache != hist).nonzero()
    assert diff.numel() > 0
    assert set(diff[:, 0].tolist()) <= {int(x) for x in w.block_table[0, :3]}


def test_fused_history_ready_chain():
    """NVFP4_ATTN_HISTORY_READY: the step's first page copies start before it
    waits for the preceding kernel. Chained after a step on another cache (the
    flag's precondition), its cache and outputs equal those of the same step
    launched with no flags, bit for bit."""
    wa = wl.custom_workload("chain_a", 21, 16, 8, 128, 16, [300, 1200, 77, 2049],
                            outliers="x20")
    wb = wl.custom_workload("chain_b", 22, 16, 8, 128, 16, [900, 17, 3000, 640],
                            outliers="x20")
    runs = {}
    for flags in ("plain", "history"):
        outs = []
        for w in (wa, wb):
            scales = wl.global_scales(w, DEV)
            hist, _, k_new, v_new = _history_cache(w, scales)
            ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
            outs.append((w, scales, hist, k_new, v_new, ws, _outputs(w)))
        torch.cuda.synchronize()
        for i, (w, scales, cache, k_new, v_new, ws, (o8, o16, o32)) in enumerate(outs):
            nk.paged_decode_append(wl.queries(w, DEV), k_new, v_new, cache,
                                   torch.from_numpy(w.block_table).to(DEV),
                                   torch.from_numpy(w.seq_lens).to(DEV),
                                   torch.tensor([scales[0], scales[1]], device=DEV), o8,
                                   dev_scalar(scales[2]), ws, o_bf16=o16, o_f32=o32,
                                   history_ready=(flags == "history" and i == 1))
        torch.cuda.synchronize()
        for o in outs:
            assert nk.read_device_status(o[5]) == (nk.NVFP4_OK, 0)
        runs[flags] = [(o[2].clone(), [t.clone() for t in o[6]]) for o in outs]
    for (ca, oa), (cb, ob) in zip(runs["plain"], runs["history"]):
        assert torch.equal(ca, cb)
        for x, y in zip(oa, ob):
            assert torch.equal(x, y)
