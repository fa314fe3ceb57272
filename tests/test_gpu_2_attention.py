"""Paged attention on the GPU vs the fp64 CPU oracle.

Bar: per output row (query token, head) max |o - o_ref| <= 2e-3 * max |o_ref|
before the FP8 cast (o_f32), E4M3 output within one step of the oracle's
E4M3(o_ref / o_scale), and o_bf16 equal to bf16(E4M3 * o_scale) of such a code.
Every workload runs at full size on the GPU in the launch configuration the
benchmark uses; the oracle checks all rows of the smaller ones and sampled
sequences / query rows of the two largest."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import (build_gpu_cache, check_bf16_from_fp8, check_fp8, check_rows, oracle_case,
                           run_gpu_attention, run_oracle)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _compare(w, scales, gpu_out, case, ref):
    o8, o16, o32 = (t.cpu() for t in gpu_out)
    idx = case["out_index"]
    o64, r8, _ = ref
    hq, d = w.num_q_heads, w.head_size
    g32 = o32.numpy()[idx].reshape(-1, d)
    worst = check_rows(g32, o64.reshape(-1, d))
    check_fp8(o8.numpy()[idx], r8)
    check_bf16_from_fp8(o16.contiguous().view(torch.int16).numpy().view(np.uint16)[idx], r8, scales[2])
    assert np.isfinite(g32).all()
    return worst


@pytest.mark.parametrize("name", ["tiny_decode", "qwen3_0p6b_decode"])
def test_decode_workload_full(name):
    w = wl.make_workload(name)
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = run_gpu_attention(w, cache, scales, DEV)
    assert nk.workspace_status(out[3]) == 0
    case = oracle_case(w, range(w.num_seqs), scales, DEV)
    _compare(w, scales, out[:3], case, run_oracle(case, scales))


def test_long_decode_sampled():
    w = wl.make_workload("long_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = run_gpu_attention(w, cache, scales, DEV)
    assert nk.workspace_status(out[3]) == 0
    case = oracle_case(w, [0, 31, 63], scales, DEV)
    _compare(w, scales, out[:3], case, run_oracle(case, scales))


def test_mixed_prefill_decode_sampled():
    w = wl.make_workload("mixed_prefill_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = run_gpu_attention(w, cache, scales, DEV)
    assert nk.workspace_status(out[3]) == 0
    rows = {0: [0, 1, 7, 8, 63, 64, 1023, 2047], 7: [2, 500, 1500, 2046]}
    case = oracle_case(w, [0, 7, 8, 30, 63], scales, DEV, rows=rows)
    _compare(w, scales, out[:3], case, run_oracle(case, scales))


EDGE = [
    # (D, bs, Hq, Hkv, seq_lens, q_lens)
    (128, 16, 16, 8, [1, 16, 17, 33, 500], None),          # page edges, single key
    (64, 32, 8, 8, [1, 31, 32, 65], None),                  # G = 1, bs 32
    (256, 16, 64, 8, [3, 129, 1000], None),                 # G = 8, D 256
    (128, 32, 32, 8, [4096, 7], None),                      # G = 4
    (64, 16, 4, 2, [37, 100], [5, 1]),                       # prefill + decode mix
    (128, 16, 16, 8, [40, 300, 16], [40, 77, 2]),           # q_len == L (no cache) / ragged
    (256, 32, 16, 2, [200, 64], [130, 64]),                 # G = 8, bs 32 prefill
    (128, 16, 8, 2, [5], [9]),                              # q_len > L: early rows see nothing
    (128, 16, 12, 4, [100, 700, 2500], None),               # G = 3: odd group, lo columns cross lanes
    (64, 16, 12, 2, [90, 1300], None),                      # G = 6: separate lo fragments
    # chunked prefill on the tensor cores: M = 128 rows of (token, head)
    (128, 32, 4, 4, [700, 129], [300, 129]),                # G = 1: 128 tokens per tile
    (128, 16, 12, 4, [515, 64], [200, 3]),                  # G = 3: 42 tokens (126 rows)
    (256, 16, 40, 8, [333, 20], [90, 7]),                   # G = 5: 25 tokens (125 rows)
    (256, 16, 64, 8, [3000, 1], [700, 1]),                  # G = 8, many 64-key chunks
    (64, 32, 8, 4, [64, 65, 191], [64, 65, 2]),             # chunk and page edges, D 64
]


@pytest.mark.parametrize("D,bs,hq,hkv,lens,qlens", EDGE)
def test_edge_cases(D, bs, hq, hkv, lens, qlens):
    w = wl.custom_workload("edge", 100 + D + bs + len(lens), hq, hkv, D, bs, lens, qlens,
                           outliers="x20", spare_blocks=3)
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = run_gpu_attention(w, cache, scales, DEV)
    assert nk.workspace_status(out[3]) == 0
    case = oracle_case(w, range(w.num_seqs), scales, DEV)
    _compare(w, scales, out[:3], case, run_oracle(case, scales))


def test_repeat_calls_identical_and_workspace_reusable():
    """Split-KV arrival counters reset themselves: a second call on the same workspace
    gives bit-identical outputs."""
    w = wl.make_workload("qwen3_0p6b_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    q = wl.queries(w, DEV)
    k_scale, v_scale, o_scale = scales
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
    bt = torch.from_numpy(w.block_table).to(DEV)
    sl = torch.from_numpy(w.seq_lens).to(DEV)
    kvs = torch.tensor([k_scale, v_scale], dtype=torch.float32, device=DEV)
    osc = torch.tensor([o_scale], dtype=torch.float32, device=DEV)
    outs = []
    for _ in range(3):
        o8 = torch.empty((w.num_seqs, w.num_q_heads, w.head_size), dtype=torch.uint8, device=DEV)
        o32 = torch.empty((w.num_seqs, w.num_q_heads, w.head_size), dtype=torch.float32, device=DEV)
        nk.paged_attention(q, cache, bt, sl, kvs, o8, osc, ws, o_f32=o32)
        outs.append((o8.clone(), o32.clone()))
    torch.cuda.synchronize()
    for o8, o32 in outs[1:]:
        assert torch.equal(o8, outs[0][0]) and torch.equal(o32, outs[0][1])
    # no status bit was raised, and the arrival counters of the cut segments
    # are back to zero for the next call
    assert nk.workspace_status(ws) == 0
    counters = ws[256: 256 + 4 * w.num_seqs * w.num_kv_heads].view(torch.int32)
    assert int(counters.abs().sum()) == 0


def test_bad_block_id_flagged_no_fault():
    """A planted out-of-range block id is skipped (no fault) and reported through
    the C ABI's status read-back as NVFP4_ERR_DEVICE_BOUNDS; clearing resets it."""
    w = wl.custom_workload("badblk", 5, 8, 2, 128, 16, [40, 70])
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    w.block_table[1, 2] = w.num_blocks + 1000   # out of range
    out = run_gpu_attention(w, cache, scales, DEV)
    st, bits = nk.read_device_status(out[3], clear=True)
    assert st == nk.NVFP4_ERR_DEVICE_BOUNDS and bits & nk.DEV_BAD_BLOCK
    assert nk.read_device_status(out[3]) == (nk.NVFP4_OK, 0)
    assert torch.isfinite(out[2]).all()


def test_prefill_bad_block_id_flagged_no_fault():
    """An out-of-range block id inside a prefill range: its page is skipped (no
    fault), the status reads back NVFP4_ERR_DEVICE_BOUNDS, outputs are finite,
    and rows whose causal window ends before that page match the oracle."""
    w = wl.custom_workload("pf_badblk", 8, 16, 8, 128, 16, [400], [300])
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    good = int(w.block_table[0, 20])
    w.block_table[0, 20] = w.num_blocks + 77     # keys 320..335
    out = run_gpu_attention(w, cache, scales, DEV)
    st, bits = nk.read_device_status(out[3])
    assert st == nk.NVFP4_ERR_DEVICE_BOUNDS and bits & nk.DEV_BAD_BLOCK
    assert torch.isfinite(out[2]).all()
    # rows at positions < 320 never see the bad page
    rows = {0: [0, 1, 50, 150, 219]}             # positions 100 .. 319
    w.block_table[0, 20] = good                  # (the oracle's rows never read that page)
    case = oracle_case(w, [0], scales, DEV, rows=rows)
    o64, r8, _ = run_oracle(case, scales)
    idx = case["out_index"]
    check_rows(out[2].cpu().numpy()[idx].reshape(-1, w.head_size), o64.reshape(-1, w.head_size))


def test_query_range_beyond_max_q_len_flagged():
    """A prefill range longer than the host's max_q_len bound leaves rows beyond
    the launched grid unwritten and raises DEV_BAD_QLEN (read back through the
    C ABI)."""
    w = wl.custom_workload("badqlen", 6, 8, 2, 128, 16, [300, 90], [200, 1])
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    q = wl.queries(w, DEV)
    o8 = torch.zeros((w.num_q_tokens, w.num_q_heads, w.head_size), dtype=torch.uint8, device=DEV)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
    nk.paged_attention(q, cache, torch.from_numpy(w.block_table).to(DEV),
                       torch.from_numpy(w.seq_lens).to(DEV),
                       torch.tensor([scales[0], scales[1]], device=DEV), o8,
                       torch.tensor([scales[2]], device=DEV), ws,
                       qo_indptr=torch.from_numpy(w.qo_indptr).to(DEV), max_q_len=16)
    st, bits = nk.read_device_status(ws)
    assert st == nk.NVFP4_ERR_DEVICE_BOUNDS and bits & nk.DEV_BAD_QLEN


def test_bounded_wait_gives_up_and_context_survives():
    """The bounded-wait self-test: a barrier wait that no copy completes gives up
    after its poll limit, the kernel returns, DEV_TIMEOUT reads back as
    NVFP4_ERR_DEVICE_TIMEOUT, and the context still runs attention correctly."""
    word = torch.zeros(1, dtype=torch.int32, device=DEV)
    nk.wait_timeout_probe(word, polls=2000)
    st, bits = nk.read_device_status(word, clear=True)
    assert st == nk.NVFP4_ERR_DEVICE_TIMEOUT and bits == nk.DEV_TIMEOUT
    assert nk.read_device_status(word) == (nk.NVFP4_OK, 0)
    w = wl.make_workload("tiny_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    out = run_gpu_attention(w, cache, scales, DEV)
    assert nk.read_device_status(out[3]) == (nk.NVFP4_OK, 0)
    case = oracle_case(w, range(w.num_seqs), scales, DEV)
    _compare(w, scales, out[:3], case, run_oracle(case, scales))


def test_output_scale_and_sm_scale_arguments():
    """A non-default sm_scale and a small o_scale (saturating FP8) behave as specified."""
    w = wl.make_workload("tiny_decode")
    scales = (1.0, 1.0, 0.002)
    cache = build_gpu_cache(w, scales, DEV)
    q = wl.queries(w, DEV)
    o8 = torch.empty((2, 4, 64), dtype=torch.uint8, device=DEV)
    o32 = torch.empty((2, 4, 64), dtype=torch.float32, device=DEV)
    ws = nk.alloc_workspace(2, 4, 2, 64, DEV)
    nk.paged_attention(q, cache, torch.from_numpy(w.block_table).to(DEV),
                       torch.from_numpy(w.seq_lens).to(DEV), torch.ones(2, device=DEV), o8,
                       torch.tensor([0.002], device=DEV), ws, sm_scale=0.3, o_f32=o32)
    torch.cuda.synchronize()
    case = oracle_case(w, [0, 1], scales, DEV)
    import oracle
    o64, r8, _ = oracle.paged_attention(case["q"], case["cache"], case["block_table"],
                                        case["seq_lens"], None, 1.0, 1.0, 0.3, 0.002)
    check_rows(o32.cpu().numpy().reshape(-1, 64), o64.reshape(-1, 64))
    check_fp8(o8.cpu().numpy(), r8)
    assert ((r8.astype(np.int64) & 0x7F) == 0x7E).any()        # some outputs saturate at 448
    assert ((o8.cpu().numpy().astype(np.int64) & 0x7F) == 0x7E).any()


def test_metadata_ready_after_writer_matches_default():
    """The writer appends every sequence's last token, then attention runs as its
    programmatic dependent with NVFP4_ATTN_METADATA_READY (block table and lengths
    read before the writer finishes): outputs equal those of the default launch."""
    w = wl.make_workload("qwen3_0p6b_decode")
    scales = wl.global_scales(w, DEV)
    k_scale, v_scale, o_scale = scales
    B = w.num_seqs
    hist = nk.alloc_kv_cache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_size, DEV)
    ks = torch.tensor([k_scale], dtype=torch.float32, device=DEV)
    vs = torch.tensor([v_scale], dtype=torch.float32, device=DEV)
    k_new, v_new, slots = [], [], []
    for b in range(B):
        L = int(w.seq_lens[b])
        k, v = wl.seq_kv(w, b, DEV)
        nk.quantize_append_paged(k[:L - 1], v[:L - 1], hist,
                                 torch.from_numpy(w.slots_for_seq(b, 0, L - 1)).to(DEV), ks, vs)
        k_new.append(k[L - 1:])
        v_new.append(v[L - 1:])
        slots.append(w.slots_for_seq(b, L - 1)[:1])
    k_new = torch.cat(k_new).contiguous()
    v_new = torch.cat(v_new).contiguous()
    slots = torch.from_numpy(np.concatenate(slots).astype(np.int64)).to(DEV)
    q = wl.queries(w, DEV)
    bt = torch.from_numpy(w.block_table).to(DEV)
    sl = torch.from_numpy(w.seq_lens).to(DEV)
    kvs = torch.tensor([k_scale, v_scale], dtype=torch.float32, device=DEV)
    osc = torch.tensor([o_scale], dtype=torch.float32, device=DEV)
    outs = []
    for ready in (False, True):
        cache = hist.clone()
        ws = nk.alloc_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
        o8 = torch.empty((B, w.num_q_heads, w.head_size), dtype=torch.uint8, device=DEV)
        o32 = torch.empty((B, w.num_q_heads, w.head_size), dtype=torch.float32, device=DEV)
        nk.quantize_append_paged(k_new, v_new, cache, slots, ks, vs)
        nk.paged_attention(q, cache, bt, sl, kvs, o8, osc, ws, o_f32=o32, metadata_ready=ready)
        torch.cuda.synchronize()
        assert nk.workspace_status(ws) == 0
        outs.append((o8, o32))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
