"""The allocation-free paged attention entry point.

nvfp4_paged_attention_noalloc serves callers that cannot hand the library a
workspace (code given only its input and output buffers by a host framework,
or running while another allocator owns the device memory). It runs the same
kernels on a fixed scratch array inside the library. Checked here through the
C ABI against nvfp4_paged_attention on the same inputs, within the attention
tolerance of the other tests, on two calls in a row (the array keeps the
previous call's contents, so the second call checks that each call resets
what must start at zero). This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import build_gpu_cache, check_fp8, check_rows, dev_scalar

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(w):
    shape = (w.num_q_tokens, w.num_q_heads, w.head_size)
    return (torch.empty(shape, dtype=torch.uint8, device=DEV),
            torch.empty(shape, dtype=torch.bfloat16, device=DEV),
            torch.empty(shape, dtype=torch.float32, device=DEV))


@pytest.mark.parametrize("make", [
    lambda: wl.make_workload("qwen3_0p6b_decode"),
    lambda: wl.custom_workload("noalloc_mixed", 77, 8, 4, 256, 16, [300, 1000, 57, 4096],
                               [64, 1, 1, 1]),
])
def test_noalloc_matches_workspace_entry_point(make):
    w = make()
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    q = wl.queries(w, DEV)
    bt = torch.from_numpy(w.block_table).to(DEV)
    sl = torch.from_numpy(w.seq_lens).to(DEV)
    qo = None if w.is_decode else torch.from_numpy(w.qo_indptr).to(DEV)
    kvs = torch.tensor([scales[0], scales[1]], dtype=torch.float32, device=DEV)
    osc = dev_scalar(scales[2])

    nk.noalloc_status(clear=True)        # the status word is sticky across calls
    ref8, ref16, ref32 = _outputs(w)
    ws = nk.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_size, DEV)
    nk.paged_attention(q, cache, bt, sl, kvs, ref8, osc, ws, qo_indptr=qo, max_q_len=w.max_q_len,
                       o_bf16=ref16, o_f32=ref32)
    for call in range(2):
        o8, o16, o32 = _outputs(w)
        o8.fill_(0xFF)
        o32.fill_(float("nan"))
        nk.paged_attention_noalloc(q, cache, bt, sl, kvs, o8, osc, qo_indptr=qo,
                                   max_q_len=w.max_q_len, o_bf16=o16, o_f32=o32)
        torch.cuda.synchronize()
        d = w.head_size
        check_rows(o32.cpu().numpy().reshape(-1, d), ref32.cpu().numpy().reshape(-1, d).astype(np.float64))
        check_fp8(o8.cpu().numpy(), ref8.cpu().numpy())
        assert nk.noalloc_status() == (nk.NVFP4_OK, 0)


def test_noalloc_reports_device_status():
    """A planted out-of-range block id: the allocation-free call skips the page
    like the workspace call does, and its status read-back reports it (then
    clears it)."""
    w = wl.custom_workload("noalloc_badblk", 5, 8, 2, 128, 16, [40, 70])
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    w.block_table[1, 2] = w.num_blocks + 1000
    nk.noalloc_status(clear=True)
    o8, o16, o32 = _outputs(w)
    nk.paged_attention_noalloc(wl.queries(w, DEV), cache, torch.from_numpy(w.block_table).to(DEV),
                               torch.from_numpy(w.seq_lens).to(DEV),
                               torch.tensor([scales[0], scales[1]], device=DEV), o8,
                               dev_scalar(scales[2]), o_f32=o32)
    st, bits = nk.noalloc_status(clear=True)
    assert st == nk.NVFP4_ERR_DEVICE_BOUNDS and bits & nk.DEV_BAD_BLOCK
    assert nk.noalloc_status() == (nk.NVFP4_OK, 0)
    assert torch.isfinite(o32).all()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """64 query heads over 8 kv heads at head_size 256 need ~39 MB of split-KV
    partial slots, more than the fixed 12 MiB array: the call must fail with
    NVFP4_ERR_WORKSPACE before launching anything. The buffers are real and
    valid anyway."""
    B, HQ, HKV, D = 4, 64, 8, 256
    assert nk.workspace_size(B, HQ, HKV, D) > 12 << 20
    q = torch.zeros((B, HQ, D), dtype=torch.bfloat16, device=DEV)
    cache = nk.alloc_kv_cache(1, 16, HKV, D, DEV)
    bt = torch.zeros((B, 1), dtype=torch.int32, device=DEV)
    sl = torch.ones(B, dtype=torch.int32, device=DEV)
    o8 = torch.empty((B, HQ, D), dtype=torch.uint8, device=DEV)
    with pytest.raises(nk.Nvfp4Error) as e:
        nk.paged_attention_noalloc(q, cache, bt, sl, torch.ones(2, device=DEV), o8,
                                   torch.ones(1, device=DEV))
    assert e.value.status == nk.NVFP4_ERR_WORKSPACE
