"""FP8-E4M3 KV variant (nvfp4_fp8kv_quantize_append_paged,
nvfp4_fp8kv_paged_attention): the comparison format of "FlashInfer backend adds
end-to-end NVFP4 KV cache support", review highlights. Writer bit-exact vs the
oracle's FP8 writer (untouched rows kept); attention within the same bars as
the NVFP4 path (2e-3 per row before the FP8 cast, 1 E4M3 step after)."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import (build_gpu_cache, check_bf16_from_fp8, check_fp8, check_rows, dev_scalar,
                           oracle_case, run_gpu_attention, run_oracle, u16)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_fp8kv_writer_append_sweep_bit_exact():
    """The append sweep's shape (8192 tokens, 5% slots -1) into a 4096-block
    FP8 cache (slots drawn within it), sentinel-filled: every row named by a
    slot equals the oracle's, every other byte is untouched."""
    app = wl.make_append("append_sweep", num_blocks=4096)
    k, v = app.kv(DEV)
    gk, gv = app.scales(k, v)
    slots = app.slot_mapping()
    cache = nk.alloc_fp8_kv_cache(app.num_blocks, app.block_size, app.num_kv_heads, app.head_size, DEV)
    cache.fill_(0xA5)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    nk.quantize_append_paged(k, v, cache, torch.from_numpy(slots).to(DEV), dev_scalar(gk),
                             dev_scalar(gv), device_status=st, fp8=True)
    ref = np.full(tuple(cache.shape), 0xA5, np.uint8)
    oracle.fp8kv_quantize_append_paged(u16(k), u16(v), ref, slots, gk, gv, app.block_size)
    assert np.array_equal(cache.cpu().numpy(), ref)
    assert nk.read_device_status(st) == (nk.NVFP4_OK, 0)


def _compare(w, scales, out, case):
    o8, o16, o32 = (t.cpu() for t in out[:3])
    o64, r8, _ = run_oracle(case, scales)
    idx = case["out_index"]
    d = w.head_size
    check_rows(o32.numpy()[idx].reshape(-1, d), o64.reshape(-1, d))
    check_fp8(o8.numpy()[idx], r8)
    check_bf16_from_fp8(o16.contiguous().view(torch.int16).numpy().view(np.uint16)[idx], r8,
                        scales[2])


def test_fp8kv_decode_qwen3_0p6b_decode():
    w = wl.make_workload("qwen3_0p6b_decode")
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV, fp8=True)
    out = run_gpu_attention(w, cache, scales, DEV, fp8=True)
    assert nk.read_device_status(out[3]) == (nk.NVFP4_OK, 0)
    _compare(w, scales, out, oracle_case(w, range(w.num_seqs), scales, DEV, fp8=True))


FP8_EDGE = [
    # (D, bs, Hq, Hkv, seq_lens, q_lens)
    (128, 16, 16, 8, [1, 16, 17, 33, 500], None),
    (64, 32, 8, 8, [1, 31, 32, 65], None),                  # G = 1, D 64
    (256, 16, 64, 8, [3, 129, 1000], None),                 # G = 8, D 256
    (128, 32, 12, 4, [100, 700, 2500], None),               # G = 3, bs 32
    (128, 16, 16, 8, [40, 300, 16], [40, 77, 2]),           # chunked prefill + decode
    (256, 16, 64, 8, [1500, 90], [600, 1]),                 # prefill, G = 8, D 256
]


@pytest.mark.parametrize("D,bs,hq,hkv,lens,qlens", FP8_EDGE)
def test_fp8kv_attention_edges(D, bs, hq, hkv, lens, qlens):
    w = wl.custom_workload("fp8edge", 500 + D + bs + len(lens), hq, hkv, D, bs, lens, qlens,
                           outliers="x20", spare_blocks=3)
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV, sentinel=0xFF, fp8=True)   # NaN codes in stale rows
    out = run_gpu_attention(w, cache, scales, DEV, fp8=True)
    assert nk.read_device_status(out[3]) == (nk.NVFP4_OK, 0)
    assert torch.isfinite(out[2]).all()
    _compare(w, scales, out, oracle_case(w, range(w.num_seqs), scales, DEV, fp8=True))
