"""Host-side workload bookkeeping used by the benchmark (no GPU needed)."""
from nvfp4_quantized_paged_append_b200 import workloads as wl


def test_prefill_flops_counts_visible_keys():
    # seq 0: L = 5, q_len = 3 -> rows at positions 2, 3, 4 see 3 + 4 + 5 = 12 keys
    # seq 1: decode (q_len 1) -> not counted
    # seq 2: L = 2, q_len = 4 -> positions -2, -1, 0, 1 see 0 + 0 + 1 + 2 = 3 keys
    w = wl.custom_workload("flops", 1, 4, 2, 64, 16, [5, 40, 2], [3, 1, 4])
    assert w.prefill_flops() == (12 + 3) * 4 * 4 * 64
    assert wl.make_workload("qwen3_0p6b_decode").prefill_flops() == 0


def test_kv_bytes_counts_rows_without_block_padding():
    w = wl.custom_workload("bytes", 2, 8, 8, 128, 16, [1, 17, 100])
    assert w.kv_bytes() == (1 + 17 + 100) * 8 * 2 * 72
