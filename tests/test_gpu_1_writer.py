"""Writer and dequant on the GPU vs the CPU oracle: bit-exact.

Covers the codec edge cases (ties, saturation, subnormal and zero scales,
negative zero), the hand-worked rows, every workload's append (full size, or
sampled sequences for the two largest), the untouched-row invariant on a
sentinel-filled cache, strided inputs, bad slots, and the dequant helper."""
import os

import numpy as np
import pytest
import torch

import nvfp4_quantized_paged_append_b200 as nk
import oracle
from nvfp4_quantized_paged_append_b200 import workloads as wl
from paged_helpers import build_gpu_cache, dev_scalar, oracle_case, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _gpu_write(k, v, slots, nb, bs, gk, gv, sentinel=None, status=None):
    T, H, D = k.shape
    cache = nk.alloc_kv_cache(nb, bs, H, D, DEV)
    if sentinel is not None:
        cache.copy_(torch.from_numpy(sentinel))
    nk.quantize_append_paged(k.to(DEV), v.to(DEV), cache, torch.from_numpy(slots).to(DEV),
                             dev_scalar(gk), dev_scalar(gv), device_status=status)
    torch.cuda.synchronize()
    return cache.cpu().numpy()


def _oracle_write(k, v, slots, nb, bs, gk, gv, sentinel=None):
    T, H, D = k.shape
    cache = np.zeros((nb, 2, H, bs, nk.full_dim(D)), np.uint8) if sentinel is None else sentinel.copy()
    oracle.quantize_append_paged(u16(k), u16(v), cache, slots, gk, gv, bs)
    return cache


def test_golden_rows_through_gpu_writer():
    rows = []
    with open(os.path.join(GOLDEN, "worked_rows.txt")) as f:
        for ln in f:
            if ln.startswith("#") or not ln.strip():
                continue
            g, xs, hx = [p.strip() for p in ln.split(";")]
            rows.append((float(g), [float(x) for x in xs.split()], bytes.fromhex(hx)))
    for g, xs, want in rows:
        # a head_size-64 row = the same 16-value group four times
        x = np.tile(np.array(xs, np.float32), 4).reshape(1, 1, 64)
        k = _bf16(x)
        cache = _gpu_write(k, k, np.array([0], np.int64), 1, 16, g, g)
        row = cache[0, 0, 0, 0]
        assert bytes(row[:32]) == want[:8] * 4, (g, xs)
        assert bytes(row[32:]) == want[8:] * 4, (g, xs)


def _codec_cases(rng, T, H, D):
    """bf16 rows aimed at the rounding decisions: grid points, midpoints
    (ties) and their neighbours times random E4M3 scales, plus noise."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, 7, 100], np.float32)
    n = T * H * D // 16
    sb = rng.integers(1, 0x7F, n).astype(np.uint8)
    S = torch.from_numpy(sb).view(torch.float8_e4m3fn).float().numpy()
    vals = rng.choice(grid, (n, 16)) * S[:, None] * rng.choice([-1, 1], (n, 16))
    vals *= np.where(rng.random((n, 16)) < 0.2, 1 + rng.choice([-1, 1], (n, 16)) * 2.0 ** -8, 1.0)
    noise = rng.standard_normal((n, 16)) * S[:, None] * rng.uniform(0.1, 4, (n, 1))
    vals = np.where(rng.random((n, 16)) < 0.25, noise, vals)
    vals[rng.random(n) < 0.03] = 0.0
    neg0 = rng.random((n, 16)) < 0.02
    vals = np.where(neg0, -0.0, vals)
    return vals.reshape(T, H, D).astype(np.float32)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("g", [1.0, 0.5, 3.0e-3, 1.7, 1.0 / 64])
def test_codec_bruteforce_bit_exact(D, g):
    rng = np.random.default_rng(D * 7 + int(g * 1000))
    T, H, bs = 512, 2, 16
    x = _codec_cases(rng, T, H, D) * np.float32(g)
    k = _bf16(x)
    v = _bf16(x[::-1].copy())
    nb = T // bs
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    got = _gpu_write(k, v, slots, nb, bs, g, g)
    want = _oracle_write(k, v, slots, nb, bs, g, g)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("D,H", [(64, 1), (64, 8), (128, 2), (128, 4), (256, 2), (256, 8)])
@pytest.mark.parametrize("g", [0.37, 2.0 ** 110, 2.0 ** -120])
def test_codec_bruteforce_every_writer_mapping(D, H, g):
    """The same codec cases through each writer mapping: one CTA per token
    (D 64, H 1), one thread per 16-element group (D 64 H 8, D 128 H 2), two
    groups per thread (D 128 H 4, D 256 H 2 / 8); global scales that send the
    effective scale above 2^100 (IEEE-division path) or make 6 g and the
    scales subnormal."""
    rng = np.random.default_rng(D * 13 + H)
    T, bs = 256, 16
    x = _codec_cases(rng, T, H, D) * np.float32(g)
    k = _bf16(x)
    v = _bf16(-x[::-1].copy())
    nb = T // bs + 2
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[rng.random(T) < 0.05] = -1
    got = _gpu_write(k, v, slots, nb, bs, g, g * 0.75)
    want = _oracle_write(k, v, slots, nb, bs, g, g * 0.75)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("name", ["tiny_decode", "qwen3_0p6b_decode"])
def test_writer_decode_workloads_full(name):
    w = wl.make_workload(name)
    scales = wl.global_scales(w, DEV)
    sentinel = 0xA5
    cache = build_gpu_cache(w, scales, DEV, sentinel=sentinel).cpu().numpy()
    ref = np.full_like(cache, sentinel)
    for b in range(w.num_seqs):
        k, v = wl.seq_kv(w, b, DEV)
        oracle.quantize_append_paged(u16(k), u16(v), ref, w.slots_for_seq(b), scales[0], scales[1],
                                     w.block_size)
    assert np.array_equal(cache, ref)


def test_writer_append_sweep_full():
    a = wl.make_append()
    k, v = a.kv(DEV)
    gk, gv = a.scales(k, v)
    slots = a.slot_mapping()
    rng = np.random.default_rng(0)
    # sentinel: random bytes in the touched pages' neighbourhood would be 1.2 GB on the host;
    # a constant byte is enough to see any stray write
    cache = nk.alloc_kv_cache(a.num_blocks, a.block_size, a.num_kv_heads, a.head_size, DEV)
    cache.fill_(0x5A)
    nk.quantize_append_paged(k, v, cache, torch.from_numpy(slots).to(DEV), dev_scalar(gk),
                             dev_scalar(gv))
    torch.cuda.synchronize()
    got = cache.cpu().numpy()
    ref = np.full_like(got, 0x5A)
    oracle.quantize_append_paged(u16(k), u16(v), ref, slots, gk, gv, a.block_size)
    assert np.array_equal(got, ref)
    del rng


@pytest.mark.parametrize("name,seqs", [("long_decode", [0, 37, 63]),
                                       ("mixed_prefill_decode", [0, 5, 8, 40, 63])])
def test_writer_large_workloads_sampled(name, seqs):
    w = wl.make_workload(name)
    scales = wl.global_scales(w, DEV)
    cache = build_gpu_cache(w, scales, DEV)
    case = oracle_case(w, seqs, scales, DEV)
    blocks = []
    for b in seqs:
        blocks += [int(x) for x in w.block_table[b, : -(-int(w.seq_lens[b]) // w.block_size)]]
    blocks = list(dict.fromkeys(blocks))
    got = cache[torch.tensor(blocks, device=DEV)].cpu().numpy()
    assert np.array_equal(got, case["cache"])


def test_strided_inputs_and_skipped_slots():
    """k/v as views into a fused qkv buffer (token stride > Hkv*D); -1 slots skip."""
    rng = np.random.default_rng(1)
    T, H, D, bs, nb = 96, 4, 128, 16, 8
    qkv = _bf16(rng.standard_normal((T, 3 * H * D)).astype(np.float32) * 2)
    k = qkv[:, H * D: 2 * H * D].view(T, H, D)
    v = qkv[:, 2 * H * D:].view(T, H, D)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[::7] = -1
    sentinel = rng.integers(0, 256, (nb, 2, H, bs, nk.full_dim(D))).astype(np.uint8)
    cache = torch.from_numpy(sentinel).to(DEV)
    kd, vd = k.to(DEV), v.to(DEV)       # keeps the strided view on the device
    qkvd = qkv.to(DEV)
    kd = qkvd[:, H * D: 2 * H * D].view(T, H, D)
    vd = qkvd[:, 2 * H * D:].view(T, H, D)
    assert kd.stride(0) == 3 * H * D
    nk.quantize_append_paged(kd, vd, cache, torch.from_numpy(slots).to(DEV), dev_scalar(0.01),
                             dev_scalar(0.02))
    torch.cuda.synchronize()
    ref = _oracle_write(k.contiguous(), v.contiguous(), slots, nb, bs, 0.01, 0.02, sentinel)
    assert np.array_equal(cache.cpu().numpy(), ref)


def test_bad_slot_is_flagged_and_skipped():
    rng = np.random.default_rng(2)
    T, H, D, bs, nb = 8, 2, 64, 16, 2
    k = _bf16(rng.standard_normal((T, H, D)).astype(np.float32))
    slots = np.arange(T, dtype=np.int64)
    slots[3] = nb * bs + 5
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = _gpu_write(k, k, slots, nb, bs, 1.0, 1.0, status=status)
    assert int(status.item()) & nk.DEV_BAD_SLOT
    ok = slots.copy()
    ok[3] = -1
    want = _oracle_write(k, k, ok, nb, bs, 1.0, 1.0)
    assert np.array_equal(got, want)


def test_empty_append_is_noop():
    cache = nk.alloc_kv_cache(2, 16, 2, 64, DEV)
    e = torch.empty((0, 2, 64), dtype=torch.bfloat16, device=DEV)
    nk.quantize_append_paged(e, e, cache, torch.empty(0, dtype=torch.int64, device=DEV),
                             dev_scalar(1.0), dev_scalar(1.0))
    assert int(cache.sum()) == 0


@pytest.mark.parametrize("D,bs", [(64, 16), (128, 32), (256, 16)])
def test_dequantize_paged_bit_exact(D, bs):
    rng = np.random.default_rng(D + bs)
    H, nb = 3, 12
    cache_np = rng.integers(0, 256, (nb, 2, H, bs, nk.full_dim(D))).astype(np.uint8)
    cache_np[..., D // 2:] = rng.integers(0, 0x7E, (nb, 2, H, bs, D // 16))  # finite scales
    ids = np.array([5, 0, 11, 5, 7], np.int32)
    gk, gv = 0.37, 2.5
    want = oracle.dequantize_paged(cache_np, ids, gk, gv)
    cache = torch.from_numpy(cache_np).to(DEV)
    kvs = torch.tensor([gk, gv], dtype=torch.float32, device=DEV)
    out = nk.dequantize_paged(cache, torch.from_numpy(ids).to(DEV), kvs)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), want)


def test_dequantize_skips_out_of_range_ids():
    cache = nk.alloc_kv_cache(2, 16, 1, 64, DEV)
    out = torch.full((2, 2, 1, 16, 64), 7.0, dtype=torch.bfloat16, device=DEV)
    ids = torch.tensor([1, 9], dtype=torch.int32, device=DEV)
    nk.dequantize_paged(cache, ids, torch.ones(2, device=DEV), out=out)
    torch.cuda.synchronize()
    assert float(out[0].abs().max()) == 0.0 and float(out[1].min()) == 7.0
