"""Pins for the CPU oracle: each checks it against something other than itself.

Sources: the NVFP4 KV-cache pages ("FlashInfer backend adds end-to-end NVFP4 KV
cache support": cache shape and HND test construction; "Move NVFP4 GEMM
management into NvFp4LinearKernel": packed FP4 pairs, E4M3 scale per 16) and
the method statement (E4M3(amax/(6*global)) then RNE onto the E2M1 grid).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ formats
def test_e2m1_grid_matches_pages():
    with open(os.path.join(GOLDEN, "e2m1_grid.txt")) as f:
        grid = [float(x) for x in [ln for ln in f if not ln.startswith("#")][0].split()]
    assert [oracle.e2m1_decode(c) for c in range(8)] == grid
    for c in range(8):
        v = oracle.e2m1_decode(c | 8)
        assert v == -grid[c] and math.copysign(1.0, v) == -1.0


def test_e4m3_decode_all_codes_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(got) and math.isnan(ref[c])
        else:
            assert got == ref[c], hex(c)
    assert oracle.e4m3_decode(0x7E) == 448.0           # largest finite, the 448 of amax/(6*448)
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9        # smallest subnormal


def _e4m3_probe_values():
    rng = np.random.default_rng(11)
    mags = [oracle.e4m3_decode(c) for c in range(127)]
    vals = []
    for a, b in zip(mags[:-1], mags[1:]):
        mid = np.float32((a + b) / 2)
        vals += [a, b, float(mid), float(np.nextafter(mid, np.float32(0))),
                 float(np.nextafter(mid, np.float32(1e9)))]
    vals += list(np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)).astype(np.float32))
    vals += [0.0, 2.0 ** -10, 2.0 ** -11, 1e-30, 448.0]
    vals = np.array(vals, np.float32)
    return np.concatenate([vals, -vals])


def test_e4m3_encode_rne_vs_torch_in_range():
    vals = _e4m3_probe_values()
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def test_e4m3_encode_satfinite():
    for x in (448.0, 449.0, 464.0, 1e6, float(np.float32(3.4e38)), float("inf")):
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def _brute_nearest_e2m1(q: Fraction) -> int:
    """Nearest E2M1 grid value to the exact rational q; ties -> even code."""
    grid = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]
    a = abs(q)
    if a >= 6:
        code = 7
    else:
        dists = [abs(a - g) for g in grid]
        best = min(dists)
        cands = [i for i, d in enumerate(dists) if d == best]
        code = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
    return code


def test_e2m1_encode_every_bf16_magnitude_below_8():
    # every positive finite bf16 pattern up to 8, against exact-rational brute force
    bits = np.arange(0, 0x4100, dtype=np.uint32)          # 0x4100 = bf16(8.0)
    vals = (bits << 16).view(np.float32)
    for v in vals:
        c = oracle.e2m1_encode(float(v))
        assert c == _brute_nearest_e2m1(Fraction(float(v))), float(v)
        cn = oracle.e2m1_encode(-float(v))
        assert cn == (_brute_nearest_e2m1(Fraction(float(v))) | 8), -float(v)


def test_element_codes_exact_rational_at_unit_global_scale():
    """At g = 1 the fp32 division x / S cannot move x/S across a tie or a
    rounding threshold: bf16 x has 8 significant bits, S (E4M3) 4, so the
    decision equals exact-rational RNE. Checked over bf16 x in groups with
    random scales: the row writer vs Fractions."""
    rng = np.random.default_rng(5)
    for trial in range(400):
        sb = int(rng.integers(1, 0x7F))          # positive finite scale byte
        S = oracle.e4m3_decode(sb)
        # elements on/near the grid times S, plus random bf16 values, all <= 6*S
        x = (rng.choice([0, .5, 1, 1.5, 2, 3, 4, 6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5], 16)
             * rng.choice([-1, 1], 16) * S)
        x = np.where(rng.random(16) < 0.3, rng.uniform(-6 * S, 6 * S, 16), x)
        x[0] = 6 * S                              # amax = 6*S so the scale reproduces sb
        xb = _bf16_bits(x.astype(np.float32))
        xf = xb.astype(np.uint32) << 16
        xf = xf.view(np.float32)
        if float(np.abs(xf).max()) != 6 * S:
            continue                              # 6*S not representable in bf16
        row = oracle.quantize_row(xb, 1.0)
        assert row[8] == sb
        for i in range(16):
            code = (row[i // 2] >> (4 * (i % 2))) & 0xF
            want = _brute_nearest_e2m1(Fraction(float(xf[i])) / Fraction(S))
            if math.copysign(1.0, float(xf[i])) < 0:
                want |= 8
            assert code == want, (trial, i, float(xf[i]), S)


def test_f32_to_bf16_vs_torch():
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        ((rng.integers(0, 2 ** 16, 2000, dtype=np.uint32) << 16) | 0x8000).view(np.float32),  # ties
        np.array([0.0, -0.0, 1e-40, 3.3e38, -3.3e38], np.float32)])
    vals = vals[np.isfinite(vals)]                       # NaN payloads are unspecified
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)
    for b in (0x3F80, 0xC2F7, 0x0001, 0x7F7F):
        assert oracle.bf16_to_f32(b) == float(torch.tensor([b], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()[0])


# ------------------------------------------------------------------ writer
def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "worked_rows.txt")) as f:
        for ln in f:
            if ln.startswith("#") or not ln.strip():
                continue
            g, xs, hx = [p.strip() for p in ln.split(";")]
            rows.append((float(g), [float(x) for x in xs.split()], bytes.fromhex(hx)))
    return rows


@pytest.mark.parametrize("case", range(8))
def test_writer_hand_worked_rows(case):
    g, xs, want = _golden_rows()[case]
    xb = _bf16_bits(np.array(xs, np.float32))
    assert np.array_equal(((xb.astype(np.uint32) << 16).view(np.float32)), np.array(xs, np.float32))
    row = oracle.quantize_row(xb, g)
    assert bytes(row) == want, (case, bytes(row).hex(" "), want.hex(" "))


def test_full_dim_and_capacity():
    # get_kv_cache_shape: last dim head_size/2 + head_size/16
    assert oracle.full_dim(64) == 36 and oracle.full_dim(128) == 72 and oracle.full_dim(256) == 144
    assert oracle.full_dim(100) < 0 and oracle.full_dim(0) < 0
    # "about 3x" KV capacity vs a 16-bit cache: 2*D bytes / full_dim bytes
    assert 3.0 <= (2 * 128) / oracle.full_dim(128) < 4.0


def test_round_trip_reproducible_rows():
    """Rows built as E2M1 code x E4M3 scale with a +-6*scale element in each
    group quantize back to exactly those codes and scales (low nibble =
    element 2j), and dequantize back to the same values."""
    rng = np.random.default_rng(9)
    for D in (16, 64, 128, 256):
        for trial in range(20):
            codes = rng.integers(0, 16, D).astype(np.uint8)
            sbs = rng.integers(1, 0x7F, D // 16).astype(np.uint8)
            for j in range(D // 16):
                codes[16 * j + rng.integers(0, 16)] = rng.choice([0x7, 0xF])
            vals = np.array([oracle.e2m1_decode(int(c)) * oracle.e4m3_decode(int(sbs[i // 16]))
                             for i, c in enumerate(codes)], np.float32)
            xb = _bf16_bits(vals)
            assert np.array_equal(((xb.astype(np.uint32) << 16).view(np.float32)), vals)
            row = oracle.quantize_row(xb, 1.0)
            packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
            # negative-zero codes (0x8) are kept only when the value is -0.0
            assert np.array_equal(row[D // 2:], sbs)
            assert np.array_equal(row[:D // 2], packed)
            cache = row.reshape(1, 1, 1, 1, -1).repeat(2, axis=1).copy()
            out = oracle.dequantize_paged(cache, np.array([0], np.int32), 1.0, 1.0)
            assert np.array_equal(out[0, 0, 0, 0], xb)


def test_writer_untouched_and_hnd_layout():
    """Sentinel-filled HND cache: only rows named by non-negative slots change,
    and each written row is found where the pages' test construction puts it:
    HND storage (NB, 2, H, bs, F) viewed through permute(0, 1, 3, 2, 4) as NHD."""
    rng = np.random.default_rng(21)
    NB, H, bs, D = 12, 3, 16, 64
    F = oracle.full_dim(D)
    T = 40
    k = _bf16_bits(rng.standard_normal((T, H, D)).astype(np.float32) * 3)
    v = _bf16_bits(rng.standard_normal((T, H, D)).astype(np.float32) * 0.2)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[rng.choice(T, 6, replace=False)] = -1
    sentinel = rng.integers(0, 256, (NB, 2, H, bs, F)).astype(np.uint8)
    cache = sentinel.copy()
    bad = oracle.quantize_append_paged(k, v, cache, slots, 0.7, 1.3, bs)
    assert bad == 0
    nhd = torch.from_numpy(cache).permute(0, 1, 3, 2, 4)            # [NB][2][bs][H][F]
    touched = np.zeros((NB, bs), bool)
    for t in range(T):
        if slots[t] < 0:
            continue
        blk, off = divmod(int(slots[t]), bs)
        touched[blk, off] = True
        for h in range(H):
            assert np.array_equal(nhd[blk, 0, off, h].numpy(), oracle.quantize_row(k[t, h].copy(), 0.7))
            assert np.array_equal(nhd[blk, 1, off, h].numpy(), oracle.quantize_row(v[t, h].copy(), 1.3))
    untouched = ~touched
    for blk in range(NB):
        for off in range(bs):
            if untouched[blk, off]:
                assert np.array_equal(cache[blk, :, :, off], sentinel[blk, :, :, off])
    # a slot beyond the cache is reported and writes nothing
    c2 = sentinel.copy()
    assert oracle.quantize_append_paged(k[:1].copy(), v[:1].copy(), c2,
                                        np.array([NB * bs], np.int64), 1.0, 1.0, bs) == 1
    assert np.array_equal(c2, sentinel)


# ------------------------------------------------------------------ attention
def _hand_cache(rng, NB, H, bs, D):
    """Random codes/scales packed by hand (independent of the writer); returns
    the cache bytes and the dense dequantized values xhat[NB][2][H][bs][D]."""
    F = D // 2 + D // 16
    codes = rng.integers(0, 16, (NB, 2, H, bs, D)).astype(np.uint8)
    sbs = rng.integers(0x10, 0x50, (NB, 2, H, bs, D // 16)).astype(np.uint8)
    cache = np.zeros((NB, 2, H, bs, F), np.uint8)
    cache[..., :D // 2] = codes[..., 0::2] | (codes[..., 1::2] << 4)
    cache[..., D // 2:] = sbs
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e2 = grid[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sc = torch.from_numpy(sbs).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    xhat = e2 * np.repeat(sc, 16, axis=-1)
    return cache, xhat


def _dense_attention(q, xhat, table, seq_lens, q_lens, G, bs, gk, gv, sm_scale):
    """softmax(Q K^T) V by matrix ops on gathered dense rows."""
    out = []
    qpos = 0
    for b, (L, ql) in enumerate(zip(seq_lens, q_lens)):
        n = np.arange(L)
        blk = table[b, n // bs]
        K = xhat[blk, 0, :, n % bs] * gk           # [L][H][D]
        V = xhat[blk, 1, :, n % bs] * gv
        for r in range(ql):
            last = L - ql + r
            for hq in range(q.shape[1]):
                h = hq // G
                z = sm_scale * (K[: last + 1, h] @ q[qpos + r, hq])
                p = np.exp(z - z.max())
                out.append((p / p.sum()) @ V[: last + 1, h])
        qpos += ql
    return np.array(out).reshape(q.shape[0], q.shape[1], -1)


@pytest.mark.parametrize("D,bs,G,q_lens,seq_lens", [
    (64, 16, 2, [1, 1], [37, 100]),
    (128, 16, 1, [1, 1, 1], [1, 16, 17]),
    (64, 32, 4, [5, 1, 3], [40, 9, 64]),
    (256, 16, 8, [1, 2], [23, 50]),
])
def test_attention_vs_dense_softmax(D, bs, G, q_lens, seq_lens):
    rng = np.random.default_rng(D + bs + G)
    Hkv = 2
    Hq = G * Hkv
    need = sum(-(-L // bs) for L in seq_lens)
    NB = need + 3
    cache, xhat = _hand_cache(rng, NB, Hkv, bs, D)
    perm = rng.permutation(NB).astype(np.int32)
    width = max(-(-L // bs) for L in seq_lens)
    table = np.zeros((len(seq_lens), width), np.int32)
    pos = 0
    for b, L in enumerate(seq_lens):
        nblk = -(-L // bs)
        table[b, :nblk] = perm[pos:pos + nblk]
        pos += nblk
    Tq = sum(q_lens)
    qf = rng.standard_normal((Tq, Hq, D)).astype(np.float32) * 0.3
    qb = _bf16_bits(qf)
    qd = ((qb.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    indptr = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    gk, gv = float(np.float32(0.05)), float(np.float32(1.7))  # fp32 values, as the ABI takes them
    o64, o8, o16 = oracle.paged_attention(qb, cache, table, np.array(seq_lens, np.int32),
                                          indptr, gk, gv, 0.0, 0.5)
    ref = _dense_attention(qd, xhat, table, seq_lens, q_lens, G, bs, gk, gv, 1 / math.sqrt(D))
    np.testing.assert_allclose(o64, ref, rtol=1e-11, atol=1e-12)
    # FP8 epilogue: E4M3(o / o_scale), then bf16(fl32(dec * o_scale))
    want8 = torch.from_numpy((ref / 0.5).astype(np.float32)).clamp(-448, 448).to(torch.float8_e4m3fn)
    mism = (want8.view(torch.uint8).numpy() != o8)
    # exact fp64 vs rounded-to-fp32 reference may differ only at an exact tie: none expected
    assert mism.sum() == 0
    deq = torch.from_numpy(o8.copy()).view(torch.float8_e4m3fn).float() * torch.tensor(0.5, dtype=torch.float32)
    assert np.array_equal(deq.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16), o16)


def test_attention_special_cases():
    rng = np.random.default_rng(4)
    D, bs, H = 64, 16, 1
    cache, xhat = _hand_cache(rng, 4, H, bs, D)
    table = np.array([[2, 0, 3]], np.int32)
    # one key: o = Vhat_0 exactly
    q = _bf16_bits(rng.standard_normal((1, 1, D)).astype(np.float32))
    o64, _, _ = oracle.paged_attention(q, cache, table, np.array([1], np.int32), None, 1.0, 1.0)
    assert np.array_equal(o64[0, 0], xhat[2, 1, 0, 0])
    # q = 0: uniform weights -> mean of Vhat over the window
    q0 = np.zeros((1, 1, D), np.uint16)
    o64, _, _ = oracle.paged_attention(q0, cache, table, np.array([40], np.int32), None, 1.0, 1.0)
    n = np.arange(40)
    mean = xhat[table[0, n // bs], 1, 0, n % bs].mean(axis=0)
    np.testing.assert_allclose(o64[0, 0], mean, rtol=1e-13, atol=1e-15)
    # two keys with logits 1 and 0 (sm_scale 1): weights e/(e+1), 1/(e+1)
    c2 = np.zeros((1, 2, 1, bs, D // 2 + D // 16), np.uint8)
    c2[0, 0, 0, 0, 0] = 0x02          # K0 = [1, 0, ...] (code 2 = 1.0), scale 1.0
    c2[0, 0, 0, 0, D // 2] = 0x38
    c2[0, 1, 0, 0, 0] = 0x07          # V0 = [6, 0, ...]
    c2[0, 1, 0, 0, D // 2] = 0x38
    c2[0, 1, 0, 1, 0] = 0x70          # V1 = [0, 6, ...]
    c2[0, 1, 0, 1, D // 2] = 0x38
    qa = _bf16_bits(np.eye(1, D, dtype=np.float32).reshape(1, 1, D))
    o64, _, _ = oracle.paged_attention(qa, c2, np.array([[0]], np.int32), np.array([2], np.int32),
                                       None, 1.0, 1.0, sm_scale=1.0)
    e = math.e
    assert o64[0, 0, 0] == pytest.approx(6 * e / (e + 1), rel=1e-15)
    assert o64[0, 0, 1] == pytest.approx(6 / (e + 1), rel=1e-15)
    # a prefill row with an empty window (q_len > L) gives zeros
    qq = _bf16_bits(rng.standard_normal((3, 1, D)).astype(np.float32))
    o64, o8, _ = oracle.paged_attention(qq, cache, table, np.array([2], np.int32),
                                        np.array([0, 3], np.int32), 1.0, 1.0)
    assert np.all(o64[0] == 0) and np.any(o64[1] != 0) and np.any(o64[2] != 0)
    assert np.array_equal(o64[1, 0], xhat[2, 1, 0, 0])          # row 1 sees key 0 only


@pytest.mark.parametrize("D,bs,H", [(64, 16, 2), (128, 32, 3), (256, 16, 1)])
def test_dequantize_paged_scales_and_block_list(D, bs, H):
    """The paged dequantize helper ("FlashInfer NVFP4 KV serving on pre-SM100
    GPUs", quick answer) on a hand-packed multi-block cache: K pages take
    k_scale and V pages v_scale (two different non-unit values), and out[i]
    holds the pages of block_ids[i] for a repeated, unordered id list.
    Expected bits: the hand-packed xhat (exact in fp32), times g in fp32,
    rounded to bf16 by torch."""
    rng = np.random.default_rng(D + bs + H)
    NB = 5
    cache, xhat = _hand_cache(rng, NB, H, bs, D)
    ids = np.array([3, 0, 3, 4, 1], np.int32)
    gk, gv = float(np.float32(0.37)), float(np.float32(2.5))
    got = oracle.dequantize_paged(cache, ids, gk, gv)
    x32 = torch.from_numpy(xhat[ids].astype(np.float32))            # exact: <= 6 significant bits
    assert np.array_equal(x32.double().numpy(), xhat[ids])
    g = torch.tensor([gk, gv], dtype=torch.float32).view(1, 2, 1, 1, 1)
    want = (x32 * g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert got.shape == (len(ids), 2, H, bs, D)
    assert np.array_equal(got, want)
    # a K/V scale swap or a scale dropped would change the bits
    swapped = (x32 * g.flip(1)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert not np.array_equal(got, swapped)


# ------------------------------------------------------------- activations
def _golden_sf_positions():
    rows = []
    with open(os.path.join(GOLDEN, "sf_swizzle_positions.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                cols, r, c, pos = (int(x) for x in line.split()[:4])
                rows.append((cols, r, c, pos))
    return rows


def test_activation_sf_positions_hand_worked():
    """Swizzled scale positions worked by hand (tests/golden)."""
    golden = _golden_sf_positions()
    assert len(golden) >= 8
    for cols, r, c, pos in golden:
        assert oracle.act_sf_index(r, c, cols) == pos, (cols, r, c)


@pytest.mark.parametrize("rows,cols", [(200, 96), (128, 64), (300, 4096 // 8), (1, 16)])
def test_activation_sf_swizzle_vs_tile_transpose(rows, cols):
    """The swizzled scales equal the plain [rows][cols/16] scales, zero-padded to
    (128k rows, 4k columns), viewed as [row bands][4 groups of 32 rows][32]
    [column tiles][4] and transposed to [band][column tile][32][4 groups][4]."""
    rng = np.random.default_rng(rows + cols)
    x = _bf16_bits(rng.standard_normal((rows, cols)).astype(np.float32) * 3)
    inv = float(np.float32(448 * 6 / 9.0))
    fp4_s, sf_s = oracle.quantize_activation(x, inv, swizzled=True)
    fp4_p, sf_p = oracle.quantize_activation(x, inv, swizzled=False)
    assert np.array_equal(fp4_s, fp4_p)
    pr, pc = -(-rows // 128) * 128, -(-(cols // 16) // 4) * 4
    pad = np.zeros((pr, pc), np.uint8)
    pad[:rows, :cols // 16] = sf_p
    want = pad.reshape(pr // 128, 4, 32, pc // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    assert np.array_equal(sf_s, want)


def test_activation_rows_are_the_kv_row_codec():
    """Each activation row is quantized exactly as a KV-cache row with the
    global scale g = fl32(1 / inv): packed codes, then the row's scales."""
    rng = np.random.default_rng(5)
    rows, cols = 37, 256
    x = _bf16_bits(rng.standard_normal((rows, cols)).astype(np.float32))
    inv = float(np.float32(2688.0 / 4.25))
    g = float(np.float32(1.0) / np.float32(inv))
    fp4, sf = oracle.quantize_activation(x, inv, swizzled=False)
    for r in range(rows):
        row = oracle.quantize_row(np.ascontiguousarray(x[r]), g)
        assert np.array_equal(fp4[r], row[:cols // 2]) and np.array_equal(sf[r], row[cols // 2:])
    # g is the inverse of inv, not inv: the scales would change with inv itself
    alt = oracle.quantize_row(np.ascontiguousarray(x[0]), inv)
    assert not np.array_equal(sf[0], alt[cols // 2:])


# ------------------------------------------------------------- FP8 KV cache
def test_fp8kv_writer_vs_torch_cast():
    """FP8 rows: E4M3 RNE of fl32(x / g), saturating at 448, checked against
    torch's float8_e4m3fn cast of the same fp32 quotient (clamped first: torch
    does not saturate); untouched rows keep their sentinel bytes."""
    rng = np.random.default_rng(12)
    T, H, D, bs, NB = 40, 2, 64, 16, 6
    kf = (rng.standard_normal((T, H, D)) * rng.choice([0.01, 1, 50], (T, H, 1))).astype(np.float32)
    vf = rng.standard_normal((T, H, D)).astype(np.float32)
    k, v = _bf16_bits(kf), _bf16_bits(vf)
    gk, gv = float(np.float32(0.013)), float(np.float32(0.7))
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[::7] = -1
    cache = np.full((NB, 2, H, bs, D), 0xC3, np.uint8)
    oracle.fp8kv_quantize_append_paged(k, v, cache, slots, gk, gv, bs)
    for x, g, kv in ((k, gk, 0), (v, gv, 1)):
        xf = torch.from_numpy((x.astype(np.uint32) << 16).view(np.float32))
        q = (xf / torch.tensor(g, dtype=torch.float32)).clamp(-448, 448)
        want = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        for t in range(T):
            if slots[t] < 0:
                continue
            blk, off = divmod(int(slots[t]), bs)
            assert np.array_equal(cache[blk, kv, :, off], want[t])
    live = {divmod(int(s), bs) for s in slots if s >= 0}
    for blk in range(NB):
        for off in range(bs):
            if (blk, off) not in live:
                assert (cache[blk, :, :, off] == 0xC3).all()


def test_fp8kv_attention_vs_dense_softmax():
    """FP8-row attention: fp64 oracle vs dense softmax(QK^T)V over hand-packed
    E4M3 rows decoded by torch, with GQA, prefill rows and g != 1."""
    rng = np.random.default_rng(13)
    D, bs, Hkv, G = 64, 16, 2, 2
    seq_lens, q_lens = [37, 100], [3, 1]
    NB = sum(-(-L // bs) for L in seq_lens) + 2
    codes = rng.integers(0, 256, (NB, 2, Hkv, bs, D)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                     # no NaN codes
    xhat = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    perm = rng.permutation(NB).astype(np.int32)
    table = np.zeros((2, 7), np.int32)
    table[0, :3], table[1, :7] = perm[:3], perm[3:10]
    qf = rng.standard_normal((sum(q_lens), Hkv * G, D)).astype(np.float32) * 0.05
    qb = _bf16_bits(qf)
    qd = ((qb.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    indptr = np.array([0, 3, 4], np.int32)
    gk, gv = float(np.float32(0.02)), float(np.float32(1.3))
    o64, _, _ = oracle.paged_attention(qb, codes, table, np.array(seq_lens, np.int32), indptr,
                                       gk, gv, 0.0, 1.0, kv_format=oracle.KV_FP8)
    ref = _dense_attention(qd, xhat, table, seq_lens, q_lens, G, bs, gk, gv, 1 / math.sqrt(D))
    np.testing.assert_allclose(o64, ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------ NVFP4-quantized queries (block-scaled QK^T)
@pytest.mark.parametrize("amax,g", [
    (2688.0, 1.0),            # amax / (6 g) = 448 exactly
    (2704.0, 2.0),            # just above: the next power of two
    (1.0, 2.0 ** -11),        # 1 / (6 * 2^-11) = 341.3 <= 448; 2^-12 gives 682.7
    (1.3125, 2.0 ** -11),     # = 2688 * 2^-11: the bound itself
    (1.3203125, 2.0 ** -10),  # one bf16 step above it
    (0.0, 1.0),               # all-zero row
])
def test_q_row_global_hand_worked(amax, g):
    row = _bf16_bits(np.array([amax, -0.5 * amax] + [0.0] * 14, np.float32))
    assert oracle.q_row_global(row) == g


def _qfp4_case(rng, D, bs, G, q_lens, seq_lens):
    Hkv = 2
    need = sum(-(-L // bs) for L in seq_lens)
    NB = need + 2
    cache, _ = _hand_cache(rng, NB, Hkv, bs, D)
    perm = rng.permutation(NB).astype(np.int32)
    width = max(-(-L // bs) for L in seq_lens)
    table = np.zeros((len(seq_lens), width), np.int32)
    pos = 0
    for b, L in enumerate(seq_lens):
        nblk = -(-L // bs)
        table[b, :nblk] = perm[pos:pos + nblk]
        pos += nblk
    indptr = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    return cache, table, np.array(seq_lens, np.int32), indptr, G * Hkv


@pytest.mark.parametrize("D", [128, 256])
def test_qfp4_attention_is_attention_over_the_quantized_queries(D):
    """Prefill rows: the NVFP4-Q attention equals plain attention over q-hat, the
    queries round-tripped through the activation codec (pinned above) with
    inv = 1 / g per row; q-hat (<= 6 significant bits) is exact in bf16. Decode
    rows (one query) keep their bf16 query."""
    rng = np.random.default_rng(90 + D)
    q_lens, seq_lens = [3, 1, 5], [40, 33, 70]
    cache, table, sl, indptr, Hq = _qfp4_case(rng, D, 16, 4, q_lens, seq_lens)
    Tq = sum(q_lens)
    q = _bf16_bits(rng.standard_normal((Tq, Hq, D)).astype(np.float32) * 0.7)
    qhat = q.copy()
    for b in range(len(q_lens)):
        if q_lens[b] == 1:
            continue
        for t in range(indptr[b], indptr[b + 1]):
            for h in range(Hq):
                g = oracle.q_row_global(np.ascontiguousarray(q[t, h]))
                fp4, sf = oracle.quantize_activation(np.ascontiguousarray(q[t, h][None]),
                                                     1.0 / g, swizzled=False)
                codes = np.empty(D, np.uint8)
                codes[0::2] = fp4[0] & 0xF
                codes[1::2] = fp4[0] >> 4
                grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
                e2 = grid[codes & 7] * np.where(codes & 8, -1.0, 1.0)
                sc = torch.from_numpy(sf[0].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
                vals = e2 * np.repeat(sc, 16) * g
                qhat[t, h] = _bf16_bits(vals.astype(np.float32))
                back = (qhat[t, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                assert np.array_equal(back, vals)            # exact in bf16
    gk, gv = float(np.float32(0.05)), float(np.float32(1.7))
    got = oracle.paged_attention(q, cache, table, sl, indptr, gk, gv, 0.0, 0.5, q_fp4=True)
    want = oracle.paged_attention(qhat, cache, table, sl, indptr, gk, gv, 0.0, 0.5)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    plain = oracle.paged_attention(q, cache, table, sl, indptr, gk, gv, 0.0, 0.5)
    dec = indptr[1]  # the decode row of sequence 1
    assert np.array_equal(got[0][dec], plain[0][dec])
    assert not np.array_equal(got[0], plain[0])      # the prefill rows did change


def test_qfp4_identity_on_representable_queries():
    """Queries on the E2M1 grid times per-group powers of two (each group holding
    a 6) are fixed points of the quantizer: the NVFP4-Q attention equals the plain
    one exactly."""
    rng = np.random.default_rng(17)
    D = 256
    q_lens, seq_lens = [4, 2], [50, 21]
    cache, table, sl, indptr, Hq = _qfp4_case(rng, D, 16, 2, q_lens, seq_lens)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    Tq = sum(q_lens)
    vals = grid[rng.integers(0, 8, (Tq, Hq, D))] * np.where(rng.random((Tq, Hq, D)) < 0.5, -1, 1)
    vals = vals.astype(np.float32)
    vals[..., ::16] = 6.0                                   # each group's amax is 6 * 2^j
    vals *= np.repeat(2.0 ** (np.arange(D // 16) % 3), 16).astype(np.float32)
    q = _bf16_bits(vals)
    gk, gv = float(np.float32(0.05)), float(np.float32(1.7))
    got = oracle.paged_attention(q, cache, table, sl, indptr, gk, gv, 0.0, 0.5, q_fp4=True)
    want = oracle.paged_attention(q, cache, table, sl, indptr, gk, gv, 0.0, 0.5)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
