"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point the header declares, and rejects bad arguments before any
CUDA call."""
import ctypes
import os
import re

import pytest

import nvfp4_quantized_paged_append_b200 as nk
from nvfp4_quantized_paged_append_b200 import build as nkbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nkbuild.build()
    return nk.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "nvfp4kv.h")).read()
    return re.findall(r"NVFP4KV_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", src)


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 6
    for n in names:
        assert hasattr(L, n), n


def test_full_dim(L):
    assert [nk.full_dim(d) for d in (16, 64, 128, 256)] == [9, 36, 72, 144]
    assert nk.full_dim(0) == -1 and nk.full_dim(100) == -1 and nk.full_dim(-16) == -1


def test_status_strings(L):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert nk.status_string(s) and nk.status_string(s) != "unknown status"
    assert nk.status_string(-99) == "unknown status"


def test_status_from_device_bits(L):
    """Device status bits map to the read-back codes: a timeout outranks the
    bounds bits; no bit is NVFP4_OK."""
    f = L.nvfp4_status_from_bits
    assert f(0) == nk.NVFP4_OK
    for b in (nk.DEV_BAD_SLOT, nk.DEV_BAD_BLOCK, nk.DEV_BAD_QLEN,
              nk.DEV_BAD_SLOT | nk.DEV_BAD_BLOCK):
        assert f(b) == nk.NVFP4_ERR_DEVICE_BOUNDS
    for b in (nk.DEV_TIMEOUT, nk.DEV_TIMEOUT | nk.DEV_BAD_BLOCK):
        assert f(b) == nk.NVFP4_ERR_DEVICE_TIMEOUT


def test_status_readback_and_probe_validation(L):
    """Null or misaligned status words and out-of-range poll limits are
    rejected before any CUDA call."""
    bits = ctypes.c_uint32(7)
    assert L.nvfp4_read_device_status(None, ctypes.byref(bits), 0, None) == nk.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_read_device_status(ctypes.c_void_p(0x1002), None, 0, None) == \
        nk.NVFP4_ERR_INVALID_ARG
    assert bits.value == 7                                   # untouched on rejection
    assert L.nvfp4_wait_timeout_probe(None, 100, None) == nk.NVFP4_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x1000)
    assert L.nvfp4_wait_timeout_probe(fake, 0, None) == nk.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_wait_timeout_probe(fake, (1 << 24) + 1, None) == nk.NVFP4_ERR_INVALID_ARG


def _append(L, **kw):
    a = dict(k=None, v=None, ks=128 * 8, vs=128 * 8, T=4, H=8, D=128, cache=None, nb=10, bs=16,
             slots=None, kscale=None, vscale=None, status=None, stream=None)
    a.update(kw)
    P = ctypes.c_void_p
    return L.nvfp4_quantize_append_paged(a["k"], a["v"], a["ks"], a["vs"], a["T"], a["H"], a["D"],
                                         a["cache"], a["nb"], a["bs"], a["slots"], a["kscale"],
                                         a["vscale"], a["status"], a["stream"])


def test_append_validation(L):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    assert _append(L) == nk.NVFP4_ERR_INVALID_ARG                      # null pointers
    assert _append(L, T=0) == nk.NVFP4_OK                              # empty: no-op
    assert _append(L, D=100) == nk.NVFP4_ERR_INVALID_ARG
    assert _append(L, D=96) == nk.NVFP4_ERR_UNSUPPORTED
    assert _append(L, bs=8) == nk.NVFP4_ERR_UNSUPPORTED
    assert _append(L, T=-1) == nk.NVFP4_ERR_INVALID_ARG
    full = dict(k=fake, v=fake, cache=fake, slots=fake, kscale=fake, vscale=fake)
    assert _append(L, ks=100, **full) == nk.NVFP4_ERR_INVALID_ARG      # stride < row
    assert _append(L, ks=1028, **full) == nk.NVFP4_ERR_INVALID_ARG     # stride not 16-B multiple
    assert _append(L, **dict(full, k=ctypes.c_void_p(0x1002))) == nk.NVFP4_ERR_INVALID_ARG  # misaligned


def _attn(L, **kw):
    a = dict(q=None, qs=16 * 128, tq=4, hq=16, cache=None, nb=10, bs=16, hkv=8, D=128, bt=None,
             mb=4, sl=None, qo=None, B=4, mq=1, kvs=None, sm=0.0, o8=None, osc=None, o16=None,
             o32=None, ws=None, wsb=0, stream=None)
    a.update(kw)
    return L.nvfp4_paged_attention(a["q"], a["qs"], a["tq"], a["hq"], a["cache"], a["nb"], a["bs"],
                                   a["hkv"], a["D"], a["bt"], a["mb"], a["sl"], a["qo"], a["B"],
                                   a["mq"], a["kvs"], a["sm"], a["o8"], a["osc"], a["o16"],
                                   a["o32"], a["ws"], a["wsb"], a["stream"])


def test_attention_validation(L):
    fake = ctypes.c_void_p(0x1000)
    full = dict(q=fake, cache=fake, bt=fake, sl=fake, kvs=fake, o8=fake, osc=fake)
    assert _attn(L) == nk.NVFP4_ERR_INVALID_ARG
    assert _attn(L, B=0) == nk.NVFP4_OK
    assert _attn(L, hq=12) == nk.NVFP4_ERR_INVALID_ARG          # Hq % Hkv
    assert _attn(L, hq=128) == nk.NVFP4_ERR_UNSUPPORTED         # G = 16
    assert _attn(L, D=96, qs=16 * 96) == nk.NVFP4_ERR_UNSUPPORTED
    assert _attn(L, mq=4) == nk.NVFP4_ERR_INVALID_ARG           # prefill needs qo_indptr
    assert _attn(L, tq=2) == nk.NVFP4_ERR_INVALID_ARG           # decode needs one q per seq
    assert _attn(L, **full) == nk.NVFP4_ERR_WORKSPACE           # no workspace
    need = nk.workspace_size(4, 16, 8, 128)
    assert need > 0 and need % 256 == 0
    assert _attn(L, ws=ctypes.c_void_p(0x100000), wsb=need - 1, **full) == nk.NVFP4_ERR_WORKSPACE
    assert _attn(L, ws=ctypes.c_void_p(0x100010), wsb=need, **full) == nk.NVFP4_ERR_WORKSPACE  # alignment


def test_workspace_size_monotone(L):
    assert nk.workspace_size(1, 16, 8, 128) <= nk.workspace_size(64, 16, 8, 128)
    assert nk.workspace_size(8, 64, 8, 256) > nk.workspace_size(8, 64, 8, 128)
    assert nk.workspace_size(-1, 16, 8, 128) == 0


def test_dequant_validation(L):
    P = ctypes.c_void_p
    f = L.nvfp4_dequantize_paged
    assert f(None, 10, 16, 8, 128, None, 4, None, None, None) == nk.NVFP4_ERR_INVALID_ARG
    assert f(None, 10, 16, 8, 128, None, 0, None, None, None) == nk.NVFP4_OK
    assert f(None, 10, 16, 8, 48, None, 4, None, None, None) == nk.NVFP4_ERR_UNSUPPORTED


def _attn_ex(L, flags, **kw):
    a = dict(q=None, qs=16 * 128, tq=4, hq=16, cache=None, nb=10, bs=16, hkv=8, D=128, bt=None,
             mb=4, sl=None, qo=None, B=4, mq=1, kvs=None, sm=0.0, o8=None, osc=None, o16=None,
             o32=None, ws=None, wsb=0, stream=None)
    a.update(kw)
    return L.nvfp4_paged_attention_ex(a["q"], a["qs"], a["tq"], a["hq"], a["cache"], a["nb"],
                                      a["bs"], a["hkv"], a["D"], a["bt"], a["mb"], a["sl"], a["qo"],
                                      a["B"], a["mq"], a["kvs"], a["sm"], a["o8"], a["osc"],
                                      a["o16"], a["o32"], a["ws"], a["wsb"], flags, a["stream"])


def test_attention_flags_and_output_alignment(L):
    """Unknown launch flags are rejected; the known flag changes no validation.
    Output pointers must allow the pair stores (fp8 2 B, bf16 4 B, fp32 8 B)."""
    fake = ctypes.c_void_p(0x1000)
    full = dict(q=fake, cache=fake, bt=fake, sl=fake, kvs=fake, o8=fake, osc=fake)
    ready = nk.NVFP4_ATTN_METADATA_READY
    assert _attn_ex(L, 0x8, **full) == nk.NVFP4_ERR_INVALID_ARG
    assert _attn_ex(L, nk.NVFP4_ATTN_QFP4, **full) == nk.NVFP4_ERR_UNSUPPORTED  # head size 128
    assert _attn_ex(L, nk.NVFP4_ATTN_HISTORY_READY, B=0) == nk.NVFP4_OK
    assert _attn_ex(L, nk.NVFP4_ATTN_HISTORY_READY | ready, **full) == nk.NVFP4_ERR_WORKSPACE
    assert _attn_ex(L, 0x80000000, B=0) == nk.NVFP4_ERR_INVALID_ARG
    assert _attn_ex(L, ready, B=0) == nk.NVFP4_OK
    assert _attn_ex(L, ready, **full) == nk.NVFP4_ERR_WORKSPACE      # same checks as flags = 0
    assert _attn_ex(L, 0, **full) == _attn(L, **full)
    ws = dict(ws=ctypes.c_void_p(0x100000), wsb=nk.workspace_size(4, 16, 8, 128))
    assert _attn(L, **dict(full, o8=ctypes.c_void_p(0x1001)), **ws) == nk.NVFP4_ERR_INVALID_ARG
    assert _attn(L, o16=ctypes.c_void_p(0x1002), **full, **ws) == nk.NVFP4_ERR_INVALID_ARG
    assert _attn(L, o32=ctypes.c_void_p(0x1004), **full, **ws) == nk.NVFP4_ERR_INVALID_ARG


def test_binding_rejects_bad_attention_tensors(L):
    """The Python binding checks shapes and dtypes (both attention calls) before
    any pointer reaches the library."""
    import torch
    cache = torch.zeros((4, 2, 2, 16, 72), dtype=torch.uint8)
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16)
    bt = torch.zeros((2, 3), dtype=torch.int32)
    sl = torch.ones(2, dtype=torch.int32)
    kvs = torch.ones(2)
    o8 = torch.zeros((2, 4, 128), dtype=torch.uint8)
    osc = torch.ones(1)
    ws = torch.zeros(1024, dtype=torch.uint8)
    for call in (lambda **kw: nk.paged_attention(workspace=ws, **kw),
                 lambda **kw: nk.paged_attention_noalloc(**kw)):
        def run(**over):
            args = dict(q=q, cache=cache, block_table=bt, seq_lens=sl, kv_scales=kvs, o_fp8=o8,
                        o_scale=osc)
            args.update(over)
            return call(**args)
        with pytest.raises(ValueError):
            run(q=q.float())                                   # q dtype
        with pytest.raises(ValueError):
            run(block_table=bt.long())                         # block table dtype
        with pytest.raises(ValueError):
            run(seq_lens=sl.long())                            # lengths dtype
        with pytest.raises(ValueError):
            run(o_fp8=torch.zeros((2, 4, 64), dtype=torch.uint8))  # output shape
        with pytest.raises(ValueError):
            run(cache=torch.zeros((4, 2, 2, 16, 70), dtype=torch.uint8))  # not a full_dim


def test_fused_decode_append_validation(L):
    """The fused decode step rejects bad arguments before any CUDA call."""
    P = ctypes.c_void_p
    fake = P(0x1000)

    def call(**kw):
        a = dict(q=fake, qs=16 * 128, hq=16, k=fake, v=fake, ks=8 * 128, vs=8 * 128, cache=fake,
                 nb=100, bs=16, hkv=8, d=128, bt=fake, mb=10, sl=fake, B=4, kvs=fake,
                 o8=fake, os=fake, ws=fake, wsb=1 << 30, flags=0)
        a.update(kw)
        return L.nvfp4_paged_decode_append(a["q"], a["qs"], a["hq"], a["k"], a["v"], a["ks"],
                                           a["vs"], a["cache"], a["nb"], a["bs"], a["hkv"],
                                           a["d"], a["bt"], a["mb"], a["sl"], a["B"], a["kvs"],
                                           0.0, a["o8"], a["os"], None, None, a["ws"], a["wsb"],
                                           a["flags"], None)
    assert call(k=None) == nk.NVFP4_ERR_INVALID_ARG
    assert call(v=None) == nk.NVFP4_ERR_INVALID_ARG
    assert call(ks=8 * 128 - 8) == nk.NVFP4_ERR_INVALID_ARG        # stride below a token row
    assert call(k=P(0x1008)) == nk.NVFP4_ERR_INVALID_ARG            # rows not 16-byte aligned
    assert call(flags=0x4) == nk.NVFP4_ERR_INVALID_ARG
    assert call(flags=0x3, B=0) == nk.NVFP4_OK                      # both known flags
    assert call(wsb=16) == nk.NVFP4_ERR_WORKSPACE
    assert call(d=96) == nk.NVFP4_ERR_UNSUPPORTED
    assert call(B=0) == nk.NVFP4_OK                                 # empty batch: nothing to do


def test_activation_validation(L):
    """The activation quantizer rejects bad shapes and pointers before any CUDA
    call; its scale-buffer size follows the padded tile layout."""
    fake = ctypes.c_void_p(0x1000)
    q = L.nvfp4_quantize_activation
    assert q(None, 4, 96, 96, fake, fake, fake, 1, None) == nk.NVFP4_ERR_INVALID_ARG
    assert q(fake, 4, 100, 104, fake, fake, fake, 1, None) == nk.NVFP4_ERR_INVALID_ARG   # cols % 16
    assert q(fake, 4, 96, 90, fake, fake, fake, 1, None) == nk.NVFP4_ERR_INVALID_ARG     # stride < cols
    assert q(fake, 4, 96, 100, fake, fake, fake, 1, None) == nk.NVFP4_ERR_INVALID_ARG    # stride % 8
    assert q(ctypes.c_void_p(0x1008), 4, 96, 96, fake, fake, fake, 1, None) == \
        nk.NVFP4_ERR_INVALID_ARG                                                         # x alignment
    assert q(fake, 0, 96, 96, None, None, None, 1, None) == nk.NVFP4_OK                   # no rows
    assert nk.activation_sf_bytes(200, 96, True) == 256 * 8
    assert nk.activation_sf_bytes(200, 96, False) == 200 * 6
    assert nk.activation_sf_bytes(4, 100, True) == 0
