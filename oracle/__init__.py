"""CPU oracle for the NVFP4 paged KV cache -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct restatement (C, fp64 attention) of what the GPU
path computes; see ``nvfp4_oracle.c`` for the definitions and the page
sections they follow. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. It shares no code with
the CUDA path and never imports it.

Arrays are numpy: bf16 data travels as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import numpy as np

from .build import build  # noqa: E402  (gcc build of the C oracle)


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32, f32, f64, u8 = (ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                  ctypes.c_double, ctypes.c_uint8)
        _lib.nvo_e2m1_decode.argtypes = [u8]
        _lib.nvo_e2m1_decode.restype = f64
        _lib.nvo_e4m3_decode.argtypes = [u8]
        _lib.nvo_e4m3_decode.restype = f64
        _lib.nvo_e4m3_encode.argtypes = [f64]
        _lib.nvo_e4m3_encode.restype = u8
        _lib.nvo_e2m1_encode.argtypes = [f64]
        _lib.nvo_e2m1_encode.restype = u8
        _lib.nvo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.nvo_bf16_to_f32.restype = f32
        _lib.nvo_f32_to_bf16.argtypes = [f32]
        _lib.nvo_f32_to_bf16.restype = ctypes.c_uint16
        _lib.nvo_full_dim.argtypes = [i64]
        _lib.nvo_full_dim.restype = i64
        _lib.nvo_quantize_row.argtypes = [P, ctypes.c_int, f32, P]
        _lib.nvo_quantize_row.restype = None
        _lib.nvo_quantize_append_paged.argtypes = [
            P, P, i64, i64, i64, ctypes.c_int, ctypes.c_int, P, i64, ctypes.c_int,
            P, f32, f32]
        _lib.nvo_quantize_append_paged.restype = i64
        _lib.nvo_dequantize_paged.argtypes = [
            P, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, i64, f32, f32, P]
        _lib.nvo_dequantize_paged.restype = None
        _lib.nvo_paged_attention.argtypes = [
            P, i64, ctypes.c_int, P, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            P, ctypes.c_int, P, P, ctypes.c_int, f32, f32, f64, f32, P, P, P]
        _lib.nvo_paged_attention.restype = None
        _lib.nvo_paged_attention_fmt.argtypes = _lib.nvo_paged_attention.argtypes + [ctypes.c_int]
        _lib.nvo_paged_attention_fmt.restype = None
        _lib.nvo_paged_attention_qfp4.argtypes = _lib.nvo_paged_attention.argtypes
        _lib.nvo_paged_attention_qfp4.restype = None
        _lib.nvo_q_row_global.argtypes = [P, ctypes.c_int]
        _lib.nvo_q_row_global.restype = f32
        _lib.nvo_fp8kv_quantize_append_paged.argtypes = _lib.nvo_quantize_append_paged.argtypes
        _lib.nvo_fp8kv_quantize_append_paged.restype = i64
        _lib.nvo_act_sf_bytes.argtypes = [i64, i64, ctypes.c_int]
        _lib.nvo_act_sf_bytes.restype = i64
        _lib.nvo_act_sf_index.argtypes = [i64, i64, i64]
        _lib.nvo_act_sf_index.restype = i64
        _lib.nvo_quantize_activation.argtypes = [P, i64, i64, i64, f32, P, P, ctypes.c_int]
        _lib.nvo_quantize_activation.restype = None
        del i32
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _need(a, dtype, name):
    if a.dtype != dtype or not a.flags["C_CONTIGUOUS"]:
        raise TypeError(f"{name}: need C-contiguous {dtype}, got {a.dtype}")


# ---------------------------------------------------------------- formats
def e2m1_decode(code: int) -> float:
    return lib().nvo_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return lib().nvo_e4m3_decode(code)


def e4m3_encode(x: float) -> int:
    return lib().nvo_e4m3_encode(float(x))


def e2m1_encode(x: float) -> int:
    return lib().nvo_e2m1_encode(float(x))


def bf16_to_f32(bits: int) -> float:
    return lib().nvo_bf16_to_f32(bits)


def f32_to_bf16(x: float) -> int:
    return lib().nvo_f32_to_bf16(x)


def full_dim(head_size: int) -> int:
    return lib().nvo_full_dim(head_size)


# ---------------------------------------------------------------- writer
def quantize_row(x_bf16: np.ndarray, g: float) -> np.ndarray:
    """One row of head_size bf16 values -> full_dim bytes."""
    _need(x_bf16, np.uint16, "x")
    d = x_bf16.shape[-1]
    row = np.zeros(full_dim(d), np.uint8)
    lib().nvo_quantize_row(_ptr(x_bf16), d, g, _ptr(row))
    return row


def quantize_append_paged(k, v, cache, slot_mapping, k_scale, v_scale,
                          block_size, k_token_stride=None, v_token_stride=None):
    """In-place writer on a numpy HND cache uint8[NB][2][Hkv][bs][F].

    k, v: uint16 [T][Hkv][D] (or [T][stride] with the given token strides).
    Returns the number of tokens whose slot lay beyond the cache.
    """
    _need(k, np.uint16, "k")
    _need(v, np.uint16, "v")
    _need(cache, np.uint8, "cache")
    _need(slot_mapping, np.int64, "slot_mapping")
    nb, two, hkv, bs, f = cache.shape
    assert two == 2 and bs == block_size
    d = (f * 16) // 9
    T = slot_mapping.shape[0]
    ks = k_token_stride if k_token_stride is not None else hkv * d
    vs = v_token_stride if v_token_stride is not None else hkv * d
    return lib().nvo_quantize_append_paged(
        _ptr(k), _ptr(v), ks, vs, T, hkv, d, _ptr(cache), nb, bs,
        _ptr(slot_mapping), k_scale, v_scale)


def dequantize_paged(cache, block_ids, k_scale, v_scale):
    """bf16 bits uint16[len(block_ids)][2][Hkv][bs][D] of the listed blocks."""
    _need(cache, np.uint8, "cache")
    _need(block_ids, np.int32, "block_ids")
    nb, _, hkv, bs, f = cache.shape
    d = (f * 16) // 9
    out = np.zeros((block_ids.shape[0], 2, hkv, bs, d), np.uint16)
    lib().nvo_dequantize_paged(_ptr(cache), nb, bs, hkv, d, _ptr(block_ids),
                               block_ids.shape[0], k_scale, v_scale, _ptr(out))
    return out


# ---------------------------------------------------------------- attention
KV_NVFP4, KV_FP8 = 0, 1


def fp8kv_quantize_append_paged(k, v, cache, slot_mapping, k_scale, v_scale, block_size):
    """FP8-E4M3 writer on a numpy HND cache uint8[NB][2][Hkv][bs][D]:
    E4M3_RNE_satfinite(fl32(x / g)) per element."""
    _need(k, np.uint16, "k")
    _need(v, np.uint16, "v")
    _need(cache, np.uint8, "cache")
    _need(slot_mapping, np.int64, "slot_mapping")
    nb, two, hkv, bs, d = cache.shape
    assert two == 2 and bs == block_size
    T = slot_mapping.shape[0]
    return lib().nvo_fp8kv_quantize_append_paged(
        _ptr(k), _ptr(v), hkv * d, hkv * d, T, hkv, d, _ptr(cache), nb, bs,
        _ptr(slot_mapping), k_scale, v_scale)


def paged_attention(q, cache, block_table, seq_lens, qo_indptr, k_scale,
                    v_scale, sm_scale=0.0, o_scale=1.0, kv_format=KV_NVFP4, q_fp4=False):
    """fp64 paged attention. Returns (o_f64, o_fp8, o_bf16_bits).

    q: uint16 [Tq][Hq][D]; cache uint8[NB][2][Hkv][bs][F] (F = D/2 + D/16 for
    NVFP4, D for FP8 rows); block_table int32 [B][max_blocks]; seq_lens int32
    [B]; qo_indptr int32 [B+1] or None. q_fp4 (NVFP4 cache only): the query
    rows of sequences with more than one query are NVFP4-quantized first
    (global scale per row, see q_row_global).
    """
    _need(q, np.uint16, "q")
    _need(cache, np.uint8, "cache")
    _need(block_table, np.int32, "block_table")
    _need(seq_lens, np.int32, "seq_lens")
    if qo_indptr is not None:
        _need(qo_indptr, np.int32, "qo_indptr")
    tq, hq, d = q.shape
    nb, _, hkv, bs, f = cache.shape
    B, mb = block_table.shape
    o64 = np.zeros((tq, hq, d), np.float64)
    o8 = np.zeros((tq, hq, d), np.uint8)
    o16 = np.zeros((tq, hq, d), np.uint16)
    if q_fp4:
        if kv_format != KV_NVFP4:
            raise ValueError("q_fp4 is defined over the NVFP4 cache")
        lib().nvo_paged_attention_qfp4(
            _ptr(q), tq, hq, _ptr(cache), nb, bs, hkv, d, _ptr(block_table), mb,
            _ptr(seq_lens), _ptr(qo_indptr), B, k_scale, v_scale, sm_scale, o_scale,
            _ptr(o64), _ptr(o8), _ptr(o16))
    else:
        lib().nvo_paged_attention_fmt(
            _ptr(q), tq, hq, _ptr(cache), nb, bs, hkv, d, _ptr(block_table), mb,
            _ptr(seq_lens), _ptr(qo_indptr), B, k_scale, v_scale, sm_scale, o_scale,
            _ptr(o64), _ptr(o8), _ptr(o16), int(kv_format))
    return o64, o8, o16


def q_row_global(row) -> float:
    """Global scale of an NVFP4-quantized query row (bf16 bits uint16[D]): the
    smallest power of two g with amax / (6 g) <= 448 (1 for a zero row)."""
    _need(row, np.uint16, "row")
    return float(lib().nvo_q_row_global(_ptr(row), int(row.shape[-1])))


# ---------------------------------------------------------------- activations
def act_sf_bytes(rows: int, cols: int, swizzled: bool) -> int:
    return int(lib().nvo_act_sf_bytes(rows, cols, int(swizzled)))


def act_sf_index(r: int, c: int, cols: int) -> int:
    """Byte position of scale (row r, scale column c) in the swizzled layout."""
    return int(lib().nvo_act_sf_index(r, c, cols))


def quantize_activation(x, global_scale_inv, swizzled=True):
    """bf16 bits uint16[rows][cols] -> (uint8[rows][cols/2] packed E2M1,
    uint8 scales: swizzled flat array, or [rows][cols/16])."""
    _need(x, np.uint16, "x")
    rows, cols = x.shape
    fp4 = np.zeros((rows, cols // 2), np.uint8)
    n = act_sf_bytes(rows, cols, swizzled)
    sf = np.zeros(n, np.uint8)
    lib().nvo_quantize_activation(_ptr(x), rows, cols, cols, global_scale_inv, _ptr(fp4),
                                  _ptr(sf), int(swizzled))
    return fp4, (sf if swizzled else sf.reshape(rows, cols // 16))

