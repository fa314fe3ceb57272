"""NVFP4 paged KV cache for B200 (sm_100a).

Thin Python binding over the C ABI in ``include/nvfp4kv.h`` (``libnvfp4kv.so``,
built in-tree by ``python -m nvfp4_quantized_paged_append_b200.build``).
Every function below only marshals torch tensors into pointers, sizes and the
current CUDA stream; all work runs in the library's kernels. There is no CPU
fallback: if the library is missing, the first call into it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4kv.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = -1
NVFP4_ERR_UNSUPPORTED = -2
NVFP4_ERR_CUDA = -3
NVFP4_ERR_WORKSPACE = -4
NVFP4_ERR_DEVICE_BOUNDS = -5
NVFP4_ERR_DEVICE_TIMEOUT = -6

DEV_BAD_SLOT = 0x1
DEV_BAD_BLOCK = 0x2
DEV_TIMEOUT = 0x4
DEV_BAD_QLEN = 0x8
NVFP4_ATTN_METADATA_READY = 0x1
NVFP4_ATTN_HISTORY_READY = 0x2
NVFP4_ATTN_QFP4 = 0x4


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what}: {status_string(status)} ({status})"
        if status == NVFP4_ERR_CUDA:
            msg += f": {lib().nvfp4_last_cuda_error().decode()}"
        super().__init__(msg)
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnvfp4kv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m nvfp4_quantized_paged_append_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, f32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                            ctypes.c_size_t)
    L.nvfp4_kv_full_dim.argtypes = [i64]
    L.nvfp4_kv_full_dim.restype = i64
    L.nvfp4_status_string.argtypes = [ctypes.c_int]
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_last_cuda_error.argtypes = []
    L.nvfp4_last_cuda_error.restype = ctypes.c_char_p
    L.nvfp4_quantize_append_paged.argtypes = [P, P, i64, i64, i64, i32, i32, P, i64, i32, P, P, P,
                                              P, P]
    L.nvfp4_quantize_append_paged.restype = ctypes.c_int
    L.nvfp4_paged_attention_workspace_size.argtypes = [i32, i32, i32, i32]
    L.nvfp4_paged_attention_workspace_size.restype = sz
    L.nvfp4_paged_attention.argtypes = [P, i64, i64, i32, P, i64, i32, i32, i32, P, i32, P, P,
                                        i32, i32, P, f32, P, P, P, P, P, sz, P]
    L.nvfp4_paged_attention.restype = ctypes.c_int
    L.nvfp4_paged_attention_ex.argtypes = [P, i64, i64, i32, P, i64, i32, i32, i32, P, i32, P,
                                           P, i32, i32, P, f32, P, P, P, P, P, sz,
                                           ctypes.c_uint32, P]
    L.nvfp4_paged_attention_ex.restype = ctypes.c_int
    L.nvfp4_paged_attention_noalloc.argtypes = [P, i64, i64, i32, P, i64, i32, i32, i32, P,
                                                i32, P, P, i32, i32, P, f32, P, P, P, P, P]
    L.nvfp4_paged_attention_noalloc.restype = ctypes.c_int
    L.nvfp4_fp8kv_quantize_append_paged.argtypes = L.nvfp4_quantize_append_paged.argtypes
    L.nvfp4_fp8kv_quantize_append_paged.restype = ctypes.c_int
    L.nvfp4_fp8kv_paged_attention.argtypes = L.nvfp4_paged_attention_ex.argtypes
    L.nvfp4_fp8kv_paged_attention.restype = ctypes.c_int
    L.nvfp4_paged_decode_append.argtypes = [P, i64, i32, P, P, i64, i64, P, i64, i32, i32, i32,
                                            P, i32, P, i32, P, f32, P, P, P, P, P, sz,
                                            ctypes.c_uint32, P]
    L.nvfp4_paged_decode_append.restype = ctypes.c_int
    L.nvfp4_activation_sf_bytes.argtypes = [i64, i64, ctypes.c_int]
    L.nvfp4_activation_sf_bytes.restype = sz
    L.nvfp4_quantize_activation.argtypes = [P, i64, i64, i64, P, P, P, ctypes.c_int, P]
    L.nvfp4_quantize_activation.restype = ctypes.c_int
    L.nvfp4_dequantize_paged.argtypes = [P, i64, i32, i32, i32, P, i64, P, P, P]
    L.nvfp4_dequantize_paged.restype = ctypes.c_int
    L.nvfp4_read_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, P]
    L.nvfp4_read_device_status.restype = ctypes.c_int
    L.nvfp4_status_from_bits.argtypes = [ctypes.c_uint32]
    L.nvfp4_status_from_bits.restype = ctypes.c_int
    L.nvfp4_paged_attention_noalloc_status.argtypes = [ctypes.POINTER(ctypes.c_uint32),
                                                       ctypes.c_int, P]
    L.nvfp4_paged_attention_noalloc_status.restype = ctypes.c_int
    L.nvfp4_wait_timeout_probe.argtypes = [P, i32, P]
    L.nvfp4_wait_timeout_probe.restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != NVFP4_OK:
        raise Nvfp4Error(status, what)


def full_dim(head_size: int) -> int:
    """head_size/2 + head_size/16 bytes per cache row (-1 if invalid)."""
    return int(lib().nvfp4_kv_full_dim(head_size))


def kv_cache_shape(num_blocks: int, block_size: int, num_kv_heads: int, head_size: int):
    """Logical (NHD) shape of the cache: (num_blocks, 2, block_size, num_kv_heads, full_dim)."""
    return (num_blocks, 2, block_size, num_kv_heads, full_dim(head_size))


def alloc_kv_cache(num_blocks: int, block_size: int, num_kv_heads: int, head_size: int,
                   device="cuda") -> torch.Tensor:
    """uint8 cache in HND storage order: (num_blocks, 2, num_kv_heads, block_size, full_dim)."""
    return torch.zeros((num_blocks, 2, num_kv_heads, block_size, full_dim(head_size)),
                       dtype=torch.uint8, device=device)


def _cache_dims(cache: torch.Tensor, fp8: bool = False):
    if cache.dtype != torch.uint8 or cache.dim() != 5 or cache.shape[1] != 2 or not cache.is_contiguous():
        raise ValueError("cache must be a contiguous uint8 HND tensor (NB, 2, Hkv, bs, row bytes)")
    nb, _, hkv, bs, f = cache.shape
    if fp8:
        return nb, hkv, bs, f
    d = f * 16 // 9
    if full_dim(d) != f:
        raise ValueError(f"cache last dim {f} is not a valid full_dim")
    return nb, hkv, bs, d


def alloc_fp8_kv_cache(num_blocks: int, block_size: int, num_kv_heads: int, head_size: int,
                       device="cuda") -> torch.Tensor:
    """uint8 FP8-E4M3 cache in HND order: (num_blocks, 2, num_kv_heads, block_size, head_size)."""
    return torch.zeros((num_blocks, 2, num_kv_heads, block_size, head_size), dtype=torch.uint8,
                       device=device)


def quantize_append_paged(k: torch.Tensor, v: torch.Tensor, cache: torch.Tensor,
                          slot_mapping: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                          device_status: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None, fp8: bool = False) -> None:
    """Quantize bf16 k/v [T, Hkv, D] into the NVFP4 HND cache at slot_mapping
    (fp8=True: into an FP8-E4M3 cache of head_size-byte rows)."""
    nb, hkv, bs, d = _cache_dims(cache, fp8)
    T = slot_mapping.shape[0]
    for name, x in (("k", k), ("v", v)):
        if x.dtype != torch.bfloat16 or x.shape != (T, hkv, d) or x.stride(2) != 1 or x.stride(1) != d:
            raise ValueError(f"{name} must be bf16 [T, {hkv}, {d}] with contiguous heads")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    fn = lib().nvfp4_fp8kv_quantize_append_paged if fp8 else lib().nvfp4_quantize_append_paged
    st = fn(_ptr(k), _ptr(v), k.stride(0), v.stride(0), T, hkv, d, _ptr(cache), nb, bs,
            _ptr(slot_mapping), _ptr(k_scale), _ptr(v_scale), _ptr(device_status), _stream(stream))
    _check(st, "nvfp4_quantize_append_paged")


def workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_size: int) -> int:
    return int(lib().nvfp4_paged_attention_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                          head_size))


def alloc_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_size: int,
                    device="cuda") -> torch.Tensor:
    """Zero-filled workspace (uint8). Its first 4 bytes are the device status word."""
    n = workspace_size(num_seqs, num_q_heads, num_kv_heads, head_size)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def read_device_status(status_word: torch.Tensor, clear: bool = False,
                       stream: Optional[torch.cuda.Stream] = None):
    """(status code, DEV_* bits) of a device status word -- a workspace (its
    first 4 bytes) or a writer's device_status -- through
    nvfp4_read_device_status (synchronizes the stream; clear resets it)."""
    bits = ctypes.c_uint32(0)
    st = lib().nvfp4_read_device_status(_ptr(status_word), ctypes.byref(bits), int(clear),
                                        _stream(stream))
    if st not in (NVFP4_OK, NVFP4_ERR_DEVICE_BOUNDS, NVFP4_ERR_DEVICE_TIMEOUT):
        _check(st, "nvfp4_read_device_status")
    return st, int(bits.value)


def workspace_status(workspace: torch.Tensor) -> int:
    """Device status bits (DEV_*) recorded in a workspace (synchronizes)."""
    return read_device_status(workspace)[1]


def noalloc_status(clear: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """(status code, DEV_* bits) of the allocation-free entry point's scratch
    status word on the current device (synchronizes; clear resets it)."""
    bits = ctypes.c_uint32(0)
    st = lib().nvfp4_paged_attention_noalloc_status(ctypes.byref(bits), int(clear),
                                                    _stream(stream))
    if st not in (NVFP4_OK, NVFP4_ERR_DEVICE_BOUNDS, NVFP4_ERR_DEVICE_TIMEOUT):
        _check(st, "nvfp4_paged_attention_noalloc_status")
    return st, int(bits.value)


def wait_timeout_probe(status_word: torch.Tensor, polls: int = 1000,
                       stream: Optional[torch.cuda.Stream] = None) -> None:
    """Launch the bounded-wait self-test: a wait that nothing completes gives up
    after `polls` polls and ORs DEV_TIMEOUT into status_word (int32 device)."""
    _check(lib().nvfp4_wait_timeout_probe(_ptr(status_word), polls, _stream(stream)),
           "nvfp4_wait_timeout_probe")


def _attention_dims(q, cache, block_table, seq_lens, qo_indptr, o_fp8, o_bf16, o_f32, fp8=False):
    """Shape and dtype checks shared by the attention calls; returns
    (num_blocks, Hkv, block_size, D, Tq, Hq, num_seqs, max_blocks_per_seq)."""
    nb, hkv, bs, d = _cache_dims(cache, fp8)
    tq, hq, dq = q.shape
    if q.dtype != torch.bfloat16 or dq != d or q.stride(2) != 1 or q.stride(1) != d:
        raise ValueError("q must be bf16 [Tq, Hq, D] with contiguous heads")
    B, mb = block_table.shape
    if block_table.dtype != torch.int32 or not block_table.is_contiguous():
        raise ValueError("block_table must be contiguous int32 [B, max_blocks]")
    if seq_lens.dtype != torch.int32 or qo_indptr is not None and qo_indptr.dtype != torch.int32:
        raise ValueError("seq_lens / qo_indptr must be int32")
    for name, o, dt in (("o_fp8", o_fp8, torch.uint8), ("o_bf16", o_bf16, torch.bfloat16),
                        ("o_f32", o_f32, torch.float32)):
        if o is not None and (o.dtype != dt or o.shape != (tq, hq, d) or not o.is_contiguous()):
            raise ValueError(f"{name} must be contiguous {dt} [Tq, Hq, D]")
    return nb, hkv, bs, d, tq, hq, B, mb


def paged_attention(q: torch.Tensor, cache: torch.Tensor, block_table: torch.Tensor,
                    seq_lens: torch.Tensor, kv_scales: torch.Tensor, o_fp8: torch.Tensor,
                    o_scale: torch.Tensor, workspace: torch.Tensor,
                    qo_indptr: Optional[torch.Tensor] = None, max_q_len: int = 1,
                    sm_scale: float = 0.0, o_bf16: Optional[torch.Tensor] = None,
                    o_f32: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None,
                    metadata_ready: bool = False, fp8: bool = False,
                    history_ready: bool = False, q_fp4: bool = False) -> None:
    """Paged decode / chunked-prefill attention; writes o_fp8 (and o_bf16/o_f32).
    metadata_ready: the kernel launched just before on the stream writes none of
    block_table, seq_lens, qo_indptr, kv_scales, o_scale and workspace, so the
    attention kernel may read them while that kernel finishes
    (NVFP4_ATTN_METADATA_READY; q and the cache are read only after it).
    history_ready: that kernel writes no cache page either, so the first page
    copies start early too (NVFP4_ATTN_HISTORY_READY; implies metadata_ready).
    fp8: the cache holds FP8-E4M3 rows (nvfp4_fp8kv_paged_attention).
    q_fp4: prefill rows compute q K^T on the block-scaled tensor-core path with
    each query row quantized to NVFP4 (NVFP4_ATTN_QFP4; head size 256)."""
    nb, hkv, bs, d, tq, hq, B, mb = _attention_dims(q, cache, block_table, seq_lens, qo_indptr,
                                                    o_fp8, o_bf16, o_f32, fp8)
    fn = lib().nvfp4_fp8kv_paged_attention if fp8 else lib().nvfp4_paged_attention_ex
    st = fn(
        _ptr(q), q.stride(0), tq, hq, _ptr(cache), nb, bs, hkv, d, _ptr(block_table), mb,
        _ptr(seq_lens), _ptr(qo_indptr), B, max_q_len, _ptr(kv_scales), float(sm_scale),
        _ptr(o_fp8), _ptr(o_scale), _ptr(o_bf16), _ptr(o_f32), _ptr(workspace),
        workspace.numel() * workspace.element_size(),
        _attn_flags(metadata_ready, history_ready) | (NVFP4_ATTN_QFP4 if q_fp4 else 0),
        _stream(stream))
    _check(st, "nvfp4_paged_attention")


def _attn_flags(metadata_ready: bool, history_ready: bool) -> int:
    return (NVFP4_ATTN_METADATA_READY if metadata_ready else 0) | \
        (NVFP4_ATTN_HISTORY_READY if history_ready else 0)


def paged_decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                        cache: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
                        kv_scales: torch.Tensor, o_fp8: torch.Tensor, o_scale: torch.Tensor,
                        workspace: torch.Tensor, sm_scale: float = 0.0,
                        o_bf16: Optional[torch.Tensor] = None,
                        o_f32: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None,
                        metadata_ready: bool = False, history_ready: bool = False) -> None:
    """One decode step in one launch: write every sequence's newest k/v row
    (position seq_lens[b] - 1) into the NVFP4 cache and run decode attention
    over all keys. q [B, Hq, D], k_new / v_new [B, Hkv, D] bf16. metadata_ready
    and history_ready as for paged_attention (history: the keys before
    position seq_lens[b] - 1)."""
    nb, hkv, bs, d, tq, hq, B, mb = _attention_dims(q, cache, block_table, seq_lens, None,
                                                    o_fp8, o_bf16, o_f32)
    for name, x in (("k_new", k_new), ("v_new", v_new)):
        if x.dtype != torch.bfloat16 or x.shape != (B, hkv, d) or x.stride(2) != 1 or \
                x.stride(1) != d:
            raise ValueError(f"{name} must be bf16 [{B}, {hkv}, {d}] with contiguous heads")
    if tq != B:
        raise ValueError("q must hold one token per sequence")
    st = lib().nvfp4_paged_decode_append(
        _ptr(q), q.stride(0), hq, _ptr(k_new), _ptr(v_new), k_new.stride(0), v_new.stride(0),
        _ptr(cache), nb, bs, hkv, d, _ptr(block_table), mb, _ptr(seq_lens), B, _ptr(kv_scales),
        float(sm_scale), _ptr(o_fp8), _ptr(o_scale), _ptr(o_bf16), _ptr(o_f32), _ptr(workspace),
        workspace.numel() * workspace.element_size(),
        _attn_flags(metadata_ready, history_ready), _stream(stream))
    _check(st, "nvfp4_paged_decode_append")


def paged_attention_noalloc(q: torch.Tensor, cache: torch.Tensor, block_table: torch.Tensor,
                            seq_lens: torch.Tensor, kv_scales: torch.Tensor, o_fp8: torch.Tensor,
                            o_scale: torch.Tensor, qo_indptr: Optional[torch.Tensor] = None,
                            max_q_len: int = 1, sm_scale: float = 0.0,
                            o_bf16: Optional[torch.Tensor] = None,
                            o_f32: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> None:
    """paged_attention for callers that cannot hand over a workspace: the
    library uses its own fixed scratch array (see nvfp4_paged_attention_noalloc
    in include/nvfp4kv.h: one array per GPU, shared by all calls, so calls must
    not overlap on the GPU; sizes beyond it raise)."""
    nb, hkv, bs, d, tq, hq, B, mb = _attention_dims(q, cache, block_table, seq_lens, qo_indptr,
                                                    o_fp8, o_bf16, o_f32)
    st = lib().nvfp4_paged_attention_noalloc(
        _ptr(q), q.stride(0), tq, hq, _ptr(cache), nb, bs, hkv, d, _ptr(block_table), mb,
        _ptr(seq_lens), _ptr(qo_indptr), B, max_q_len, _ptr(kv_scales), float(sm_scale),
        _ptr(o_fp8), _ptr(o_scale), _ptr(o_bf16), _ptr(o_f32), _stream(stream))
    _check(st, "nvfp4_paged_attention_noalloc")


def dequantize_paged(cache: torch.Tensor, block_ids: torch.Tensor, kv_scales: torch.Tensor,
                     out: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """bf16 [len(block_ids), 2, Hkv, bs, D] pages of the listed blocks."""
    nb, hkv, bs, d = _cache_dims(cache)
    n = block_ids.shape[0]
    if out is None:
        out = torch.empty((n, 2, hkv, bs, d), dtype=torch.bfloat16, device=cache.device)
    if block_ids.dtype != torch.int32:
        raise ValueError("block_ids must be int32")
    st = lib().nvfp4_dequantize_paged(_ptr(cache), nb, bs, hkv, d, _ptr(block_ids), n,
                                      _ptr(kv_scales), _ptr(out), _stream(stream))
    _check(st, "nvfp4_dequantize_paged")
    return out


def activation_sf_bytes(rows: int, cols: int, swizzled: bool = True) -> int:
    return int(lib().nvfp4_activation_sf_bytes(rows, cols, int(swizzled)))


def quantize_activation(x: torch.Tensor, global_scale_inv: torch.Tensor, swizzled: bool = True,
                        out_fp4: Optional[torch.Tensor] = None,
                        out_sf: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None):
    """bf16 x [rows, cols] -> (packed E2M1 uint8 [rows, cols/2], E4M3 scales:
    a flat swizzled uint8 array, or [rows, cols/16] when swizzled is False)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be bf16 [rows, cols] with contiguous rows")
    rows, cols = x.shape
    if out_fp4 is None:
        out_fp4 = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    n = activation_sf_bytes(rows, cols, swizzled)
    if out_sf is None:
        out_sf = torch.empty(n, dtype=torch.uint8, device=x.device)
    if out_fp4.dtype != torch.uint8 or out_fp4.shape != (rows, cols // 2) or \
            not out_fp4.is_contiguous():
        raise ValueError("out_fp4 must be contiguous uint8 [rows, cols/2]")
    if out_sf.dtype != torch.uint8 or out_sf.numel() < n or not out_sf.is_contiguous():
        raise ValueError(f"out_sf must be contiguous uint8 with >= {n} bytes")
    st = lib().nvfp4_quantize_activation(_ptr(x), rows, cols, x.stride(0), _ptr(global_scale_inv),
                                         _ptr(out_fp4), _ptr(out_sf), int(swizzled),
                                         _stream(stream))
    _check(st, "nvfp4_quantize_activation")
    return out_fp4, (out_sf if swizzled else out_sf[:n].view(rows, cols // 16))

