"""Seeded synthetic inputs for the NVFP4 paged KV cache.

This module only draws random numbers and lays out metadata (sequence
lengths, block tables, slot mappings, global scales from an amax). It holds
none of the method's arithmetic, and both the CUDA path's tests/benchmark and
the CPU oracle take their inputs from here.

Workloads (shapes follow the NVFP4 KV-cache pages: the paged layout of
"FlashInfer backend adds end-to-end NVFP4 KV cache support" and the small
Qwen3-0.6B-class serving runs of "FlashInfer NVFP4 KV serving on pre-SM100
GPUs"):

  tiny_decode     batch 2, ctx 37/100, 4 q / 2 kv heads, head_size 64,
                  block_size 16, 16 blocks in a shuffled table, N(0,1),
                  kv_scale 1.0, o_scale 1.0, one query per sequence.
  qwen3_0p6b_decode
                  16 q / 8 kv heads, head_size 128, block_size 16, batch 32,
                  ctx ~ U[512, 4096], N(0,1) with 2% of (head, channel) pairs
                  scaled x20, random block tables.
  append_sweep    8192 new tokens, 8 kv heads, head_size 128, cache of 65536
                  blocks x 16, random unique slots with 5% set to -1.
  long_decode     32 q / 8 kv heads, head_size 128, block_size 32, batch 64,
                  ctx 32768 each, 2% of channels Student-t(3), split-KV.
  mixed_prefill_decode
                  64 q / 8 kv heads, head_size 256, block_size 16; 8 sequences
                  prefilling 2048 causal queries over 8192 cached tokens and
                  56 decode sequences with ctx ~ U[1024, 16384].

Per-tensor global scales follow amax / (6 * 448) (the largest E2M1 magnitude
times the largest E4M3 magnitude), kv_scale 1.0 for the tiny case; the output
scale is amax(V) / 448, an upper bound on |o| / 448 since each output row is a
convex combination of V rows.

Random numbers: numpy PCG64 for metadata (always on the host), torch
generators for tensor data. Tensor data for a sequence is drawn from its own
generator (seeded from the workload seed and the sequence index), so any one
sequence can be regenerated alone on the same device.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

E2M1_MAX = 6.0
E4M3_MAX = 448.0

WORKLOADS = ("tiny_decode", "qwen3_0p6b_decode", "append_sweep", "long_decode",
             "mixed_prefill_decode")
SEEDS = {name: i + 1 for i, name in enumerate(WORKLOADS)}


@dataclasses.dataclass
class PagedWorkload:
    """Host-side description of a paged attention workload."""

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    seq_lens: np.ndarray          # int32 [B]: keys per sequence (cached + new)
    q_lens: np.ndarray            # int32 [B]: new query tokens per sequence
    num_blocks: int
    block_table: np.ndarray       # int32 [B][max_blocks_per_seq]
    outliers: str = "none"        # "none" | "x20" | "student_t3"
    unit_scales: bool = False     # kv_scale = o_scale = 1.0
    outlier_frac: float = 0.02

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def qo_indptr(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)

    @property
    def num_q_tokens(self) -> int:
        return int(self.q_lens.sum())

    @property
    def max_q_len(self) -> int:
        return int(self.q_lens.max()) if self.num_seqs else 0

    @property
    def is_decode(self) -> bool:
        return bool(np.all(self.q_lens == 1))

    @property
    def full_dim(self) -> int:
        return self.head_size // 2 + self.head_size // 16

    def kv_bytes(self) -> int:
        """NVFP4 K+V row bytes the attention must read (no block padding)."""
        return int(self.seq_lens.astype(np.int64).sum()) * self.num_kv_heads * 2 * self.full_dim

    def prefill_flops(self) -> int:
        """Causal QK^T + PV FLOPs of the multi-token query ranges: 4 * D per
        (query row, visible key, query head)."""
        total = 0
        for b in range(self.num_seqs):
            ql, L = int(self.q_lens[b]), int(self.seq_lens[b])
            if ql <= 1:
                continue
            p = L - ql + np.arange(ql, dtype=np.int64)   # absolute position of each row
            total += int(np.clip(p + 1, 0, None).sum())
        return total * self.num_q_heads * 4 * self.head_size

    def subset(self, seqs: Sequence[int]):
        """(workload over the listed sequences, int64 indices of their query
        tokens in this workload's q). The subset shares this workload's cache
        (same num_blocks and block ids); its tensor data is not redrawn."""
        seqs = [int(b) for b in seqs]
        ind = self.qo_indptr
        tok = np.concatenate([np.arange(ind[b], ind[b + 1], dtype=np.int64) for b in seqs])
        sub = dataclasses.replace(self, name=f"{self.name}[{len(seqs)} seqs]",
                                  seq_lens=self.seq_lens[seqs].copy(),
                                  q_lens=self.q_lens[seqs].copy(),
                                  block_table=np.ascontiguousarray(self.block_table[seqs]))
        return sub, tok

    def slots_for_seq(self, b: int, start: int = 0, stop: Optional[int] = None) -> np.ndarray:
        """Cache slots of tokens start..stop-1 of sequence b (int64)."""
        stop = int(self.seq_lens[b]) if stop is None else stop
        n = np.arange(start, stop, dtype=np.int64)
        blocks = self.block_table[b, n // self.block_size].astype(np.int64)
        return blocks * self.block_size + n % self.block_size

    def outlier_mask(self) -> np.ndarray:
        """bool [num_kv_heads][head_size] of outlier (head, channel) pairs."""
        rng = np.random.default_rng([self.seed, 7])
        n = self.num_kv_heads * self.head_size
        k = int(round(self.outlier_frac * n)) if self.outliers != "none" else 0
        mask = np.zeros(n, bool)
        mask[rng.choice(n, size=k, replace=False)] = True
        return mask.reshape(self.num_kv_heads, self.head_size)


def _block_tables(rng, seq_lens, block_size, num_blocks=None):
    need = [math.ceil(int(L) / block_size) for L in seq_lens]
    total = sum(need)
    nb = total if num_blocks is None else num_blocks
    assert nb >= total
    perm = rng.permutation(nb).astype(np.int32)
    width = max(need) if need else 1
    table = np.zeros((len(seq_lens), width), np.int32)
    pos = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    return table, nb


def make_workload(name: str) -> PagedWorkload:
    """Host metadata for one of the named paged-attention workloads."""
    seed = SEEDS[name]
    rng = np.random.default_rng(seed)
    if name == "tiny_decode":
        seq_lens = np.array([37, 100], np.int32)
        table, nb = _block_tables(rng, seq_lens, 16, num_blocks=16)
        return PagedWorkload(name, seed, 4, 2, 64, 16, seq_lens,
                             np.ones(2, np.int32), nb, table, "none", True)
    if name == "qwen3_0p6b_decode":
        seq_lens = rng.integers(512, 4096, size=32, endpoint=True).astype(np.int32)
        table, nb = _block_tables(rng, seq_lens, 16)
        return PagedWorkload(name, seed, 16, 8, 128, 16, seq_lens,
                             np.ones(32, np.int32), nb, table, "x20")
    if name == "long_decode":
        seq_lens = np.full(64, 32768, np.int32)
        table, nb = _block_tables(rng, seq_lens, 32, num_blocks=65536)
        return PagedWorkload(name, seed, 32, 8, 128, 32, seq_lens,
                             np.ones(64, np.int32), nb, table, "student_t3")
    if name == "mixed_prefill_decode":
        dec = rng.integers(1024, 16384, size=56, endpoint=True).astype(np.int32)
        seq_lens = np.concatenate([np.full(8, 8192 + 2048, np.int32), dec])
        q_lens = np.concatenate([np.full(8, 2048, np.int32), np.ones(56, np.int32)])
        table, nb = _block_tables(rng, seq_lens, 16)
        return PagedWorkload(name, seed, 64, 8, 256, 16, seq_lens, q_lens, nb,
                             table, "none")
    raise KeyError(name)


def custom_workload(name, seed, num_q_heads, num_kv_heads, head_size, block_size,
                    seq_lens: Sequence[int], q_lens: Optional[Sequence[int]] = None,
                    outliers="none", unit_scales=False, spare_blocks=0) -> PagedWorkload:
    """A workload with explicit shapes (for parity sweeps and edge cases)."""
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, np.int32)
    q_lens = np.ones_like(seq_lens) if q_lens is None else np.asarray(q_lens, np.int32)
    need = sum(math.ceil(int(L) / block_size) for L in seq_lens)
    table, nb = _block_tables(rng, seq_lens, block_size, num_blocks=max(need, 1) + spare_blocks)
    return PagedWorkload(name, seed, num_q_heads, num_kv_heads, head_size, block_size,
                         seq_lens, q_lens, nb, table, outliers, unit_scales)


# --------------------------------------------------------------- tensor data
def _gen(device, *key) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence(list(key)).generate_state(1, np.uint64)[0] >> 1))
    return g


def _draw(shape, gen, device, outliers, mask_t):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if outliers == "x20":
        x = torch.where(mask_t, x * 20.0, x)
    elif outliers == "student_t3":
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        c = torch.randn((3,) + tuple(shape), generator=gen, device=device,
                        dtype=torch.float32).square().sum(0)
        t = z / torch.sqrt(c / 3.0)
        x = torch.where(mask_t, t, x)
    return x.to(torch.bfloat16)


def seq_kv(w: PagedWorkload, b: int, device="cpu", start: int = 0,
           stop: Optional[int] = None):
    """bf16 K, V [stop-start][Hkv][D] for tokens start..stop-1 of sequence b."""
    L = int(w.seq_lens[b])
    stop = L if stop is None else stop
    shape = (L, w.num_kv_heads, w.head_size)
    mask_t = torch.from_numpy(w.outlier_mask()).to(device)
    k = _draw(shape, _gen(device, w.seed, 1, b), device, w.outliers, mask_t)
    v = _draw(shape, _gen(device, w.seed, 2, b), device, w.outliers, mask_t)
    return k[start:stop].contiguous(), v[start:stop].contiguous()


def queries(w: PagedWorkload, device="cpu") -> torch.Tensor:
    """bf16 Q [num_q_tokens][Hq][D], N(0,1)."""
    g = _gen(device, w.seed, 3)
    return torch.randn((w.num_q_tokens, w.num_q_heads, w.head_size), generator=g,
                       device=device, dtype=torch.float32).to(torch.bfloat16)


def global_scales(w: PagedWorkload, device="cpu"):
    """(k_scale, v_scale, o_scale) as Python floats (fp32 values).

    amax over every sequence's K (resp. V) / (6 * 448); 1.0 for unit-scale
    workloads. o_scale = amax(V) / 448.
    """
    if w.unit_scales:
        return 1.0, 1.0, 1.0
    ak = torch.zeros((), device=device)
    av = torch.zeros((), device=device)
    for b in range(w.num_seqs):
        k, v = seq_kv(w, b, device)
        ak = torch.maximum(ak, k.float().abs().amax())
        av = torch.maximum(av, v.float().abs().amax())
    ak, av = float(ak), float(av)
    f32 = np.float32
    return (float(f32(ak) / f32(E2M1_MAX * E4M3_MAX)),
            float(f32(av) / f32(E2M1_MAX * E4M3_MAX)),
            float(f32(av) / f32(E4M3_MAX)))


# ------------------------------------------------------------- append sweep
@dataclasses.dataclass
class AppendWorkload:
    name: str
    seed: int
    num_tokens: int
    num_kv_heads: int
    head_size: int
    num_blocks: int
    block_size: int
    skip_frac: float

    @property
    def full_dim(self) -> int:
        return self.head_size // 2 + self.head_size // 16

    def slot_mapping(self) -> np.ndarray:
        """int64 [T]: unique random slots, skip_frac of them set to -1."""
        rng = np.random.default_rng(self.seed)
        slots = rng.choice(self.num_blocks * self.block_size, size=self.num_tokens,
                           replace=False).astype(np.int64)
        n_skip = int(round(self.skip_frac * self.num_tokens))
        slots[rng.choice(self.num_tokens, size=n_skip, replace=False)] = -1
        return slots

    def kv(self, device="cpu"):
        shape = (self.num_tokens, self.num_kv_heads, self.head_size)
        k = torch.randn(shape, generator=_gen(device, self.seed, 1), device=device,
                        dtype=torch.float32).to(torch.bfloat16)
        v = torch.randn(shape, generator=_gen(device, self.seed, 2), device=device,
                        dtype=torch.float32).to(torch.bfloat16)
        return k, v

    def scales(self, k, v):
        f32 = np.float32
        return (float(f32(float(k.float().abs().amax())) / f32(E2M1_MAX * E4M3_MAX)),
                float(f32(float(v.float().abs().amax())) / f32(E2M1_MAX * E4M3_MAX)))

    def live_tokens(self) -> int:
        return int((self.slot_mapping() >= 0).sum())

    def algorithmic_bytes(self) -> int:
        """bf16 K+V read + NVFP4 rows written + 8 B of slot, live tokens only."""
        n = self.live_tokens()
        return n * self.num_kv_heads * (2 * self.head_size * 2 + 2 * self.full_dim) + 8 * n


def make_append(name: str = "append_sweep", num_tokens=8192, num_kv_heads=8,
                head_size=128, num_blocks=65536, block_size=16, skip_frac=0.05,
                seed=None) -> AppendWorkload:
    return AppendWorkload(name, SEEDS.get(name, 3) if seed is None else seed, num_tokens,
                          num_kv_heads, head_size, num_blocks, block_size, skip_frac)
