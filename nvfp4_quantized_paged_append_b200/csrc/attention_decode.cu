// Paged decode attention over the NVFP4 cache, split-KV across the whole GPU.
//
// What it computes ("FlashInfer backend adds end-to-end NVFP4 KV cache
// support": the decode kernel reads the packed E2M1 data plus the split-out
// FP8 block scales through a block table and writes FP8 output that is
// dequantized back to the model dtype): for every decode sequence b and query
// head hq, o = softmax(sm_scale * q K^T) V over the sequence's keys, with
// K = E2M1 * E4M3 * k_scale and V likewise with v_scale.
//
// Work decomposition (B200: 148 SMs, one persistent CTA per SM): a sequence's
// keys are cut into units of 64 tokens (32 for head_size 256). The units of
// all (sequence, kv head) segments are laid end to end and the flattened range
// is cut into equal contiguous pieces, one per warp of the whole grid, so
// every warp streams the same number of bytes whatever the length mix. Warps
// never wait for one another: a segment cut across warps leaves (acc, m, l)
// partials in the workspace. When all warps of a block are done, the block
// takes one arrival ticket per cut segment it holds pieces of (atomic, no
// waiting); the block whose ticket completes a segment merges the partials
// with the log-sum-exp rule and writes the output.
//
// Each warp runs its own kStages-deep pipeline: one bulk async copy
// (cp.async.bulk) per K page and per V page of a unit into shared memory,
// completed on the stage's mbarrier. Pages are contiguous
// block_size*full_dim bytes in the HND layout. Block ids are fetched and
// checked 32 units ahead, one unit per lane.
//
// Math per 16-token tile (all G <= 8 query heads of the kv head at once):
//   S^T[tok][n] = Khat[tok][:] . q[n][:]     mma.m16n8k16, A = Khat (f16,
//                                              dequantized in registers:
//                                              cvt e2m1x2->f16x2, times the
//                                              E4M3 scale; exact), B = q (f16,
//                                              scaled by a power of two)
//   online softmax in fp32 (exp2 domain) over the unit's keys; the running
//   max moves only when a logit exceeds it by more than 2^8, which a lane
//   detects on its own values (one vote, no reduction, in the common case)
//   O^T[d][n] += Vhat^T[d][tok] P[tok][n]     mma.m16n8k16, A = Vhat^T built
//                                              from nibble-transposed bytes,
//                                              P = f16 hi + f16 lo moved from
//                                              the S^T accumulator layout with
//                                              movmatrix
// The contraction index of both products is permuted so that each lane's
// fragments come from contiguous bytes of a row (the same permutation is
// applied to q, and the PV output rows map back to d on the way out).
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace nvfp4kv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;  // lazy max: P stays <= 2^8
// dynamic shared memory a decode CTA may use (of the 227 KB an SM offers one
// block, minus the kernel's static shared memory)
constexpr size_t kDecodeSmemBudget = 226 * 1024;

// One persistent CTA per SM: all of an SM's warps belong to the same block, so
// none of them is starved behind an older co-resident block. head_size 256
// needs more registers and larger rows: 32-token units and fewer warps.
// KV row formats: NVFP4 (E2M1 pairs + E4M3 block scales, D/2 + D/16 bytes)
// and FP8 (one E4M3 byte per element, D bytes; per-tensor scale only).
constexpr int kFmtNvfp4 = 0, kFmtFp8 = 1;

template <int D, int FMT = kFmtNvfp4>
struct DecodeCfg {
  // FP8 rows are larger: 32-token units above head_size 64 keep the page rings
  // of all warps within shared memory
  static constexpr int kUnitTok = (D == 256 || (FMT == kFmtFp8 && D == 128)) ? 32 : 64;
  static constexpr int kMaxWarps = (D == 256) ? 8 : 12;
  static constexpr int kStages = (D == 64) ? 3 : 2;  // units in flight per warp
};

template <int D, int BS, int FMT = kFmtNvfp4>
struct DecodeShape {
  static constexpr int kStages = DecodeCfg<D, FMT>::kStages;
  static constexpr int UT = DecodeCfg<D, FMT>::kUnitTok;  // keys per unit
  static constexpr int T = UT / 16;                        // 16-token tiles per unit
  static constexpr int F = FMT == kFmtFp8 ? D : D / 2 + D / 16;
  static constexpr int PAGE = BS * F;                  // bytes of one (block, K|V, head) page
  static constexpr int U = UT >= BS ? UT / BS : 1;     // pages per unit
  static constexpr int STAGE = 2 * UT * F;             // [K0][V0][K1][V1].. bytes
  static constexpr int NCH = D / 16;                   // MMA chunks along d
  static_assert(PAGE % 16 == 0, "pages must be 16-byte multiples");
  static_assert(UT % BS == 0, "a unit holds whole pages");
  static_assert(U <= 4, "at most four pages per unit");
  // K tile t of a stage (V tile t follows its K tile by PAGE bytes)
  // stage layout: the unit's K pages, then its V pages
  static constexpr int ktile(int t) { return (16 * t / BS) * PAGE + ((16 * t) % BS) * F; }
  static constexpr int VOFF = U * PAGE;  // V tile t = K tile t + VOFF
  // a unit's pages in one or two gather4 tensor copies (4 rows of one page
  // each) when a page fits one box row (<= 256 eight-byte elements)
  static constexpr bool kGather = (U == 2 || U == 4) && PAGE / 8 <= 256;
  // per warp: page ring, query rows of one kv head, kStages + 1 mbarriers,
  // per-stage page masks
  static size_t per_warp(int group) {
    return (size_t)kStages * STAGE + (size_t)group * D * 2 + 8 * (kStages + 1) + 4 * kStages;
  }
  // per block: unit prefix, units per kv head, keys and query token per sequence
  static size_t fixed(int num_seqs) { return 16 * (size_t)num_seqs + 8; }
  static int warps_for(int num_seqs, int group) {
    const size_t f = fixed(num_seqs), pw = per_warp(group);
    if (f + pw > kDecodeSmemBudget) return 0;
    return (int)std::min<size_t>(DecodeCfg<D, FMT>::kMaxWarps, (kDecodeSmemBudget - f) / pw);
  }
  static size_t smem_bytes(int num_seqs, int group, int warps) {
    return warps * per_warp(group) + fixed(num_seqs);
  }
};

__device__ __forceinline__ float warp_max_g(float x) {  // over lanes with equal t4
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
  return x;
}

__device__ __forceinline__ float warp_sum_g(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  x += __shfl_xor_sync(0xffffffffu, x, 16);
  return x;
}

// Output pointers and scale of the epilogue.
struct OutPtrs {
  uint8_t* o_fp8;
  __nv_bfloat16* o_bf16;  // may be null
  float* o_f32;           // may be null
  float inv_os, o_scale;
};

// Final epilogue for one output element (o already in output units):
// E4M3(o / o_scale), and optionally fp32 o and bf16(E4M3 * o_scale).
__device__ __forceinline__ void write_output(const OutPtrs& op, int64_t idx, float o) {
  if (op.o_f32) op.o_f32[idx] = o;
  const uint32_t code = f32_to_e4m3(o * op.inv_os);
  op.o_fp8[idx] = (uint8_t)code;
  if (op.o_bf16) op.o_bf16[idx] = __float2bfloat16_rn(__fmul_rn(e4m3_to_f32(code), op.o_scale));
}

// Two adjacent output elements (idx even; the entry point checks that the
// output pointers are aligned for the pair stores).
__device__ __forceinline__ void write_output2(const OutPtrs& op, int64_t idx, float o0,
                                              float o1) {
  if (op.o_f32) *reinterpret_cast<float2*>(op.o_f32 + idx) = make_float2(o0, o1);
  const uint32_t codes = f32x2_to_e4m3x2(o0 * op.inv_os, o1 * op.inv_os);
  *reinterpret_cast<uint16_t*>(op.o_fp8 + idx) = (uint16_t)codes;
  if (op.o_bf16) {
    const uint32_t h2 = e4m3x2_to_f16x2(codes);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    *reinterpret_cast<__nv_bfloat162*>(op.o_bf16 + idx) =
        __floats2bfloat162_rn(__fmul_rn(f.x, op.o_scale), __fmul_rn(f.y, op.o_scale));
  }
}

// floor(num / den) for 0 <= num, 0 < den < 2^31 and a quotient below 2^22:
// a float estimate (approximate reciprocal), corrected by a step or two.
__device__ __forceinline__ int div_floor(long long num, int den) {
  float rc;
  asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(rc) : "f"((float)den));
  int q = (int)((float)num * rc);
  long long r = num - (long long)q * den;
  while (r < 0) {
    --q;
    r += den;
  }
  while (r >= den) {
    ++q;
    r -= den;
  }
  return q;
}

// Read-only global load that stays where it is written (a plain read-only load
// may be moved next to its first use, which would put its latency back on the
// critical path).
__device__ __forceinline__ int ldg_early(const int* p) {
  int v;
  asm volatile("ld.global.nc.b32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}

// The b in [0, n) with cum[b] <= f < cum[b + 1] (cum non-decreasing, cum[0]
// <= f < cum[n]): binary search over the prefix in shared memory.
__device__ __forceinline__ int seek_bs(const int* cum, int n, int f) {
  int lo = 0, hi = n;  // cum[lo] <= f < cum[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cum[mid] <= f) lo = mid; else hi = mid;
  }
  return lo;
}

// Shared-memory loads at a 32-bit shared address.
template <int Bytes>
__device__ __forceinline__ void lds_words(uint32_t a, uint32_t* w) {
  if constexpr (Bytes == 16) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(a));
  } else if constexpr (Bytes == 8) {
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(w[0]), "=r"(w[1]) : "r"(a));
  } else {
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(w[0]) : "r"(a));
  }
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}

// Per-lane byte offsets inside a 16-token tile (constant for the kernel).
struct LaneOffsets {
  uint32_t k0, k1;              // K data segment of rows g8, g8+8
  uint32_t ks0, ks1;            // K scale bytes of rows g8, g8+8
  uint32_t va, vb, vc, vd;      // V data of tokens 2t4, 2t4+1, 2t4+8, 2t4+9
  uint32_t vsa, vsb, vsc, vsd;  // V scale bytes of those tokens
};

template <int D>
__device__ __forceinline__ LaneOffsets lane_offsets(int g8, int t4) {
  constexpr int F = D / 2 + D / 16;
  LaneOffsets o;
  o.k0 = g8 * F + t4 * (D / 8);
  o.k1 = o.k0 + 8 * F;
  o.ks0 = g8 * F + D / 2 + t4 * (D / 64);
  o.ks1 = o.ks0 + 8 * F;
  o.va = (2 * t4) * F + g8 * (D / 16);
  o.vb = o.va + F;
  o.vc = o.va + 8 * F;
  o.vd = o.va + 9 * F;
  const int vg = (D == 64) ? (g8 >> 1) : (D == 128 ? g8 : 2 * g8);
  o.vsa = (2 * t4) * F + D / 2 + vg;
  o.vsb = o.vsa + F;
  o.vsc = o.vsa + 8 * F;
  o.vsd = o.vsa + 9 * F;
  return o;
}

// S^T tile (16 keys x 8 columns) for one 16-token tile at shared address kt.
// Rows >= valid get zero scales and -inf logits (MASK only).
template <int D, bool MASK>
__device__ __forceinline__ void qk_tile(uint32_t kt, const LaneOffsets& lo, int valid, int g8,
                                        const uint32_t (&bq)[D / 16][2], float (&sacc)[4]) {
  constexpr int SEG = D / 8;
  uint32_t kw0[SEG / 4], kw1[SEG / 4];
  if constexpr (SEG == 32) {
    lds_words<16>(kt + lo.k0, kw0);
    lds_words<16>(kt + lo.k0 + 16, kw0 + 4);
    lds_words<16>(kt + lo.k1, kw1);
    lds_words<16>(kt + lo.k1 + 16, kw1 + 4);
  } else if constexpr (SEG == 16) {
    lds_words<8>(kt + lo.k0, kw0);
    lds_words<8>(kt + lo.k0 + 8, kw0 + 2);
    lds_words<8>(kt + lo.k1, kw1);
    lds_words<8>(kt + lo.k1 + 8, kw1 + 2);
  } else {
    lds_words<4>(kt + lo.k0, kw0);
    lds_words<4>(kt + lo.k0 + 4, kw0 + 1);
    lds_words<4>(kt + lo.k1, kw1);
    lds_words<4>(kt + lo.k1 + 4, kw1 + 1);
  }
  constexpr int NG = (D / 64) > 0 ? D / 64 : 1;
  uint32_t sc0[NG], sc1[NG];
  {
    uint32_t x0, x1;
    if constexpr (D == 256) {
      lds_words<4>(kt + lo.ks0, &x0);
      lds_words<4>(kt + lo.ks1, &x1);
    } else if constexpr (D == 128) {
      x0 = lds_u16(kt + lo.ks0);
      x1 = lds_u16(kt + lo.ks1);
    } else {
      x0 = prmt(lds_u8(kt + lo.ks0), 0u, 0x0000);
      x1 = prmt(lds_u8(kt + lo.ks1), 0u, 0x0000);
    }
    if constexpr (MASK) {
      x0 = (g8 < valid) ? x0 : 0u;
      x1 = (g8 + 8 < valid) ? x1 : 0u;
    }
    if constexpr (D == 64) {
      sc0[0] = e4m3x2_to_f16x2(x0);
      sc1[0] = e4m3x2_to_f16x2(x1);
    } else {
#pragma unroll
      for (int h2 = 0; h2 < NG / 2; ++h2) {
        const uint32_t p0 = e4m3x2_to_f16x2(x0 >> (16 * h2));
        const uint32_t p1 = e4m3x2_to_f16x2(x1 >> (16 * h2));
        sc0[2 * h2] = prmt(p0, 0u, 0x1010);
        sc0[2 * h2 + 1] = prmt(p0, 0u, 0x3232);
        sc1[2 * h2] = prmt(p1, 0u, 0x1010);
        sc1[2 * h2 + 1] = prmt(p1, 0u, 0x3232);
      }
    }
  }
  // two accumulators halve the dependent MMA chain; word i feeds chunks 2i
  // (bytes 0, 1) and 2i + 1 (bytes 2, 3)
  float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < SEG / 4; ++i) {
    uint32_t x0[4], x1[4];
    e2m1x8_to_f16x2x4(kw0[i], x0);
    e2m1x8_to_f16x2x4(kw1[i], x1);
    const uint32_t s0 = sc0[i >> 1], s1 = sc1[i >> 1];
    uint32_t af[4];
    af[0] = hmul2_u32(x0[0], s0);
    af[1] = hmul2_u32(x1[0], s1);
    af[2] = hmul2_u32(x0[1], s0);
    af[3] = hmul2_u32(x1[1], s1);
    mma_f16_16816(sacc, af, bq[2 * i]);
    af[0] = hmul2_u32(x0[2], s0);
    af[1] = hmul2_u32(x1[2], s1);
    af[2] = hmul2_u32(x0[3], s0);
    af[3] = hmul2_u32(x1[3], s1);
    mma_f16_16816(s2, af, bq[2 * i + 1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) sacc[i] += s2[i];
  if constexpr (MASK) {
    if (g8 >= valid) sacc[0] = sacc[1] = -INFINITY;
    if (g8 + 8 >= valid) sacc[2] = sacc[3] = -INFINITY;
  }
}

// 8x8 transpose of 16-bit elements across the warp (lane i holds row i/4,
// columns 2(i%4) and 2(i%4)+1 before and after).
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// P^T of one tile (accumulator layout: pr[0..1] = row g8, columns 2t4, 2t4+1;
// pr[2..3] = row g8+8) -> B fragments b0 = P[2t4, 2t4+1][g8],
// b1 = P[2t4+8, 2t4+9][g8]. P = hi + lo (f16 each). DUP (G <= 4): the
// duplicate columns G..2G-1 carry lo in place of hi (lo_sel picks the halves).
// Otherwise a second fragment pair carries lo.
template <bool DUP>
__device__ __forceinline__ void p_fragments(const float (&pr)[4], uint32_t lo_sel,
                                            uint32_t (&bp)[2], uint32_t (&bpl)[2]) {
  const uint32_t h01 = pack_f16x2(pr[0], pr[1]);
  const uint32_t h23 = pack_f16x2(pr[2], pr[3]);
  const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  const uint32_t l01 = pack_f16x2(pr[0] - f01.x, pr[1] - f01.y);
  const uint32_t l23 = pack_f16x2(pr[2] - f23.x, pr[3] - f23.y);
  if constexpr (DUP) {
    bp[0] = movm_trans(prmt(h01, l01, lo_sel));
    bp[1] = movm_trans(prmt(h23, l23, lo_sel));
    bpl[0] = bpl[1] = 0u;
  } else {
    bp[0] = movm_trans(h01);
    bp[1] = movm_trans(h23);
    bpl[0] = movm_trans(l01);
    bpl[1] = movm_trans(l23);
  }
}

// O^T += Vhat^T P for one 16-token tile at shared address vt.
template <int D, bool MASK, bool DUP>
__device__ __forceinline__ void pv_tile(uint32_t vt, const LaneOffsets& lo, int valid, int t4,
                                        const uint32_t (&bp)[2], const uint32_t (&bpl)[2],
                                        float (&acc)[D / 16][4]) {
  constexpr int VB = D / 16;  // lane's data bytes per token
  constexpr int VW = VB / 4;
  uint32_t v0[VW], v1[VW], v2[VW], v3[VW];
  lds_words<VB>(vt + lo.va, v0);
  lds_words<VB>(vt + lo.vb, v1);
  lds_words<VB>(vt + lo.vc, v2);
  lds_words<VB>(vt + lo.vd, v3);
  constexpr int NGV = (D == 256) ? 2 : 1;
  uint32_t scA[NGV], scB[NGV];
  {
    uint32_t xa, xb, xc, xd;
    if constexpr (D == 256) {
      xa = lds_u16(vt + lo.vsa);
      xb = lds_u16(vt + lo.vsb);
      xc = lds_u16(vt + lo.vsc);
      xd = lds_u16(vt + lo.vsd);
    } else {
      xa = lds_u8(vt + lo.vsa);
      xb = lds_u8(vt + lo.vsb);
      xc = lds_u8(vt + lo.vsc);
      xd = lds_u8(vt + lo.vsd);
    }
    if constexpr (MASK) {
      xa = (2 * t4 < valid) ? xa : 0u;
      xb = (2 * t4 + 1 < valid) ? xb : 0u;
      xc = (2 * t4 + 8 < valid) ? xc : 0u;
      xd = (2 * t4 + 9 < valid) ? xd : 0u;
    }
    scA[0] = e4m3x2_to_f16x2(prmt(xa, xb, 0x0040));
    scB[0] = e4m3x2_to_f16x2(prmt(xc, xd, 0x0040));
    if constexpr (NGV == 2) {
      scA[1] = e4m3x2_to_f16x2(prmt(xa, xb, 0x0051));
      scB[1] = e4m3x2_to_f16x2(prmt(xc, xd, 0x0051));
    }
  }
#pragma unroll
  for (int j = 0; j < VW; ++j) {
    const uint32_t a_lo = (v0[j] & 0x0F0F0F0Fu) | ((v1[j] << 4) & 0xF0F0F0F0u);
    const uint32_t a_hi = ((v0[j] >> 4) & 0x0F0F0F0Fu) | (v1[j] & 0xF0F0F0F0u);
    const uint32_t b_lo = (v2[j] & 0x0F0F0F0Fu) | ((v3[j] << 4) & 0xF0F0F0F0u);
    const uint32_t b_hi = ((v2[j] >> 4) & 0x0F0F0F0Fu) | (v3[j] & 0xF0F0F0F0u);
    uint32_t xa_lo[4], xa_hi[4], xb_lo[4], xb_hi[4];
    e2m1x8_to_f16x2x4(a_lo, xa_lo);
    e2m1x8_to_f16x2x4(a_hi, xa_hi);
    e2m1x8_to_f16x2x4(b_lo, xb_lo);
    e2m1x8_to_f16x2x4(b_hi, xb_hi);
    const int gi = (D == 256) ? (j >> 1) : 0;  // chunk m = 4j + by, group m / 8
#pragma unroll
    for (int by = 0; by < 4; ++by) {
      const int m = 4 * j + by;  // rows d0 = g8*D/8 + 2m, d1 = d0 + 1
      uint32_t af[4];
      af[0] = hmul2_u32(xa_lo[by], scA[gi]);
      af[1] = hmul2_u32(xa_hi[by], scA[gi]);
      af[2] = hmul2_u32(xb_lo[by], scB[gi]);
      af[3] = hmul2_u32(xb_hi[by], scB[gi]);
      mma_f16_16816(acc[m], af, bp);
      if constexpr (!DUP) mma_f16_16816(acc[m], af, bpl);
    }
  }
}

// FP8 rows: per-lane byte offsets inside a 16-token tile. K: lane t4 owns
// bytes [t4 D/4, (t4+1) D/4) of rows g8 and g8+8 (MMA chunk c uses its word c);
// V: bytes [g8 D/8, (g8+1) D/8) of tokens 2t4, 2t4+1, 2t4+8, 2t4+9.
template <int D>
__device__ __forceinline__ LaneOffsets lane_offsets_fp8(int g8, int t4) {
  LaneOffsets o;
  o.k0 = g8 * D + t4 * (D / 4);
  o.k1 = o.k0 + 8 * D;
  o.ks0 = o.ks1 = 0;
  o.va = (2 * t4) * D + g8 * (D / 8);
  o.vb = o.va + D;
  o.vc = o.va + 8 * D;
  o.vd = o.va + 9 * D;
  o.vsa = o.vsb = o.vsc = o.vsd = 0;
  return o;
}

// S^T tile from FP8 rows: E4M3 pairs convert exactly to f16 (no block scale:
// the per-tensor scale is folded into the logit scale). Rows >= valid are
// zeroed (stale bytes may hold NaN codes) and get -inf logits (MASK only).
template <int D, bool MASK>
__device__ __forceinline__ void qk_tile_fp8(uint32_t kt, const LaneOffsets& lo, int valid, int g8,
                                            const uint32_t (&bq)[D / 16][2], float (&sacc)[4]) {
  constexpr int NW = D / 16;  // words per lane and row = MMA chunks
  uint32_t kw0[NW], kw1[NW];
#pragma unroll
  for (int i = 0; i < NW; i += 4) {
    if constexpr (NW >= 4) {
      lds_words<16>(kt + lo.k0 + 4 * i, kw0 + i);
      lds_words<16>(kt + lo.k1 + 4 * i, kw1 + i);
    }
  }
  if constexpr (MASK) {
    const bool z0 = g8 >= valid, z1 = g8 + 8 >= valid;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      kw0[i] = z0 ? 0u : kw0[i];
      kw1[i] = z1 ? 0u : kw1[i];
    }
  }
  float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < NW; ++c) {
    uint32_t af[4];
    af[0] = e4m3x2_to_f16x2(kw0[c] & 0xFFFFu);
    af[1] = e4m3x2_to_f16x2(kw1[c] & 0xFFFFu);
    af[2] = e4m3x2_to_f16x2(kw0[c] >> 16);
    af[3] = e4m3x2_to_f16x2(kw1[c] >> 16);
    if (c & 1) mma_f16_16816(s2, af, bq[c]); else mma_f16_16816(sacc, af, bq[c]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) sacc[i] += s2[i];
  if constexpr (MASK) {
    if (g8 >= valid) sacc[0] = sacc[1] = -INFINITY;
    if (g8 + 8 >= valid) sacc[2] = sacc[3] = -INFINITY;
  }
}

// O^T += Vhat^T P for one 16-token tile of FP8 rows: A fragments pair the same
// element of two tokens (byte interleave, then an exact E4M3 -> f16 pair).
template <int D, bool MASK, bool DUP>
__device__ __forceinline__ void pv_tile_fp8(uint32_t vt, const LaneOffsets& lo, int valid, int t4,
                                            const uint32_t (&bp)[2], const uint32_t (&bpl)[2],
                                            float (&acc)[D / 16][4]) {
  constexpr int VB = D / 8;  // lane's bytes per token
  constexpr int VW = VB / 4;
  uint32_t v0[VW], v1[VW], v2[VW], v3[VW];
  if constexpr (VB >= 16) {
#pragma unroll
    for (int i = 0; i < VW; i += 4) {
      lds_words<16>(vt + lo.va + 4 * i, v0 + i);
      lds_words<16>(vt + lo.vb + 4 * i, v1 + i);
      lds_words<16>(vt + lo.vc + 4 * i, v2 + i);
      lds_words<16>(vt + lo.vd + 4 * i, v3 + i);
    }
  } else {
    lds_words<8>(vt + lo.va, v0);
    lds_words<8>(vt + lo.vb, v1);
    lds_words<8>(vt + lo.vc, v2);
    lds_words<8>(vt + lo.vd, v3);
  }
  if constexpr (MASK) {
    const bool za = 2 * t4 >= valid, zb = 2 * t4 + 1 >= valid;
    const bool zc = 2 * t4 + 8 >= valid, zd = 2 * t4 + 9 >= valid;
#pragma unroll
    for (int j = 0; j < VW; ++j) {
      v0[j] = za ? 0u : v0[j];
      v1[j] = zb ? 0u : v1[j];
      v2[j] = zc ? 0u : v2[j];
      v3[j] = zd ? 0u : v3[j];
    }
  }
#pragma unroll
  for (int j = 0; j < VW; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // chunk m = 2j + h: bytes 2m (even d) and 2m + 1 (odd d)
      const int m = 2 * j + h;
      const uint32_t se = h ? 0x0062u : 0x0040u, so = h ? 0x0073u : 0x0051u;
      uint32_t af[4];
      af[0] = e4m3x2_to_f16x2(prmt(v0[j], v1[j], se));
      af[1] = e4m3x2_to_f16x2(prmt(v0[j], v1[j], so));
      af[2] = e4m3x2_to_f16x2(prmt(v2[j], v3[j], se));
      af[3] = e4m3x2_to_f16x2(prmt(v2[j], v3[j], so));
      mma_f16_16816(acc[m], af, bp);
      if constexpr (!DUP) mma_f16_16816(acc[m], af, bpl);
    }
  }
}

// One unit of T 16-token tiles in the stage at shared address sbase. MASK:
// tile t holds valid[t] usable keys (0: skipped).
// 16-token tiles per step of a unit's rolled tile loop: two keep the unit's
// code small enough for the instruction cache and still overlap two tiles'
// shared-memory loads and MMAs (measured against 1 and 4 per step)
constexpr int kDecodeTilesPerStep = 2;

template <int D, int BS, bool MASK, bool DUP, int FMT, int TBM>
__device__ __forceinline__ void decode_unit(uint32_t sbase, int rem, int pmask, const LaneOffsets& lo,
                                            const uint32_t (&bq)[D / 16][2], float qmult,
                                            uint32_t lo_sel, float (&m_run)[2], float (&l_run)[2],
                                            float (&acc)[D / 16][4], int g8, int t4) {
  using S = DecodeShape<D, BS, FMT>;
  constexpr int T = S::T, NCH = S::NCH;
  constexpr int TB = TBM < T ? TBM : T;
  static_assert(T % TB == 0, "tiles per step divide the unit");
  // TB tiles per step of a rolled loop (TB == T: the whole unit at once)
#pragma unroll 1
  for (int t0 = 0; t0 < T; t0 += TB) {
  int valid[TB];
  bool any = !MASK;
#pragma unroll
  for (int tb = 0; tb < TB; ++tb) {
    int v = 16;
    if constexpr (MASK) {
      const int t = t0 + tb;
      v = min(16, rem - 16 * t);
      if (v < 0 || !((pmask >> (16 * t / BS)) & 1)) v = 0;
      any |= v > 0;
    }
    valid[tb] = v;
  }
  if (!any) continue;  // (warp-uniform)
  float s[TB][4];
#pragma unroll
  for (int t = 0; t < TB; ++t) {
    s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.0f;
    if (!MASK || valid[t] > 0) {
      if constexpr (FMT == kFmtFp8)
        qk_tile_fp8<D, MASK>(sbase + S::ktile(t0 + t), lo, MASK ? valid[t] : 16, g8, bq, s[t]);
      else
        qk_tile<D, MASK>(sbase + S::ktile(t0 + t), lo, MASK ? valid[t] : 16, g8, bq, s[t]);
    } else {
      s[t][0] = s[t][1] = s[t][2] = s[t][3] = -INFINITY;
    }
  }
  // ---- online softmax (log2 units). x = s * qmult - m_run; the max moves only
  // when some x exceeds the threshold (or on the first keys of a column).
  float x[TB][4];
  float mx0 = -INFINITY, mx1 = -INFINITY;
  {
    const float mu0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
    const float mu1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      x[t][0] = fmaf(s[t][0], qmult, -mu0);
      x[t][1] = fmaf(s[t][1], qmult, -mu1);
      x[t][2] = fmaf(s[t][2], qmult, -mu0);
      x[t][3] = fmaf(s[t][3], qmult, -mu1);
      mx0 = fmaxf(mx0, fmaxf(x[t][0], x[t][2]));
      mx1 = fmaxf(mx1, fmaxf(x[t][1], x[t][3]));
    }
  }
  const bool up = mx0 > (m_run[0] == -INFINITY ? -INFINITY : kRescaleThresh) ||
                  mx1 > (m_run[1] == -INFINITY ? -INFINITY : kRescaleThresh);
  if (__any_sync(0xffffffffu, up)) {
    float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      c0 = fmaxf(c0, fmaxf(s[t][0], s[t][2]));
      c1 = fmaxf(c1, fmaxf(s[t][1], s[t][3]));
    }
    const float m0 = warp_max_g(c0) * qmult, m1 = warp_max_g(c1) * qmult;
    const float n0 = fmaxf(m_run[0], m0), n1 = fmaxf(m_run[1], m1);
    const float nu0 = (n0 == -INFINITY) ? 0.f : n0;
    const float nu1 = (n1 == -INFINITY) ? 0.f : n1;
    // ex2(-inf) = 0 clears a column seen for the first time (its acc and l are 0)
    const float al0 = ex2(m_run[0] - nu0);
    const float al1 = ex2(m_run[1] - nu1);
    m_run[0] = n0;
    m_run[1] = n1;
    l_run[0] *= al0;
    l_run[1] *= al1;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      acc[c][0] *= al0;
      acc[c][1] *= al1;
      acc[c][2] *= al0;
      acc[c][3] *= al1;
    }
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      x[t][0] = fmaf(s[t][0], qmult, -nu0);
      x[t][1] = fmaf(s[t][1], qmult, -nu1);
      x[t][2] = fmaf(s[t][2], qmult, -nu0);
      x[t][3] = fmaf(s[t][3], qmult, -nu1);
    }
  }
  float p[TB][4];
#pragma unroll
  for (int t = 0; t < TB; ++t) {
#pragma unroll
    for (int i = 0; i < 4; ++i) p[t][i] = ex2(x[t][i]);
    l_run[0] += p[t][0] + p[t][2];
    l_run[1] += p[t][1] + p[t][3];
  }
#pragma unroll
  for (int t = 0; t < TB; ++t) {
    if (!MASK || valid[t] > 0) {
      uint32_t bp[2], bpl[2];
      p_fragments<DUP>(p[t], lo_sel, bp, bpl);
      if constexpr (FMT == kFmtFp8)
        pv_tile_fp8<D, MASK, DUP>(sbase + S::ktile(t0 + t) + S::VOFF, lo, MASK ? valid[t] : 16,
                                  t4, bp, bpl, acc);
      else
        pv_tile<D, MASK, DUP>(sbase + S::ktile(t0 + t) + S::VOFF, lo, MASK ? valid[t] : 16, t4,
                              bp, bpl, acc);
    }
  }
  }
}

// Merge of one head of a cut segment: its contributors' partials combined
// with the log-sum-exp rule, then the output. Contributor i (a warp of the
// decode grid) left (acc, m, l) in slot 0 if the segment is where its piece
// starts, else in slot 1. Loads of a batch of contributors are all issued
// before any is used (one round trip to L2 per batch).
template <int D>
__device__ __forceinline__ void merge_head(const OutPtrs& op, int num_q_heads,
                                           const float* partials, const float* part_ml, int G,
                                           int h, int n, int qt, int i_first, int i_last,
                                           int seg_start, int W, int n_eff, int lane,
                                           float v_scale) {
  constexpr int CH = 8;       // contributors per batch
  constexpr int J = D / 32;   // elements of d per lane
  const int nc = i_last - i_first + 1;
  float M = -INFINITY, lsum = 0.0f;
  float sum[J];
#pragma unroll
  for (int j = 0; j < J; ++j) sum[j] = 0.0f;
  for (int c0 = 0; c0 < nc; c0 += CH) {
    const int cnt = min(CH, nc - c0);
    // lane r < cnt: contributor c0 + r's slot and (m, l)
    unsigned long long ps_mine = 0;
    float mi = -INFINITY, li = 0.0f;
    if (lane < cnt) {
      const int i = i_first + c0 + lane;
      const int si = div_floor((long long)i * W, n_eff);
      ps_mine = (unsigned long long)i * 2 + ((si >= seg_start) ? 0 : 1);
      mi = __ldcg(part_ml + (ps_mine * G + n) * 2);
      li = __ldcg(part_ml + (ps_mine * G + n) * 2 + 1);
    }
    float v[CH][J];
#pragma unroll
    for (int r = 0; r < CH; ++r) {
      const unsigned long long ps = __shfl_sync(0xffffffffu, ps_mine, r);
#pragma unroll
      for (int j = 0; j < J; ++j)
        v[r][j] = (r < cnt) ? __ldcg(partials + (ps * G + n) * D + lane + 32 * j) : 0.0f;
    }
    // rescale what is accumulated so far to the new running max
    float mx = mi;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float Mn = fmaxf(M, mx);
    const float Mu = (Mn == -INFINITY) ? 0.0f : Mn;
    const float al = ex2(M - Mu);
    lsum *= al;
#pragma unroll
    for (int j = 0; j < J; ++j) sum[j] *= al;
    M = Mn;
    const float sc = ex2(mi - Mu);
    float lw = li * sc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
    lsum += lw;
#pragma unroll
    for (int r = 0; r < CH; ++r) {
      const float wr = __shfl_sync(0xffffffffu, sc, r);
#pragma unroll
      for (int j = 0; j < J; ++j) sum[j] += v[r][j] * wr;
    }
  }
  const float scl = (lsum > 0.0f) ? v_scale / lsum : 0.0f;
  const long long obase = ((long long)qt * num_q_heads + h * G + n) * D;
#pragma unroll
  for (int j = 0; j < J; ++j) write_output(op, obase + lane + 32 * j, sum[j] * scl);
}

}  // namespace

template <int D, int BS, bool DUP, int FMT>
__global__ void __launch_bounds__(DecodeCfg<D, FMT>::kMaxWarps * 32, 1)
    decode_attention_kernel(const __grid_constant__ AttentionArgs a) {
  using S = DecodeShape<D, BS, FMT>;
  constexpr int kStages = S::kStages;
  constexpr int PAGE = S::PAGE, NCH = S::NCH, U = S::U, UT = S::UT;
  constexpr int STAGE = S::STAGE;
  extern __shared__ __align__(128) uint8_t smem[];
  const int nw = blockDim.x >> 5;
  const int Hkv = a.num_kv_heads, G = a.num_q_heads / Hkv;
  const int B = a.num_seqs;
  const int QB = G * D * 2;  // bytes of the query rows of one kv head
  uint8_t* ring = smem;
  uint8_t* qbuf = ring + (size_t)nw * kStages * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(qbuf + (size_t)nw * QB);  // [nw][kStages + 1]
  int* stage_ok = reinterpret_cast<int*>(bars + nw * (kStages + 1));
  int* cum = stage_ok + nw * kStages;  // [B + 1] unit prefix
  int* sub = cum + B + 1;              // [B] units per kv head
  int* slen = sub + B;                 // [B] keys
  int* sqt = slen + B;                 // [B] query token
  __shared__ int warp_tot[DecodeCfg<D, FMT>::kMaxWarps];
  __shared__ int cut_sg[2 * DecodeCfg<D, FMT>::kMaxWarps];  // [warp][slot]: cut segment or -1
  __shared__ int won[2 * DecodeCfg<D, FMT>::kMaxWarps];     // segments this block merges
  __shared__ int nwon;

  // Launched as a programmatic dependent of the previous kernel on the stream
  // (when that kernel allows it): the block may be resident early, but reads
  // nothing that kernel may write before it has completed and its writes are
  // visible. With metadata_ready the batch metadata (sequence lengths, query
  // ranges, block table) is known not to be among them and is read first.
  // With history_ready the history pages are not written by it either: the
  // first page copies start before the wait too.
  const bool history_ready = (a.flags & kAttnHistoryReady) != 0;
  const bool metadata_ready = history_ready || (a.flags & kAttnMetadataReady) != 0;
  // The next kernel on the stream, if launched as a programmatic dependent,
  // may start its blocks on SMs this grid frees; like this one, it waits for
  // this grid's completion before reading anything this grid writes.
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  if (!metadata_ready) grid_dependency_wait();
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.workspace);
  const WorkspaceLayout wl = workspace_layout(B, Hkv, D, G);
  int* counters = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.counters_off);
  float* partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.partials_off);
  float* part_ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.ml_off);
  if (tid < 2 * DecodeCfg<D, FMT>::kMaxWarps) cut_sg[tid] = -1;
  if (tid == 0) nwon = 0;

  // ---- 1. unit prefix over decode sequences (q_len == 1): a sequence has
  // ceil(pages / U) units per kv head, with at least one page (an empty
  // sequence still writes its zero row) and at most what its block table row
  // maps.
  int carry = 0;
  for (int base = 0; base < B; base += nw * 32) {
    const int b = base + tid;
    int val = 0;
    if (b < B) {
      const int q0 = a.qo_indptr ? a.qo_indptr[b] : b;
      const int ql = a.qo_indptr ? a.qo_indptr[b + 1] - q0 : 1;
      const int L = a.seq_lens[b];
      // a query range longer than the host's bound is not fully served by the
      // prefill grid (sized from max_q_len): flagged, by block 0 only
      if (ql > max(1, a.max_q_len) && blockIdx.x == 0) atomicOr(status, kDevBadQlen);
      const int pages = min(a.max_blocks_per_seq, max(1, (L + BS - 1) / BS));
      const int ub = (pages + U - 1) / U;
      val = (ql == 1) ? ub * Hkv : 0;
      sub[b] = (ql == 1) ? ub : 0;
      slen[b] = L;
      sqt[b] = q0;
    }
    int x = val;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < nw; ++i) {
      before += (i < w) ? warp_tot[i] : 0;
      total += warp_tot[i];
    }
    if (b < B) cum[b] = carry + before + x - val;
    carry += total;
    __syncthreads();
  }
  if (tid == 0) cum[B] = carry;
  __syncthreads();
  // From here on every warp works alone: no block-wide barrier follows.

  // ---- 2. this warp's contiguous piece [s, e) of the W flattened units
  const int W = cum[B];
  const int n_eff = min((int)gridDim.x * nw, W);
  // the warp whose piece holds unit f
  auto warp_of = [&](int f) { return div_floor((long long)(f + 1) * n_eff - 1, W); };
  const float v_scale = __ldg(a.kv_scales + 1);
  const float o_scale = __ldg(a.o_scale);
  const OutPtrs op{a.o_fp8, reinterpret_cast<__nv_bfloat16*>(a.o_bf16), a.o_f32, 1.0f / o_scale,
                   o_scale};
  const int gw = blockIdx.x * nw + w;
  if (gw < n_eff) {  // (idle warps go straight to the block's merge step)
    const int s = div_floor((long long)gw * W, n_eff);
    const int e = div_floor((long long)(gw + 1) * W, n_eff);
    // (sequence, kv head, first unit of the segment) of flattened unit f
    auto locate = [&](int f, int& b, int& h, int& seg_start) {
      b = seek_bs(cum, B, f);
      const int ub = sub[b];
      h = div_floor(f - cum[b], ub);
      seg_start = cum[b] + h * ub;
    };

    const int nk = e - s;

    uint64_t* my_bars = bars + w * (kStages + 1);  // stage barriers, then the query barrier
    uint64_t* q_bar = my_bars + kStages;
    int* my_ok = stage_ok + w * kStages;
    uint8_t* my_ring_p = ring + (size_t)w * kStages * STAGE;
    uint8_t* my_q = qbuf + (size_t)w * QB;
    const uint32_t my_ring = smem_u32(my_ring_p);
    const uint32_t my_q_s = smem_u32(my_q);
    if (lane == 0) {
      for (int st = 0; st <= kStages; ++st) mbar_init(&my_bars[st], 1);
      fence_mbar_init();
    }
    __syncwarp();
    // query rows of kv head h of sequence b into this warp's query buffer
    auto fetch_q = [&](int b, int h) {
      if (lane == 0) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q) +
                             ((long long)sqt[b] * a.q_token_stride + (long long)h * G * D) * 2;
        mbar_arrive_expect_tx(q_bar, QB);
        bulk_g2s(my_q, src, QB, q_bar);
      }
    };

    bool poisoned = false;
    // Block ids are fetched 32 units at a time, lane j holding unit base + j of
    // this warp (two banks, refilled a whole batch ahead), so no global load
    // latency sits between finishing a unit and issuing the copies of the next.
    // The lane also checks them: a bad id is not copied and its page masked.
    // (Two named banks selected with conditionals: a bank index into an array
    // would put the array in local memory.)
    int bid0[U], bid1[U];
    int bmeta0 = 0, bmeta1 = 0;  // h << 16 | ok mask << 8 | pages to copy
#pragma unroll
    for (int j = 0; j < U; ++j) bid0[j] = bid1[j] = 0;
    auto batch_load = [&](int base) {
      const int bank = (base >> 5) & 1;
      int ids[U];
#pragma unroll
      for (int j = 0; j < U; ++j) ids[j] = 0;
      int meta = 0;
      if (base + lane < nk) {
        int b, hh, ss;
        const int f = s + base + lane;
        locate(f, b, hh, ss);
        const int u = f - ss;
        const int Lb = slen[b];
        const int pages = min(a.max_blocks_per_seq, max(1, (Lb + BS - 1) / BS));
        const int npg = (Lb > 0) ? min(U, pages - u * U) : 0;
        const int* row = a.block_table + (long long)b * a.max_blocks_per_seq + u * U;
        int ok = 0;
#pragma unroll
        for (int j = 0; j < U; ++j) {
          if (j < npg) {
            const int x = ldg_early(row + j);
            if (x >= 0 && x < a.num_blocks) {
              ids[j] = x;
              ok |= 1 << j;
            } else {
              atomicOr(status, kDevBadBlock);  // not copied; its tiles are masked
            }
          }
        }
        meta = (hh << 16) | ok;
      }
      if (bank) {
#pragma unroll
        for (int j = 0; j < U; ++j) bid1[j] = ids[j];
        bmeta1 = meta;
      } else {
#pragma unroll
        for (int j = 0; j < U; ++j) bid0[j] = ids[j];
        bmeta0 = meta;
      }
    };
    auto issue = [&](int k) {  // unit k of this warp into stage k % kStages
      const int st = k % kStages;
      const int bank = (k >> 5) & 1, src = k & 31;
      const int meta = __shfl_sync(0xffffffffu, bank ? bmeta1 : bmeta0, src);
      int blk[U];
#pragma unroll
      for (int j = 0; j < U; ++j) blk[j] = __shfl_sync(0xffffffffu, bank ? bid1[j] : bid0[j], src);
      const int cmask = meta & 0xFF, n_h = meta >> 16;  // pages to copy (bit j: page j)
      // The stage being refilled was last read by this warp's own ld.shared
      // instructions, all complete before the __syncwarp that precedes this
      // call; the copies only write, so no proxy fence is needed here.
      if (lane == 0) {
        my_ok[st] = meta & 0xFF;  // copied pages
        mbar_arrive_expect_tx(&my_bars[st], 2 * PAGE * __popc(cmask));
        uint8_t* dst = my_ring_p + (size_t)st * STAGE;
        // page row r of the cache: (block, K|V, head) = (r / 2Hkv, r / Hkv % 2, r % Hkv)
        if (S::kGather && cmask == (1 << U) - 1) {
          const uint32_t d = smem_u32(dst);
          if constexpr (U == 4) {
            tma_gather4(d, &a.kv_pages, blk[0] * 2 * Hkv + n_h, blk[1] * 2 * Hkv + n_h,
                        blk[2] * 2 * Hkv + n_h, blk[3] * 2 * Hkv + n_h, &my_bars[st]);
            tma_gather4(d + 4 * PAGE, &a.kv_pages, (blk[0] * 2 + 1) * Hkv + n_h,
                        (blk[1] * 2 + 1) * Hkv + n_h, (blk[2] * 2 + 1) * Hkv + n_h,
                        (blk[3] * 2 + 1) * Hkv + n_h, &my_bars[st]);
          } else {
            tma_gather4(d, &a.kv_pages, blk[0] * 2 * Hkv + n_h, blk[U - 1] * 2 * Hkv + n_h,
                        (blk[0] * 2 + 1) * Hkv + n_h, (blk[U - 1] * 2 + 1) * Hkv + n_h,
                        &my_bars[st]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < U; ++j) {
            if ((cmask >> j) & 1) {
              const uint8_t* kp = a.cache + ((long long)blk[j] * 2 * Hkv + n_h) * PAGE;
              bulk_g2s(dst + j * PAGE, kp, PAGE, &my_bars[st]);
              bulk_g2s(dst + (U + j) * PAGE, kp + (long long)Hkv * PAGE, PAGE, &my_bars[st]);
            }
          }
        }
      }
      // entering a new batch of 32: fetch the one after it into the other bank
      if ((k & 31) == 0 && k + 32 < nk) batch_load(k + 32);
    };

    batch_load(0);
    if (history_ready)
      for (int k = 0; k < min(kStages, nk); ++k) issue(k);
    if (metadata_ready) grid_dependency_wait();  // q, cache and workspace from here on
    {
      int b, h, ss;
      locate(s, b, h, ss);
      fetch_q(b, h);
    }
    if (!history_ready)
      for (int k = 0; k < min(kStages, nk); ++k) issue(k);

    const float k_scale = __ldg(a.kv_scales);
    const LaneOffsets lo = FMT == kFmtFp8 ? lane_offsets_fp8<D>(g8, t4) : lane_offsets<D>(g8, t4);
    // DUP: columns G..2G-1 of the lanes' B fragments carry lo parts
    const bool lo0 = DUP && (2 * t4 >= G) && (2 * t4 < 2 * G);
    const bool lo1 = DUP && (2 * t4 + 1 >= G) && (2 * t4 + 1 < 2 * G);
    const uint32_t lo_sel = (lo0 ? 0x0054u : 0x0010u) | (lo1 ? 0x7600u : 0x3200u);

    int k = 0;  // this warp's unit counter, continuous across portions
    int portion = 0;
    {
      const int r_hi = e;
      int seg_f0 = s;
      while (seg_f0 < r_hi) {
        int b, h, seg_start;
        locate(seg_f0, b, h, seg_start);
        const int seg_end = seg_start + sub[b];
        const int pe = min(r_hi, seg_end);
        const int L = slen[b];
        const int qt = sqt[b];

        // ---- fused append: the warp holding the segment's last unit quantizes
        // the sequence's newest K and V rows of head h (position L - 1), writes
        // them to the cache and, once that unit's pages land, over its own
        // shared-memory copy of the row (no other warp reads that page). Lanes
        // [0, D/16) take the K groups of 16 elements, [D/16, D/8) the V groups.
        constexpr int NGR = D / 16;
        const bool app = FMT == kFmtNvfp4 && a.k_new != nullptr && pe == seg_end && L >= 1;
        uint32_t app_c0 = 0u, app_c1 = 0u, app_sb = 0u;
        int app_unit = -1, app_pg = 0, app_off = 0;
        if (app && !poisoned) {
          const int pos = L - 1;
          const int pg = pos / BS;
          app_off = pos % BS;
          app_unit = pg / U;
          app_pg = pg % U;
          long long blk = -1;
          if (pg < a.max_blocks_per_seq) {
            blk = ldg_early(a.block_table + (long long)b * a.max_blocks_per_seq + pg);
            if (blk < 0 || blk >= a.num_blocks) blk = -1;  // (flagged by the block-id fetch)
          }
          if (lane < 2 * NGR) {
            const int kv = lane / NGR, j = lane % NGR;
            const __nv_bfloat16* src =
                reinterpret_cast<const __nv_bfloat16*>(kv ? a.v_new : a.k_new) +
                (long long)b * (kv ? a.v_new_stride : a.k_new_stride) + (long long)h * D + j * 16;
            const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(src));
            const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
            const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            float x[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              x[2 * i] = __uint_as_float(wv[i] << 16);
              x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
            }
            app_sb = quantize_group16(x, __ldg(a.kv_scales + kv), app_c0, app_c1);
            if (blk >= 0) {
              uint8_t* dst = const_cast<uint8_t*>(a.cache) +
                             ((blk * 2 + kv) * Hkv + h) * (long long)PAGE + app_off * S::F;
              if constexpr (S::F % 8 == 0) {
                *reinterpret_cast<uint2*>(dst + 8 * j) = make_uint2(app_c0, app_c1);
              } else {
                reinterpret_cast<uint32_t*>(dst + 8 * j)[0] = app_c0;
                reinterpret_cast<uint32_t*>(dst + 8 * j)[1] = app_c1;
              }
              dst[D / 2 + j] = (uint8_t)app_sb;
            }
          }
        }

        // ---- query fragments from this warp's query buffer: lane (g8, t4)
        // holds q[head of column g8][t4*D/4 + i]. DUP: columns G..2G-1 repeat
        // heads 0..G-1 (their P carries the lo part).
        const int qhead = DUP ? (g8 < 2 * G ? g8 % G : -1) : (g8 < G ? g8 : -1);
        uint32_t bq[NCH][2];
        float qmult;
        {
          if (!poisoned && !mbar_wait_bounded(q_bar, (uint32_t)(portion & 1))) {
            poisoned = true;
            if (lane == 0) atomicOr(status, kDevTimeout);
          }
          float qv[D / 4];
          if (qhead >= 0 && !poisoned) {
            const uint32_t qa = my_q_s + (uint32_t)(qhead * D + t4 * (D / 4)) * 2;
#pragma unroll
            for (int i = 0; i < D / 4; i += 8) {
              uint32_t wv[4];
              lds_words<16>(qa + 2 * i, wv);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                qv[i + 2 * j] = __uint_as_float(wv[j] << 16);
                qv[i + 2 * j + 1] = __uint_as_float(wv[j] & 0xFFFF0000u);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < D / 4; ++i) qv[i] = 0.0f;
          }
          float mx = 0.0f;
#pragma unroll
          for (int i = 0; i < D / 4; ++i) mx = fmaxf(mx, fabsf(qv[i]));
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          // power-of-two scale putting max|q| in [2^14, 2^15): f16 keeps every bf16 bit
          const int ex = (mx > 0.0f) ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126 : 1;
          const int sh = min(126, max(-126, 15 - ex));
          const float qs = __uint_as_float((uint32_t)(sh + 127) << 23);
          const float qds = __uint_as_float((uint32_t)(127 - sh) << 23);
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            bq[c][0] = pack_f16x2(qv[4 * c] * qs, qv[4 * c + 1] * qs);
            bq[c][1] = pack_f16x2(qv[4 * c + 2] * qs, qv[4 * c + 3] * qs);
          }
          qmult = a.sm_scale * k_scale * kLog2e * qds;  // raw MMA units -> log2 units
        }
        __syncwarp();
        {  // the next portion's query rows, while this one runs
          if (pe < r_hi && !poisoned) {
            int nb, nh, nss;
            locate(pe, nb, nh, nss);
            fetch_q(nb, nh);
          }
        }

        // ---- running state: columns n0 = 2*t4, n1 = 2*t4+1 (lazily moved max)
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.0f, 0.0f};
        float acc[NCH][4];
#pragma unroll
        for (int c = 0; c < NCH; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;

        for (int f = seg_f0; f < pe; ++f, ++k) {
          const int u = f - seg_start;
          const int st = k % kStages;
          int okbits = 0;
          if (!poisoned) {
            if (mbar_wait_bounded(&my_bars[st], (uint32_t)((k / kStages) & 1))) {
              okbits = my_ok[st];
            } else {
              poisoned = true;
              if (lane == 0) atomicOr(status, kDevTimeout);
            }
          }
          const uint32_t sbase = my_ring + st * STAGE;
          if (u == app_unit && ((okbits >> app_pg) & 1)) {
            // the newest row over this warp's copy of its page (K, then V)
            if (lane < 2 * NGR) {
              const int kv = lane / NGR, j = lane % NGR;
              uint8_t* row = my_ring_p + (size_t)st * STAGE + (kv * U + app_pg) * PAGE +
                             app_off * S::F;
              if constexpr (S::F % 8 == 0) {
                *reinterpret_cast<uint2*>(row + 8 * j) = make_uint2(app_c0, app_c1);
              } else {
                reinterpret_cast<uint32_t*>(row + 8 * j)[0] = app_c0;
                reinterpret_cast<uint32_t*>(row + 8 * j)[1] = app_c1;
              }
              row[D / 2 + j] = (uint8_t)app_sb;
            }
            // (later bulk copies refill this stage: order these writes first)
            fence_proxy_async_smem();
            __syncwarp();
          }
          const int rem = L - u * UT;  // keys of this unit (clipped per tile below)
          const int pmask = okbits & 0xFF;  // pages copied
          if (rem >= UT && pmask == (1 << U) - 1) {
            decode_unit<D, BS, false, DUP, FMT, kDecodeTilesPerStep>(
                sbase, rem, pmask, lo, bq, qmult, lo_sel, m_run, l_run, acc, g8, t4);
          } else {
            decode_unit<D, BS, true, DUP, FMT, kDecodeTilesPerStep>(
                sbase, rem, pmask, lo, bq, qmult, lo_sel, m_run, l_run, acc, g8, t4);
          }
          __syncwarp();
          if (!poisoned && k + kStages < nk) issue(k + kStages);
        }

        // ---- this warp's state for the segment piece. l per column summed
        // over the lanes' rows; DUP: the lo columns G..2G-1 folded onto heads
        // 0..G-1.
        const float l0 = warp_sum_g(l_run[0]), l1 = warp_sum_g(l_run[1]);
        if constexpr (DUP) {
          if ((G & 1) == 0) {  // column n + G sits G/2 lanes further, same slot
            const int dl = G >> 1;
#pragma unroll
            for (int m = 0; m < NCH; ++m)
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[m][i] += __shfl_down_sync(0xffffffffu, acc[m][i], dl);
          } else if (G == 1) {  // column 1 is the lo part of column 0, same lane
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
              acc[m][0] += acc[m][1];
              acc[m][2] += acc[m][3];
            }
          } else {  // G == 3: column n + 3 lives in lane t4 + (n + 3) / 2 - t4, slot (n + 3) & 1
            const int c0 = 2 * t4 + G, c1 = 2 * t4 + 1 + G;
            const int src0 = (lane & ~3) | min(3, c0 >> 1), src1 = (lane & ~3) | min(3, c1 >> 1);
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
              const float a0 = __shfl_sync(0xffffffffu, acc[m][0], src0);
              const float a1 = __shfl_sync(0xffffffffu, acc[m][1], src0);
              const float a2 = __shfl_sync(0xffffffffu, acc[m][2], src0);
              const float a3 = __shfl_sync(0xffffffffu, acc[m][3], src0);
              const float b0 = __shfl_sync(0xffffffffu, acc[m][0], src1);
              const float b1 = __shfl_sync(0xffffffffu, acc[m][1], src1);
              const float b2 = __shfl_sync(0xffffffffu, acc[m][2], src1);
              const float b3 = __shfl_sync(0xffffffffu, acc[m][3], src1);
              acc[m][0] += (c0 & 1) ? a1 : a0;
              acc[m][2] += (c0 & 1) ? a3 : a2;
              acc[m][1] += (c1 & 1) ? b1 : b0;
              acc[m][3] += (c1 & 1) ? b3 : b2;
            }
          }
        }

        const int i_first = warp_of(seg_start), i_last = warp_of(seg_end - 1);
        const bool whole = (i_first == i_last);
        const int slot = (s >= seg_start) ? 0 : 1;
        // column n = 2*t4 + j of this lane: rows d0 = g8*D/8 + 2m and d0 + 1
        // in acc[m][j] and acc[m][j + 2]
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int n = 2 * t4 + j;
          if (n < G) {
            const float ll = j ? l1 : l0;
            if (whole) {
              const float sc = (ll > 0.0f) ? v_scale / ll : 0.0f;
              const long long obase = ((long long)qt * a.num_q_heads + h * G + n) * D;
#pragma unroll
              for (int m = 0; m < NCH; ++m) {
                const int d0 = g8 * (D / 8) + 2 * m;
                write_output2(op, obase + d0, acc[m][j] * sc, acc[m][j + 2] * sc);
              }
            } else {
              const size_t ps = (size_t)gw * 2 + slot;
              float* dst = partials + (ps * G + n) * D;
#pragma unroll
              for (int m = 0; m < NCH; ++m) {
                const int d0 = g8 * (D / 8) + 2 * m;
                *reinterpret_cast<float2*>(dst + d0) = make_float2(acc[m][j], acc[m][j + 2]);
              }
              if (g8 == 0) {
                part_ml[(ps * G + n) * 2 + 0] = m_run[j];
                part_ml[(ps * G + n) * 2 + 1] = ll;
              }
            }
          }
        }
        if (!whole && lane == 0) cut_sg[2 * w + slot] = b * Hkv + h;
        __syncwarp();
        seg_f0 = pe;
        ++portion;
      }
    }
  }  // gw < n_eff

  // ---- 3. cut segments. Every thread's partial writes are made visible
  // before the block's tickets; the ticket that completes a segment's count
  // of contributing warps makes this block its merger.
  if (metadata_ready) grid_dependency_wait();  // (idle warps have not waited yet)
  __threadfence();
  __syncthreads();
  if (tid < 2 * nw) {
    const int sg = cut_sg[tid];
    bool first = sg >= 0;
    int cnt = 0;
    for (int j = 0; j < 2 * nw; ++j) {
      if (cut_sg[j] == sg) {
        ++cnt;
        if (j < tid) first = false;
      }
    }
    if (first) {
      const int b = sg / Hkv, h = sg - b * Hkv, ss = cum[b] + h * sub[b];
      const int nc = warp_of(ss + sub[b] - 1) - warp_of(ss) + 1;
      if (atomicAdd(&counters[sg], cnt) + cnt == nc) {
        counters[sg] = 0;  // every contributor has arrived: ready for the next call
        won[atomicAdd(&nwon, 1)] = sg;
      }
    }
  }
  __syncthreads();
  const int n_won = nwon;
  if (n_won > 0) {
    __threadfence();
    for (int t = w; t < n_won * G; t += nw) {  // one (segment, query head) per warp
      const int sg = won[t / G], n = t % G;
      const int b = sg / Hkv, h = sg - b * Hkv, ss = cum[b] + h * sub[b];
      merge_head<D>(op, a.num_q_heads, partials, part_ml, G, h, n, sqt[b], warp_of(ss),
                    warp_of(ss + sub[b] - 1), ss, W, n_eff, lane, v_scale);
    }
  }
}

// The driver's tensor-map encoder, looked up once through the runtime.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// The cache as rows of pages: row r is the (block r / 2Hkv, K|V, head) page of
// `page_bytes` bytes, seen as eight-byte elements; one row per box.
static cudaError_t encode_page_rows(CUtensorMap* map, const uint8_t* cache, int64_t num_blocks,
                                    int num_kv_heads, int page_bytes) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)page_bytes / 8,
                              (cuuint64_t)num_blocks * 2 * num_kv_heads};
  const cuuint64_t strides[1] = {(cuuint64_t)page_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)page_bytes / 8, 1};
  const cuuint32_t elem_strides[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(cache),
                         dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Per-device launch facts, looked up once per (device, context) under a lock
// (outside any stream capture: the first call on a device should be an eager
// one).
struct DeviceFacts {
  int sms = 0;
  unsigned long long ctx = 0;  // context the attribute was set in
  bool smem_attr_set = false;
};

template <int D, int BS, bool DUP, int FMT>
static cudaError_t launch_decode_t(const AttentionArgs& a, cudaStream_t stream) {
  using S = DecodeShape<D, BS, FMT>;
  static std::mutex facts_mutex;
  static DeviceFacts facts[64];
  const int G = a.num_q_heads / a.num_kv_heads;
  const int nw = S::warps_for(a.num_seqs, G);
  if (nw < 1) return cudaErrorInvalidValue;
  const size_t smem = S::smem_bytes(a.num_seqs, G, nw);
  auto kern = decode_attention_kernel<D, BS, DUP, FMT>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  unsigned long long ctx = 0;
  err = current_context_id(&ctx);
  if (err != cudaSuccess) return err;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lock(facts_mutex);
    DeviceFacts& f = facts[dev];
    if (!f.smem_attr_set || ctx == 0 || f.ctx != ctx) {
      // allow the largest dynamic size the device permits beside the static part
      int optin = 0;
      err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
      if (err != cudaSuccess) return err;
      cudaFuncAttributes fa;
      err = cudaFuncGetAttributes(&fa, kern);
      if (err != cudaSuccess) return err;
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 optin - (int)fa.sharedSizeBytes);
      if (err != cudaSuccess) return err;
      err = cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev);
      if (err != cudaSuccess) return err;
      f.smem_attr_set = true;
      f.ctx = ctx;
    }
    sms = f.sms;
  }
  int per_sm = 1;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nw * 32, smem);
  if (err != cudaSuccess) return err;
  int grid = sms * max(1, per_sm);
  if (grid * nw > kDecodeWarps) grid = kDecodeWarps / nw;
  AttentionArgs ag = a;
  if constexpr (S::kGather) {
    err = encode_page_rows(&ag.kv_pages, a.cache, a.num_blocks, a.num_kv_heads, S::PAGE);
    if (err != cudaSuccess) return err;
  }
  // programmatic dependent launch: the grid may be scheduled while the
  // previous kernel on the stream finishes (its blocks wait on entry)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)(nw * 32));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, ag);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

int decode_warps(int head_size, int block_size, int num_seqs, int group, int kv_format) {
#define NVFP4_WARPS_CASE(DD, BB)                                                   \
  if (head_size == DD && block_size == BB)                                         \
    return kv_format == kFmtFp8 ? DecodeShape<DD, BB, kFmtFp8>::warps_for(num_seqs, group) \
                                : DecodeShape<DD, BB, kFmtNvfp4>::warps_for(num_seqs, group);
  NVFP4_WARPS_CASE(64, 16)
  NVFP4_WARPS_CASE(64, 32)
  NVFP4_WARPS_CASE(128, 16)
  NVFP4_WARPS_CASE(128, 32)
  NVFP4_WARPS_CASE(256, 16)
  NVFP4_WARPS_CASE(256, 32)
#undef NVFP4_WARPS_CASE
  return 0;
}

cudaError_t launch_decode_attention(const AttentionArgs& a, cudaStream_t stream) {
  const bool dup = (a.num_q_heads / a.num_kv_heads) <= 4;
  const bool fp8 = a.kv_format == kFmtFp8;
#define NVFP4_DECODE_CASE(DD, BB)                                                   \
  if (a.head_size == DD && a.block_size == BB) {                                    \
    if (fp8)                                                                        \
      return dup ? launch_decode_t<DD, BB, true, kFmtFp8>(a, stream)                \
                 : launch_decode_t<DD, BB, false, kFmtFp8>(a, stream);              \
    return dup ? launch_decode_t<DD, BB, true, kFmtNvfp4>(a, stream)                \
               : launch_decode_t<DD, BB, false, kFmtNvfp4>(a, stream);              \
  }
  NVFP4_DECODE_CASE(64, 16)
  NVFP4_DECODE_CASE(64, 32)
  NVFP4_DECODE_CASE(128, 16)
  NVFP4_DECODE_CASE(128, 32)
  NVFP4_DECODE_CASE(256, 16)
  NVFP4_DECODE_CASE(256, 32)
#undef NVFP4_DECODE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace nvfp4kv
