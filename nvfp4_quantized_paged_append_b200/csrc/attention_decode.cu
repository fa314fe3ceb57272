// Paged decode attention over the NVFP4 cache, split-KV across the whole GPU.
//
// What it computes ("FlashInfer backend adds end-to-end NVFP4 KV cache
// support": the decode kernel reads the packed E2M1 data plus the split-out
// FP8 block scales through a block table and writes FP8 output that is
// dequantized back to the model dtype): for every decode sequence b and query
// head hq, o = softmax(sm_scale * q K^T) V over the sequence's keys, with
// K = E2M1 * E4M3 * k_scale and V likewise with v_scale.
//
// Work decomposition (B200: 148 SMs): a sequence's keys are cut into units of
// 32 tokens (two 16-token pages, or one 32-token page). The units of all
// (sequence, kv head) segments are laid end to end and the flattened range is
// cut into equal contiguous pieces, one per warp of the whole grid, so every
// warp streams the same number of bytes whatever the length mix. Warps never
// wait for one another: a segment cut across warps leaves (acc, m, l) partials
// in the workspace, and the last warp to finish the segment (atomic ticket, no
// waiting) merges them with the log-sum-exp rule and writes the output.
//
// Each warp runs its own kStages-deep pipeline: one bulk async copy
// (cp.async.bulk) per K page and per V page of a unit into shared memory,
// completed on the stage's mbarrier. Pages are contiguous
// block_size*full_dim bytes in the HND layout. Block ids of the next unit to
// issue are loaded one unit ahead.
//
// Math per 16-token tile (all G <= 8 query heads of the kv head at once):
//   S^T[tok][n] = Khat[tok][:] . q[n][:]     mma.m16n8k16, A = Khat (f16,
//                                              dequantized in registers:
//                                              cvt e2m1x2->f16x2, times the
//                                              E4M3 scale; exact), B = q (f16,
//                                              scaled by a power of two)
//   online softmax in fp32 (exp2 domain) over the unit's 32 keys, with the
//   running max moved only when it grows by more than 2^8
//   O^T[d][n] += Vhat^T[d][tok] P[tok][n]     mma.m16n8k16, A = Vhat^T built
//                                              from nibble-transposed bytes,
//                                              P = f16 hi + f16 lo
// The contraction index of both products is permuted so that each lane's
// fragments come from contiguous bytes of a row (the same permutation is
// applied to q, and the PV output rows map back to d on the way out).
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

namespace {

constexpr int kUnitTok = 32;     // keys per unit
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;  // lazy max: P stays <= 2^8

// One persistent CTA per SM: all of an SM's warps belong to the same block, so
// none of them is starved behind an older co-resident block. head_size 256
// needs more registers and larger pages: fewer warps and stages.
template <int D>
struct DecodeCfg {
  static constexpr int kWarps = (D == 256) ? 8 : 12;
  static constexpr int kStages = (D == 256) ? 2 : 3;  // units in flight per warp
};

template <int D, int BS>
struct DecodeShape {
  static constexpr int kWarps = DecodeCfg<D>::kWarps;
  static constexpr int kStages = DecodeCfg<D>::kStages;
  static constexpr int F = D / 2 + D / 16;
  static constexpr int PAGE = BS * F;           // bytes of one (block, K|V, head) page
  static constexpr int U = kUnitTok / BS;       // pages per unit
  static constexpr int STAGE = 2 * U * PAGE;    // [K0][V0]([K1][V1]) bytes
  static constexpr int NCH = D / 16;            // MMA chunks along d
  static_assert(PAGE % 16 == 0, "pages must be 16-byte multiples");
  static size_t smem_bytes(int num_seqs, int group) {
    return (size_t)kWarps * kStages * STAGE       // ring
           + 8 * kWarps * kStages                 // mbarriers
           + 4 * kWarps * kStages                 // per-stage page-ok bits
           + 4 * (size_t)kWarps * group * D       // per-warp state (hi + lo combined)
           + 4 * ((size_t)num_seqs + 1);          // unit prefix
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

// Final epilogue for one output element.
__device__ __forceinline__ void write_output(const AttentionArgs& a, int64_t idx, float o,
                                             float o_scale) {
  if (a.o_f32) a.o_f32[idx] = o;
  const uint32_t code = f32_to_e4m3(__fdiv_rn(o, o_scale));
  a.o_fp8[idx] = (uint8_t)code;
  if (a.o_bf16)
    reinterpret_cast<__nv_bfloat16*>(a.o_bf16)[idx] =
        __float2bfloat16_rn(__fmul_rn(e4m3_to_f32(code), o_scale));
}

// Read-only global load that stays where it is written (a plain read-only load
// may be moved next to its first use, which would put its latency back on the
// critical path).
__device__ __forceinline__ int ldg_early(const int* p) {
  int v;
  asm volatile("ld.global.nc.b32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}

// Locate flattened unit f: advance cursor b so that cum[b] <= f < cum[b+1].
__device__ __forceinline__ int seek(const int* cum, int b, int f) {
  while (cum[b + 1] <= f) ++b;
  return b;
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

// The four E2M1 pairs held in the bytes of w -> four f16x2 (low nibble ->
// low half). Unpacking with mov.b32 lets each conversion read its byte
// directly, without shifts.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&r)[4]) {
  asm("{\n"
      ".reg .b8 b0, b1, b2, b3;\n"
      "mov.b32 {b0, b1, b2, b3}, %4;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n"
      "}\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(w));
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
  constexpr int NCH = D / 16;
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

// P^T of one tile -> B fragments: b0 = P[2t4, 2t4+1][g8], b1 = P[2t4+8, 2t4+9][g8].
// P = hi + lo (f16 each). DUP (G <= 4): lanes holding the duplicate columns
// G..2G-1 send lo in place of hi. Otherwise a second fragment carries lo.
template <bool DUP>
__device__ __forceinline__ void p_fragments(const float (&pr)[4], bool lo0, bool lo1, int g8,
                                            int t4, uint32_t (&bp)[2], uint32_t (&bpl)[2]) {
  const uint32_t h_even = pack_f16x2(pr[0], pr[2]);
  const uint32_t h_odd = pack_f16x2(pr[1], pr[3]);
  const float2 fe = __half22float2(*reinterpret_cast<const __half2*>(&h_even));
  const float2 fo = __half22float2(*reinterpret_cast<const __half2*>(&h_odd));
  const uint32_t l_even = pack_f16x2(pr[0] - fe.x, pr[2] - fe.y);
  const uint32_t l_odd = pack_f16x2(pr[1] - fo.x, pr[3] - fo.y);
  const int srcA = (2 * t4) * 4 + (g8 >> 1);
  const int srcB = srcA + 4;
  if constexpr (DUP) {
    const uint32_t x_even = lo0 ? l_even : h_even;  // column 2t4: rows g8, g8+8
    const uint32_t x_odd = lo1 ? l_odd : h_odd;     // column 2t4+1
    const uint32_t ae = __shfl_sync(0xffffffffu, x_even, srcA);
    const uint32_t ao = __shfl_sync(0xffffffffu, x_odd, srcA);
    const uint32_t be = __shfl_sync(0xffffffffu, x_even, srcB);
    const uint32_t bo = __shfl_sync(0xffffffffu, x_odd, srcB);
    const uint32_t A = (g8 & 1) ? ao : ae;   // (P[2t4][g8], P[2t4+8][g8])
    const uint32_t Bv = (g8 & 1) ? bo : be;  // (P[2t4+1][g8], P[2t4+9][g8])
    bp[0] = prmt(A, Bv, 0x5410);
    bp[1] = prmt(A, Bv, 0x7632);
    bpl[0] = bpl[1] = 0u;
  } else {
    const uint32_t ae = __shfl_sync(0xffffffffu, h_even, srcA);
    const uint32_t ao = __shfl_sync(0xffffffffu, h_odd, srcA);
    const uint32_t be = __shfl_sync(0xffffffffu, h_even, srcB);
    const uint32_t bo = __shfl_sync(0xffffffffu, h_odd, srcB);
    const uint32_t A = (g8 & 1) ? ao : ae;
    const uint32_t Bv = (g8 & 1) ? bo : be;
    bp[0] = prmt(A, Bv, 0x5410);
    bp[1] = prmt(A, Bv, 0x7632);
    const uint32_t lae = __shfl_sync(0xffffffffu, l_even, srcA);
    const uint32_t lao = __shfl_sync(0xffffffffu, l_odd, srcA);
    const uint32_t lbe = __shfl_sync(0xffffffffu, l_even, srcB);
    const uint32_t lbo = __shfl_sync(0xffffffffu, l_odd, srcB);
    const uint32_t LA = (g8 & 1) ? lao : lae;
    const uint32_t LB = (g8 & 1) ? lbo : lbe;
    bpl[0] = prmt(LA, LB, 0x5410);
    bpl[1] = prmt(LA, LB, 0x7632);
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

// One 32-token unit: tiles at kt0 and kt1 (V tiles v_off bytes further);
// tile 1 is skipped when valid1 <= 0 (MASK only).
template <int D, bool MASK, bool DUP>
__device__ __forceinline__ void decode_unit(uint32_t kt0, uint32_t kt1, int valid0, int valid1,
                                            const LaneOffsets& lo, const uint32_t (&bq)[D / 16][2],
                                            float qmult, bool lo0, bool lo1, float (&m_run)[2],
                                            float (&l_run)[2], float (&acc)[D / 16][4], int g8,
                                            int t4, uint32_t v_off) {
  constexpr int NCH = D / 16;
  const bool two = !MASK || valid1 > 0;
  float sa[4] = {0.f, 0.f, 0.f, 0.f};
  float sb[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  qk_tile<D, MASK>(kt0, lo, valid0, g8, bq, sa);
  if (two) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sb[i] = 0.f;
    qk_tile<D, MASK>(kt1, lo, valid1, g8, bq, sb);
  }
  // ---- online softmax over the unit's 32 keys (log2 units, lazy max)
  float pa[4], pb[4];
  {
    const float t0 = warp_max_g(fmaxf(fmaxf(sa[0], sa[2]), fmaxf(sb[0], sb[2]))) * qmult;
    const float t1 = warp_max_g(fmaxf(fmaxf(sa[1], sa[3]), fmaxf(sb[1], sb[3]))) * qmult;
    const bool up = (t0 > m_run[0] + kRescaleThresh) || (t1 > m_run[1] + kRescaleThresh);
    if (__any_sync(0xffffffffu, up)) {
      const float n0 = fmaxf(m_run[0], t0), n1 = fmaxf(m_run[1], t1);
      // ex2(-inf) = 0 clears a column seen for the first time (its acc and l are 0)
      const float al0 = ex2(m_run[0] - (n0 == -INFINITY ? 0.f : n0));
      const float al1 = ex2(m_run[1] - (n1 == -INFINITY ? 0.f : n1));
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
    }
    const float mu0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
    const float mu1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
    pa[0] = ex2(fmaf(sa[0], qmult, -mu0));
    pa[1] = ex2(fmaf(sa[1], qmult, -mu1));
    pa[2] = ex2(fmaf(sa[2], qmult, -mu0));
    pa[3] = ex2(fmaf(sa[3], qmult, -mu1));
    pb[0] = ex2(fmaf(sb[0], qmult, -mu0));
    pb[1] = ex2(fmaf(sb[1], qmult, -mu1));
    pb[2] = ex2(fmaf(sb[2], qmult, -mu0));
    pb[3] = ex2(fmaf(sb[3], qmult, -mu1));
    l_run[0] += (pa[0] + pa[2]) + (pb[0] + pb[2]);
    l_run[1] += (pa[1] + pa[3]) + (pb[1] + pb[3]);
  }
  uint32_t bpa[2], bpla[2];
  p_fragments<DUP>(pa, lo0, lo1, g8, t4, bpa, bpla);
  pv_tile<D, MASK, DUP>(kt0 + v_off, lo, valid0, t4, bpa, bpla, acc);
  if (two) {
    uint32_t bpb[2], bplb[2];
    p_fragments<DUP>(pb, lo0, lo1, g8, t4, bpb, bplb);
    pv_tile<D, MASK, DUP>(kt1 + v_off, lo, valid1, t4, bpb, bplb, acc);
  }
}

}  // namespace

template <int D, int BS, bool DUP>
__global__ void __launch_bounds__(DecodeCfg<D>::kWarps * 32, 1)
    decode_attention_kernel(const AttentionArgs a) {
  using S = DecodeShape<D, BS>;
  constexpr int kWarps = S::kWarps, kStages = S::kStages;
  constexpr int F = S::F, PAGE = S::PAGE, NCH = S::NCH, U = S::U, STAGE = S::STAGE;
  extern __shared__ __align__(128) uint8_t smem[];
  const int Hkv = a.num_kv_heads, G = a.num_q_heads / Hkv;
  const int B = a.num_seqs;
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kWarps * kStages * STAGE);
  int* page_ok = reinterpret_cast<int*>(bars + kWarps * kStages);
  float* wstate = reinterpret_cast<float*>(page_ok + kWarps * kStages);  // [kWarps][G][D]
  int* cum = reinterpret_cast<int*>(wstate + kWarps * G * D);
  __shared__ int warp_tot[kWarps];

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.workspace);
  const WorkspaceLayout wl = workspace_layout(B, Hkv, D, G);
  int* counters = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.counters_off);
  float* partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.partials_off);
  float* part_ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.ml_off);

  // ---- 1. unit prefix over decode sequences (q_len == 1): cum[b]
  int carry = 0;
  for (int base = 0; base < B; base += kWarps * 32) {
    const int b = base + tid;
    int val = 0;
    if (b < B) {
      const int ql = a.qo_indptr ? a.qo_indptr[b + 1] - a.qo_indptr[b] : 1;
      const int L = a.seq_lens[b];
      // pages of the sequence, at least one (an empty sequence still writes
      // its zero row) and at most the block table's width; then units
      const int pages = min(a.max_blocks_per_seq, max(1, (L + BS - 1) / BS));
      val = (ql == 1) ? ((pages + U - 1) / U) * Hkv : 0;
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
#pragma unroll
    for (int i = 0; i < kWarps; ++i) {
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
  const int n_eff = min((int)gridDim.x * kWarps, W);
  const int gw = blockIdx.x * kWarps + w;
  if (gw >= n_eff) return;
  const int s = (int)((long long)gw * W / n_eff);
  const int e = (int)((long long)(gw + 1) * W / n_eff);
  auto warp_of = [&](int f) { return (int)(((long long)(f + 1) * n_eff - 1) / W); };

  uint64_t* my_bars = bars + w * kStages;
  int* my_ok = page_ok + w * kStages;
  uint8_t* my_ring_p = ring + (size_t)w * kStages * STAGE;
  const uint32_t my_ring = smem_u32(my_ring_p);
  float* my_state = wstate + (size_t)w * G * D;
  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&my_bars[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int nk = e - s;
  bool poisoned = false;

  // Block ids are fetched 32 units at a time, lane j holding unit base + j of
  // this warp (two banks, refilled a whole batch ahead), so no global load
  // latency sits between finishing a unit and issuing the copies of the next.
  int bid0[2] = {0, 0}, bid1[2] = {0, 0}, bmeta[2] = {0, 0};  // meta: h << 8 | n_pg << 1 | keys
  int l_ib = 0;  // this lane's cursor into cum
  auto batch_load = [&](int base) {
    const int bank = (base >> 5) & 1;
    bid0[bank] = bid1[bank] = bmeta[bank] = 0;
    const int f = s + base + lane;
    if (f < e) {
      l_ib = seek(cum, l_ib, f);
      const int uu = (cum[l_ib + 1] - cum[l_ib]) / Hkv;
      const int hh = (f - cum[l_ib]) / uu;
      const int u = f - cum[l_ib] - hh * uu;
      const int Lb = a.seq_lens[l_ib];
      const int pages = min(a.max_blocks_per_seq, max(1, (Lb + BS - 1) / BS));
      const int npg = min(U, pages - u * U);
      const int* row = a.block_table + (long long)l_ib * a.max_blocks_per_seq + u * U;
      if (Lb > 0) {
        bid0[bank] = ldg_early(row);
        if (U > 1 && npg > 1) bid1[bank] = ldg_early(row + 1);
      }
      bmeta[bank] = (hh << 8) | (npg << 1) | (Lb > 0 ? 1 : 0);
    }
  };
  auto issue = [&](int k) {  // unit k of this warp into stage k % kStages
    const int st = k % kStages;
    const int bank = (k >> 5) & 1, src = k & 31;
    const int meta = __shfl_sync(0xffffffffu, bmeta[bank], src);
    long long blk[2];
    blk[0] = __shfl_sync(0xffffffffu, bid0[bank], src);
    blk[1] = __shfl_sync(0xffffffffu, bid1[bank], src);
    const int n_pg = (meta >> 1) & 0x7F, n_h = meta >> 8;
    const bool has_keys = meta & 1;
    int okbits = 0;
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (j < n_pg && has_keys) {
        if (blk[j] >= 0 && blk[j] < a.num_blocks) {
          okbits |= 1 << j;
        } else {
          if (lane == 0) atomicOr(status, kDevBadBlock);
          blk[j] = 0;  // copy a valid page instead; its rows are masked
        }
      } else {
        blk[j] = 0;
      }
    }
    // The stage being refilled was last read by this warp's own ld.shared
    // instructions, all complete before the __syncwarp that precedes this
    // call; the copies only write, so no proxy fence is needed here.
    if (lane == 0) {
      my_ok[st] = okbits;
      mbar_arrive_expect_tx(&my_bars[st], 2 * PAGE * n_pg);
#pragma unroll
      for (int j = 0; j < U; ++j) {
        if (j < n_pg) {
          const uint8_t* kp = a.cache + ((blk[j] * 2) * Hkv + n_h) * (long long)PAGE;
          uint8_t* dst = my_ring_p + (size_t)st * STAGE + j * 2 * PAGE;
          bulk_g2s(dst, kp, PAGE, &my_bars[st]);
          bulk_g2s(dst + PAGE, kp + (long long)Hkv * PAGE, PAGE, &my_bars[st]);
        }
      }
    }
    // entering a new batch of 32: fetch the one after it into the other bank
    if ((k & 31) == 0 && k + 32 < nk) batch_load(k + 32);
  };

  batch_load(0);
  for (int k = 0; k < min(kStages, nk); ++k) issue(k);

  const float k_scale = __ldg(a.kv_scales);
  const float v_scale = __ldg(a.kv_scales + 1);
  const float o_scale = __ldg(a.o_scale);
  const LaneOffsets lo = lane_offsets<D>(g8, t4);
  // DUP: columns G..2G-1 of the lanes' B fragments carry lo parts
  const bool lo0 = DUP && (2 * t4 >= G) && (2 * t4 < 2 * G);
  const bool lo1 = DUP && (2 * t4 + 1 >= G) && (2 * t4 + 1 < 2 * G);

  int k = 0;  // this warp's unit counter, continuous across portions
  int seg_f0 = s;
  int cb = 0;
  while (seg_f0 < e) {
    cb = seek(cum, cb, seg_f0);
    const int b = cb;
    const int UB = (cum[b + 1] - cum[b]) / Hkv;
    const int h = (seg_f0 - cum[b]) / UB;
    const int seg_start = cum[b] + h * UB, seg_end = seg_start + UB;
    const int pe = min(e, seg_end);
    const int L = a.seq_lens[b];
    const int qt = a.qo_indptr ? a.qo_indptr[b] : b;

    // ---- query fragments: lane (g8, t4) holds q[head of column g8][t4*D/4 + i].
    // DUP: columns G..2G-1 repeat heads 0..G-1 (their P carries the lo part).
    const int qhead = DUP ? (g8 < 2 * G ? g8 % G : -1) : (g8 < G ? g8 : -1);
    uint32_t bq[NCH][2];
    float qmult;
    {
      float qv[D / 4];
      if (qhead >= 0) {
        const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                    (long long)qt * a.q_token_stride +
                                    (long long)(h * G + qhead) * D + t4 * (D / 4);
#pragma unroll
        for (int i = 0; i < D / 4; i += 8) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + i));
          const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
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

    // ---- running state: columns n0 = 2*t4, n1 = 2*t4+1 (lazily moved max)
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    float acc[NCH][4];
#pragma unroll
    for (int c = 0; c < NCH; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;

    while (k < nk && s + k < pe) {
      const int u = s + k - seg_start;
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
      const int rem = L - u * kUnitTok;
      // tile t covers keys 16t..16t+15 of the unit; page t (block_size 16) or 0
      int v0 = min(16, rem), v1 = min(16, rem - 16);
      if (BS == 16) {
        if (!(okbits & 1)) v0 = 0;
        if (!(okbits & 2)) v1 = 0;
      } else if (!(okbits & 1)) {
        v0 = v1 = 0;
      }
      const uint32_t kt0 = sbase;
      const uint32_t kt1 = (BS == 16) ? sbase + 2 * PAGE : sbase + 16 * F;
      if (v0 >= 16 && v1 >= 16) {
        decode_unit<D, false, DUP>(kt0, kt1, 16, 16, lo, bq, qmult, lo0, lo1, m_run, l_run, acc,
                                   g8, t4, PAGE);
      } else if (v0 > 0 || v1 > 0) {
        // an unusable page next to a usable one: put the usable tile first
        const bool first = v0 > 0;
        decode_unit<D, true, DUP>(first ? kt0 : kt1, first ? kt1 : kt0, first ? v0 : v1,
                                  first ? max(v1, 0) : 0, lo, bq, qmult, lo0, lo1, m_run, l_run,
                                  acc, g8, t4, PAGE);
      }
      __syncwarp();
      if (!poisoned && k + kStages < nk) issue(k + kStages);
      ++k;
    }

    // ---- this warp's state for the segment piece: m per column (uniform over
    // g8), l summed over the lanes' rows, acc per head in shared memory
    const float l0 = warp_sum_g(l_run[0]), l1 = warp_sum_g(l_run[1]);
    {
      const int n0 = 2 * t4, n1 = 2 * t4 + 1;
#pragma unroll
      for (int m = 0; m < NCH; ++m) {  // heads' own (hi) columns first
        const int d0 = g8 * (D / 8) + 2 * m;
        if (n0 < G) {
          my_state[n0 * D + d0] = acc[m][0];
          my_state[n0 * D + d0 + 1] = acc[m][2];
        }
        if (n1 < G) {
          my_state[n1 * D + d0] = acc[m][1];
          my_state[n1 * D + d0 + 1] = acc[m][3];
        }
      }
      if constexpr (DUP) {  // then add the lo columns G..2G-1 onto heads 0..G-1
        __syncwarp();
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
          const int d0 = g8 * (D / 8) + 2 * m;
          if (n0 >= G && n0 < 2 * G) {
            my_state[(n0 - G) * D + d0] += acc[m][0];
            my_state[(n0 - G) * D + d0 + 1] += acc[m][2];
          }
          if (n1 >= G && n1 < 2 * G) {
            my_state[(n1 - G) * D + d0] += acc[m][1];
            my_state[(n1 - G) * D + d0 + 1] += acc[m][3];
          }
        }
      }
      __syncwarp();
    }
    // m and l of column n live in the lanes with t4 = n / 2 (lane n / 2 has g8 = 0), slot n & 1
    auto col_ml = [&](int n, float& mm, float& ll) {
      const int src = n >> 1;
      const float ma = __shfl_sync(0xffffffffu, m_run[0], src);
      const float mb = __shfl_sync(0xffffffffu, m_run[1], src);
      const float la = __shfl_sync(0xffffffffu, l0, src);
      const float lb = __shfl_sync(0xffffffffu, l1, src);
      mm = (n & 1) ? mb : ma;
      ll = (n & 1) ? lb : la;
    };

    const int i_first = warp_of(seg_start), i_last = warp_of(seg_end - 1);
    const bool whole = (i_first == i_last);
    const int slot = (s >= seg_start) ? 0 : 1;
    for (int n = 0; n < G; ++n) {
      float mm, ll;
      col_ml(n, mm, ll);
      if (whole) {
        const float inv = (ll > 0.0f) ? 1.0f : 0.0f;
        for (int d = lane; d < D; d += 32) {
          const float o = inv != 0.0f ? __fdiv_rn(my_state[n * D + d], ll) * v_scale : 0.0f;
          write_output(a, ((long long)qt * a.num_q_heads + h * G + n) * D + d, o, o_scale);
        }
      } else {
        const size_t ps = (size_t)gw * 2 + slot;
        for (int d = lane; d < D; d += 32) partials[(ps * G + n) * D + d] = my_state[n * D + d];
        if (lane == 0) {
          part_ml[(ps * G + n) * 2 + 0] = mm;
          part_ml[(ps * G + n) * 2 + 1] = ll;
        }
      }
    }
    if (!whole) {
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(&counters[b * Hkv + h], 1) == i_last - i_first);
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        // lane c fetches contributor c's (m, l) for every head (32 at a time)
        const int nc = i_last - i_first + 1;
        for (int n0 = 0; n0 < G; n0 += 2) {  // two heads per pass
          const int nh = min(2, G - n0);
          float M[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
          float sum[2][D / 32];
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int j = 0; j < D / 32; ++j) sum[q][j] = 0.0f;
          for (int c0 = 0; c0 < nc; c0 += 32) {
            const int cnt = min(32, nc - c0);
            float mi[2] = {-INFINITY, -INFINITY}, li[2] = {0.f, 0.f};
            unsigned long long ps_mine = 0;
            if (lane < cnt) {
              const int i = i_first + c0 + lane;
              const int si = (int)((long long)i * W / n_eff);
              ps_mine = (size_t)i * 2 + ((si >= seg_start) ? 0 : 1);
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                if (q < nh) {
                  mi[q] = __ldcg(part_ml + (ps_mine * G + n0 + q) * 2);
                  li[q] = __ldcg(part_ml + (ps_mine * G + n0 + q) * 2 + 1);
                }
              }
            }
            // rescale what is accumulated so far to the new running max
            float sc[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float mx = mi[q];
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
              const float Mn = fmaxf(M[q], mx);
              const float Mu = (Mn == -INFINITY) ? 0.0f : Mn;
              const float al = ex2(M[q] - Mu);
              lsum[q] *= al;
#pragma unroll
              for (int j = 0; j < D / 32; ++j) sum[q][j] *= al;
              M[q] = Mn;
              sc[q] = ex2(mi[q] - Mu);
              float lw = li[q] * sc[q];
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
              lsum[q] += lw;
            }
            for (int c = 0; c < cnt; c += 4) {
              float v[4][2][D / 32], scv[4][2];
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const unsigned long long ps = __shfl_sync(0xffffffffu, ps_mine, (c + r) & 31);
                scv[r][0] = __shfl_sync(0xffffffffu, sc[0], (c + r) & 31);
                scv[r][1] = __shfl_sync(0xffffffffu, sc[1], (c + r) & 31);
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                  for (int j = 0; j < D / 32; ++j)
                    v[r][q][j] = (c + r < cnt && q < nh)
                                     ? __ldcg(partials + (ps * G + n0 + q) * D + lane + 32 * j)
                                     : 0.0f;
              }
#pragma unroll
              for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                  for (int j = 0; j < D / 32; ++j) sum[q][j] += v[r][q][j] * scv[r][q];
            }
          }
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (q < nh) {
#pragma unroll
              for (int j = 0; j < D / 32; ++j) {
                const int d = lane + 32 * j;
                const float o = (lsum[q] > 0.0f) ? __fdiv_rn(sum[q][j], lsum[q]) * v_scale : 0.0f;
                write_output(a, ((long long)qt * a.num_q_heads + h * G + n0 + q) * D + d, o,
                             o_scale);
              }
            }
          }
        }
        if (lane == 0) counters[b * Hkv + h] = 0;
      }
    }
    __syncwarp();
    seg_f0 = pe;
  }
}

// Per-device launch facts, looked up once (outside any stream capture: the
// first call on a device should be an eager one).
struct DeviceFacts {
  int sms = 0;
  bool smem_attr_set[2] = {false, false};
};

template <int D, int BS, bool DUP>
static cudaError_t launch_decode_t(const AttentionArgs& a, cudaStream_t stream) {
  using S = DecodeShape<D, BS>;
  constexpr int kWarps = S::kWarps;
  static DeviceFacts facts[64];
  const int G = a.num_q_heads / a.num_kv_heads;
  const size_t smem = S::smem_bytes(a.num_seqs, G);
  auto kern = decode_attention_kernel<D, BS, DUP>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  DeviceFacts& f = facts[dev & 63];
  if (!f.smem_attr_set[DUP]) {
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
    f.smem_attr_set[DUP] = true;
  }
  int per_sm = 1;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarps * 32, smem);
  if (err != cudaSuccess) return err;
  int grid = f.sms * max(1, per_sm);
  if (grid > kDecodeCtas) grid = kDecodeCtas;
  kern<<<grid, kWarps * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

size_t decode_smem_bytes(int head_size, int block_size, int num_seqs, int group) {
#define NVFP4_SMEM_CASE(DD, BB) \
  if (head_size == DD && block_size == BB) return DecodeShape<DD, BB>::smem_bytes(num_seqs, group);
  NVFP4_SMEM_CASE(64, 16)
  NVFP4_SMEM_CASE(64, 32)
  NVFP4_SMEM_CASE(128, 16)
  NVFP4_SMEM_CASE(128, 32)
  NVFP4_SMEM_CASE(256, 16)
  NVFP4_SMEM_CASE(256, 32)
#undef NVFP4_SMEM_CASE
  return 0;
}

cudaError_t launch_decode_attention(const AttentionArgs& a, cudaStream_t stream) {
  const bool dup = (a.num_q_heads / a.num_kv_heads) <= 4;
#define NVFP4_DECODE_CASE(DD, BB)                         \
  if (a.head_size == DD && a.block_size == BB)            \
    return dup ? launch_decode_t<DD, BB, true>(a, stream) \
               : launch_decode_t<DD, BB, false>(a, stream);
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
