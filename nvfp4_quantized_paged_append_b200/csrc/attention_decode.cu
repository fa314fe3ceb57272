// Paged decode attention over the NVFP4 cache, split-KV across the whole GPU.
//
// What it computes ("FlashInfer backend adds end-to-end NVFP4 KV cache
// support": the decode kernel reads the packed E2M1 data plus the split-out
// FP8 block scales through a block table and writes FP8 output that is
// dequantized back to the model dtype): for every decode sequence b and query
// head hq, o = softmax(sm_scale * q K^T) V over the sequence's keys, with
// K = E2M1 * E4M3 * k_scale and V likewise with v_scale.
//
// Work decomposition (B200: 148 SMs): the KV pages of all (sequence, kv head)
// segments are laid end to end and the flattened page range is cut into
// gridDim.x equal contiguous pieces, one per CTA, so every SM streams the same
// number of bytes whatever the length mix. A segment cut across CTAs leaves
// (acc, m, l) partials in the workspace; the last CTA to finish a segment
// (atomic ticket, no waiting) merges them with the log-sum-exp rule and
// writes the output.
//
// Inside a CTA each of the 4 warps owns every 4th page of the piece and runs
// its own 4-stage pipeline: lane 0 issues one bulk async copy (cp.async.bulk)
// per K page and per V page into shared memory, completed on the stage's
// mbarrier. Pages are contiguous block_size*full_dim bytes in the HND layout.
//
// Math per 16-token tile (all G <= 8 query heads of the kv head at once):
//   S^T[tok][n] = Khat[tok][:] . q[n][:]     mma.m16n8k16, A = Khat (f16,
//                                              dequantized in registers:
//                                              cvt e2m1x2->f16x2, times the
//                                              E4M3 scale; exact), B = q (f16,
//                                              scaled by a power of two)
//   online softmax in fp32 (exp2 domain), P rounded to f16
//   O^T[d][n] += Vhat^T[d][tok] P[tok][n]     mma.m16n8k16, A = Vhat^T built
//                                              from nibble-transposed bytes
// The contraction index of both products is permuted so that each lane's
// fragments come from contiguous bytes of a row (the same permutation is
// applied to q, and the PV output rows map back to d on the way out).
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

namespace {

constexpr int kWarps = 4;
constexpr int kStages = 4;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int BS>
struct DecodeShape {
  static constexpr int F = D / 2 + D / 16;
  static constexpr int PAGE = BS * F;  // bytes of one (block, K|V, head) page
  static constexpr int NCH = D / 16;   // MMA chunks along d
  static constexpr int KW = D / 32;    // u32 words of K data per lane per row
  static constexpr int VW = D / 64;    // u32 words of V data per lane per token (>= 1)
  static_assert(PAGE % 16 == 0, "pages must be 16-byte multiples");
  static size_t smem_bytes(int num_seqs) {
    return (size_t)kWarps * kStages * 2 * PAGE      // ring
           + 8 * kWarps * kStages                   // mbarriers
           + 4 * kWarps * kStages                   // page ok flags
           + 4 * (2 * kWarps * 8)                   // m, l
           + 4 * (size_t)kWarps * 8 * D             // acc
           + 4 * ((size_t)num_seqs + 1)             // page prefix
           + 16;                                    // flag
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

// Locate flattened page f: advance cursor b so that cum[b] <= f < cum[b+1].
__device__ __forceinline__ int seek(const int* cum, int b, int f) {
  while (cum[b + 1] <= f) ++b;
  return b;
}

}  // namespace

template <int D, int BS>
__global__ void __launch_bounds__(kWarps * 32) decode_attention_kernel(const AttentionArgs a) {
  using S = DecodeShape<D, BS>;
  constexpr int F = S::F, PAGE = S::PAGE, NCH = S::NCH;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kWarps * kStages * 2 * PAGE);
  int* page_ok = reinterpret_cast<int*>(bars + kWarps * kStages);
  float* st_m = reinterpret_cast<float*>(page_ok + kWarps * kStages);
  float* st_l = st_m + kWarps * 8;
  float* st_acc = st_l + kWarps * 8;
  int* cum = reinterpret_cast<int*>(st_acc + kWarps * 8 * D);
  int* flag = cum + a.num_seqs + 1;
  __shared__ int warp_tot[kWarps];

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int Hkv = a.num_kv_heads, G = a.num_q_heads / Hkv;
  const int B = a.num_seqs;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.workspace);
  const WorkspaceLayout wl = workspace_layout(B, Hkv, D);
  int* counters = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.counters_off);
  float* partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.partials_off);
  float* part_ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + wl.ml_off);

  // ---- 1. page prefix over decode sequences (q_len == 1): cum[b]
  int carry = 0;
  for (int base = 0; base < B; base += kWarps * 32) {
    const int b = base + tid;
    int val = 0;
    if (b < B) {
      const int ql = a.qo_indptr ? a.qo_indptr[b + 1] - a.qo_indptr[b] : 1;
      const int L = a.seq_lens[b];
      // pages of the sequence, at least one (an empty sequence still writes
      // its zero row) and at most the block table's width
      val = (ql == 1) ? min(a.max_blocks_per_seq, max(1, (L + BS - 1) / BS)) * Hkv : 0;
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
  const int W = cum[B];
  const int n_eff = min((int)gridDim.x, W);
  const int cta = blockIdx.x;
  if (cta >= n_eff) return;
  const int s = (int)((long long)cta * W / n_eff);
  const int e = (int)((long long)(cta + 1) * W / n_eff);
  auto cta_of = [&](int f) { return (int)(((long long)(f + 1) * n_eff - 1) / W); };

  // ---- 2. per-warp pipeline state
  uint64_t* my_bars = bars + w * kStages;
  int* my_ok = page_ok + w * kStages;
  uint8_t* my_ring = ring + (size_t)w * kStages * 2 * PAGE;
  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&my_bars[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int nk = (e - s > w) ? (e - s - w + kWarps - 1) / kWarps : 0;
  bool poisoned = false;
  int issue_b = 0;

  auto issue = [&](int k) {  // lane 0 only
    const int f = s + w + kWarps * k;
    issue_b = seek(cum, issue_b, f);
    const int P = (cum[issue_b + 1] - cum[issue_b]) / Hkv;
    const int within = f - cum[issue_b];
    const int h = within / P, p = within % P;
    const int L = a.seq_lens[issue_b];
    int ok = L > 0;
    long long blk = 0;
    if (ok) {
      blk = __ldg(a.block_table + (long long)issue_b * a.max_blocks_per_seq + p);
      if (blk < 0 || blk >= a.num_blocks) {
        atomicOr(status, kDevBadBlock);
        ok = 0;
        blk = 0;
      }
    }
    const int st = k % kStages;
    my_ok[st] = ok;
    const uint8_t* kp = a.cache + ((blk * 2 + 0) * Hkv + h) * (long long)PAGE;
    const uint8_t* vp = kp + (long long)Hkv * PAGE;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&my_bars[st], 2 * PAGE);
    bulk_g2s(my_ring + (size_t)st * 2 * PAGE, kp, PAGE, &my_bars[st]);
    bulk_g2s(my_ring + (size_t)st * 2 * PAGE + PAGE, vp, PAGE, &my_bars[st]);
  };

  if (lane == 0)
    for (int k = 0; k < min(kStages, nk); ++k) issue(k);

  const float k_scale = __ldg(a.kv_scales);
  const float v_scale = __ldg(a.kv_scales + 1);
  const float o_scale = __ldg(a.o_scale);

  int k = 0;  // this warp's page counter, continuous across portions
  int seg_f0 = s;
  int cb = 0;
  while (seg_f0 < e) {
    cb = seek(cum, cb, seg_f0);
    const int b = cb;
    const int P = (cum[b + 1] - cum[b]) / Hkv;
    const int h = (seg_f0 - cum[b]) / P;
    const int seg_start = cum[b] + h * P, seg_end = seg_start + P;
    const int pe = min(e, seg_end);
    const int L = a.seq_lens[b];
    const int qt = a.qo_indptr ? a.qo_indptr[b] : b;

    // ---- query fragments: lane (g8, t4) holds q[head of column g8][t4*D/4 + i].
    // With G <= 4, columns G..2G-1 repeat heads 0..G-1: their probabilities
    // carry the low-order f16 part of P (see the P^T step), so P reaches the
    // PV product with ~22 bits at no extra MMA.
    const bool dup = G <= 4;
    const int qhead = dup ? (g8 < 2 * G ? g8 % G : -1) : (g8 < G ? g8 : -1);
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
      int ex = (mx > 0.0f) ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126 : 1;
      int sh = min(126, max(-126, 15 - ex));
      const float qs = __uint_as_float((uint32_t)(sh + 127) << 23);
      const float qds = __uint_as_float((uint32_t)(127 - sh) << 23);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        bq[c][0] = pack_f16x2(qv[4 * c] * qs, qv[4 * c + 1] * qs);
        bq[c][1] = pack_f16x2(qv[4 * c + 2] * qs, qv[4 * c + 3] * qs);
      }
      qmult = a.sm_scale * k_scale * kLog2e * qds;
    }

    // ---- running state: columns n0 = 2*t4, n1 = 2*t4+1
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    float acc[NCH][4];
#pragma unroll
    for (int c = 0; c < NCH; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;

    while (k < nk && s + w + kWarps * k < pe) {
      const int f = s + w + kWarps * k;
      const int p = f - seg_start;
      const int st = k % kStages;
      bool ok = false;
      if (!poisoned) {
        if (mbar_wait_bounded(&my_bars[st], (uint32_t)((k / kStages) & 1))) {
          ok = my_ok[st] != 0;
        } else {
          poisoned = true;
          if (lane == 0) atomicOr(status, kDevTimeout);
        }
      }
      const uint8_t* kpage = my_ring + (size_t)st * 2 * PAGE;
      const uint8_t* vpage = kpage + PAGE;
#pragma unroll
      for (int tt = 0; tt < BS / 16; ++tt) {
        const int tok0 = p * BS + tt * 16;  // sequence position of tile row 0
        // ---------------- S^T = Khat q^T
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int r0 = tt * 16 + g8, r1 = r0 + 8;
          const bool v0 = ok && (tok0 + g8 < L), v1 = ok && (tok0 + g8 + 8 < L);
          const uint8_t* row0 = kpage + r0 * F;
          const uint8_t* row1 = kpage + r1 * F;
          uint32_t kw0[S::KW], kw1[S::KW];
#pragma unroll
          for (int i = 0; i < S::KW; ++i) {
            kw0[i] = ld_shared_u32(smem_u32(row0 + t4 * (D / 8) + 4 * i));
            kw1[i] = ld_shared_u32(smem_u32(row1 + t4 * (D / 8) + 4 * i));
          }
          constexpr int NG = D / 64;  // scale groups per lane
          uint32_t sc0[NG], sc1[NG];
#pragma unroll
          for (int gi = 0; gi < NG; ++gi) {
            const uint32_t b0 = v0 ? row0[D / 2 + t4 * NG + gi] : 0u;
            const uint32_t b1 = v1 ? row1[D / 2 + t4 * NG + gi] : 0u;
            sc0[gi] = e4m3x2_to_f16x2(b0 | (b0 << 8));
            sc1[gi] = e4m3x2_to_f16x2(b1 | (b1 << 8));
          }
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const int by = 2 * c;  // lane-segment byte for k = 2t4,2t4+1; +1 for k+8
            const uint32_t w0 = kw0[by >> 2], w1 = kw1[by >> 2];
            const int sh0 = 8 * (by & 3);
            uint32_t af[4];
            af[0] = hmul2_u32(e2m1x2_to_f16x2((w0 >> sh0) & 0xFFu), sc0[c / 4]);
            af[1] = hmul2_u32(e2m1x2_to_f16x2((w1 >> sh0) & 0xFFu), sc1[c / 4]);
            af[2] = hmul2_u32(e2m1x2_to_f16x2((w0 >> (sh0 + 8)) & 0xFFu), sc0[c / 4]);
            af[3] = hmul2_u32(e2m1x2_to_f16x2((w1 >> (sh0 + 8)) & 0xFFu), sc1[c / 4]);
            mma_f16_16816(sacc, af, bq[c]);
          }
          // scale to log2 units and mask rows outside the sequence
          sacc[0] = v0 ? sacc[0] * qmult : -INFINITY;
          sacc[1] = v0 ? sacc[1] * qmult : -INFINITY;
          sacc[2] = v1 ? sacc[2] * qmult : -INFINITY;
          sacc[3] = v1 ? sacc[3] * qmult : -INFINITY;
        }
        // ---------------- online softmax per column
        float pr[4];
        {
          const float mx0 = warp_max_g(fmaxf(sacc[0], sacc[2]));
          const float mx1 = warp_max_g(fmaxf(sacc[1], sacc[3]));
          const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
          const float mu0 = (mn0 == -INFINITY) ? 0.0f : mn0;
          const float mu1 = (mn1 == -INFINITY) ? 0.0f : mn1;
          const float al0 = ex2(m_run[0] - mu0), al1 = ex2(m_run[1] - mu1);
          m_run[0] = mn0;
          m_run[1] = mn1;
          pr[0] = ex2(sacc[0] - mu0);
          pr[1] = ex2(sacc[1] - mu1);
          pr[2] = ex2(sacc[2] - mu0);
          pr[3] = ex2(sacc[3] - mu1);
          l_run[0] = l_run[0] * al0 + pr[0] + pr[2];
          l_run[1] = l_run[1] * al1 + pr[1] + pr[3];
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            acc[c][0] *= al0;
            acc[c][1] *= al1;
            acc[c][2] *= al0;
            acc[c][3] *= al1;
          }
        }
        // ---------------- P^T -> B fragment: b0 = P[2t4, 2t4+1][g8], b1 = P[2t4+8, 2t4+9][g8]
        // P = hi + lo, both f16: hi = f16(p), lo = f16(p - hi). With G <= 4 the
        // lo part sits in the duplicate columns G..2G-1; otherwise it is a
        // second B fragment and a second MMA into the same accumulators.
        uint32_t bp[2], bpl[2];
        {
          float lo[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) lo[i] = pr[i] - __half2float(__float2half_rn(pr[i]));
          const bool lo0 = dup && (2 * t4 >= G) && (2 * t4 < 2 * G);
          const bool lo1 = dup && (2 * t4 + 1 >= G) && (2 * t4 + 1 < 2 * G);
          const uint32_t x_even = pack_f16x2(lo0 ? lo[0] : pr[0], lo0 ? lo[2] : pr[2]);  // col 2t4
          const uint32_t x_odd = pack_f16x2(lo1 ? lo[1] : pr[1], lo1 ? lo[3] : pr[3]);   // col 2t4+1
          const int srcA = (2 * t4) * 4 + (g8 >> 1);
          const int srcB = (2 * t4 + 1) * 4 + (g8 >> 1);
          const uint32_t ae = __shfl_sync(0xffffffffu, x_even, srcA);
          const uint32_t ao = __shfl_sync(0xffffffffu, x_odd, srcA);
          const uint32_t be = __shfl_sync(0xffffffffu, x_even, srcB);
          const uint32_t bo = __shfl_sync(0xffffffffu, x_odd, srcB);
          const uint32_t A = (g8 & 1) ? ao : ae;  // (P[2t4][g8], P[2t4+8][g8])
          const uint32_t Bv = (g8 & 1) ? bo : be; // (P[2t4+1][g8], P[2t4+9][g8])
          bp[0] = prmt(A, Bv, 0x5410);
          bp[1] = prmt(A, Bv, 0x7632);
          if (!dup) {
            const uint32_t le = pack_f16x2(lo[0], lo[2]), lodd = pack_f16x2(lo[1], lo[3]);
            const uint32_t lae = __shfl_sync(0xffffffffu, le, srcA);
            const uint32_t lao = __shfl_sync(0xffffffffu, lodd, srcA);
            const uint32_t lbe = __shfl_sync(0xffffffffu, le, srcB);
            const uint32_t lbo = __shfl_sync(0xffffffffu, lodd, srcB);
            const uint32_t LA = (g8 & 1) ? lao : lae;
            const uint32_t LB = (g8 & 1) ? lbo : lbe;
            bpl[0] = prmt(LA, LB, 0x5410);
            bpl[1] = prmt(LA, LB, 0x7632);
          } else {
            bpl[0] = bpl[1] = 0u;
          }
        }
        // ---------------- O^T += Vhat^T P
        {
          const int ta = 2 * t4, tb = 2 * t4 + 8;  // token pairs (ta, ta+1), (tb, tb+1)
          const int rows[4] = {tt * 16 + ta, tt * 16 + ta + 1, tt * 16 + tb, tt * 16 + tb + 1};
          bool vv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) vv[i] = ok && (tok0 + rows[i] - tt * 16 < L);
          uint32_t vw[4][S::VW];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < S::VW; ++j)
              vw[i][j] = ld_shared_u32(smem_u32(vpage + rows[i] * F + g8 * (D / 16) + 4 * j));
          constexpr int NGV = (D >= 128) ? D / 128 : 1;  // scale groups per lane
          uint32_t scA[NGV], scB[NGV];
#pragma unroll
          for (int gi = 0; gi < NGV; ++gi) {
            const int grp = (D == 64) ? (g8 >> 1) : g8 * NGV + gi;
            const uint32_t s0 = vv[0] ? vpage[rows[0] * F + D / 2 + grp] : 0u;
            const uint32_t s1 = vv[1] ? vpage[rows[1] * F + D / 2 + grp] : 0u;
            const uint32_t s2 = vv[2] ? vpage[rows[2] * F + D / 2 + grp] : 0u;
            const uint32_t s3 = vv[3] ? vpage[rows[3] * F + D / 2 + grp] : 0u;
            scA[gi] = e4m3x2_to_f16x2(s0 | (s1 << 8));
            scB[gi] = e4m3x2_to_f16x2(s2 | (s3 << 8));
          }
#pragma unroll
          for (int j = 0; j < S::VW; ++j) {
            const uint32_t a_lo = (vw[0][j] & 0x0F0F0F0Fu) | ((vw[1][j] & 0x0F0F0F0Fu) << 4);
            const uint32_t a_hi = ((vw[0][j] >> 4) & 0x0F0F0F0Fu) | (vw[1][j] & 0xF0F0F0F0u);
            const uint32_t b_lo = (vw[2][j] & 0x0F0F0F0Fu) | ((vw[3][j] & 0x0F0F0F0Fu) << 4);
            const uint32_t b_hi = ((vw[2][j] >> 4) & 0x0F0F0F0Fu) | (vw[3][j] & 0xF0F0F0F0u);
#pragma unroll
            for (int by = 0; by < 4; ++by) {
              const int m = 4 * j + by;  // PV chunk: rows d0 = g8*D/8 + 2m, d1 = d0 + 1
              const int gi = (D >= 128) ? m / 8 : 0;
              uint32_t af[4];
              af[0] = hmul2_u32(e2m1x2_to_f16x2((a_lo >> (8 * by)) & 0xFFu), scA[gi]);
              af[1] = hmul2_u32(e2m1x2_to_f16x2((a_hi >> (8 * by)) & 0xFFu), scA[gi]);
              af[2] = hmul2_u32(e2m1x2_to_f16x2((b_lo >> (8 * by)) & 0xFFu), scB[gi]);
              af[3] = hmul2_u32(e2m1x2_to_f16x2((b_hi >> (8 * by)) & 0xFFu), scB[gi]);
              mma_f16_16816(acc[m], af, bp);
              if (!dup) mma_f16_16816(acc[m], af, bpl);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !poisoned && k + kStages < nk) issue(k + kStages);
      ++k;
    }

    // ---- this warp's state for the portion -> shared memory
    const float l0 = warp_sum_g(l_run[0]), l1 = warp_sum_g(l_run[1]);
    if (g8 == 0) {
      st_m[w * 8 + 2 * t4] = m_run[0];
      st_m[w * 8 + 2 * t4 + 1] = m_run[1];
      st_l[w * 8 + 2 * t4] = l0;
      st_l[w * 8 + 2 * t4 + 1] = l1;
    }
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
      const int d0 = g8 * (D / 8) + 2 * m;
      float* base = st_acc + (size_t)w * 8 * D;
      base[(2 * t4) * D + d0] = acc[m][0];
      base[(2 * t4 + 1) * D + d0] = acc[m][1];
      base[(2 * t4) * D + d0 + 1] = acc[m][2];
      base[(2 * t4 + 1) * D + d0 + 1] = acc[m][3];
    }
    __syncthreads();

    const int i_first = cta_of(seg_start), i_last = cta_of(seg_end - 1);
    const bool whole = (i_first == i_last);
    const int slot = (s >= seg_start) ? 0 : 1;
    for (int idx = tid; idx < G * D; idx += kWarps * 32) {
      const int n = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int i = 0; i < kWarps; ++i) M = fmaxf(M, st_m[i * 8 + n]);
      const float Mu = (M == -INFINITY) ? 0.0f : M;
      float sum = 0.0f, lsum = 0.0f;
#pragma unroll
      for (int i = 0; i < kWarps; ++i) {
        const float sc = ex2(st_m[i * 8 + n] - Mu);
        const float* sa = st_acc + (size_t)i * 8 * D;
        sum += (dup ? sa[n * D + d] + sa[(n + G) * D + d] : sa[n * D + d]) * sc;
        lsum += st_l[i * 8 + n] * sc;
      }
      if (whole) {
        const float o = (lsum > 0.0f) ? __fdiv_rn(sum, lsum) * v_scale : 0.0f;
        write_output(a, ((long long)qt * a.num_q_heads + h * G + n) * D + d, o, o_scale);
      } else {
        const size_t ps = (size_t)cta * 2 + slot;
        partials[(ps * 8 + n) * D + d] = sum;
        if (d == 0) {
          part_ml[(ps * 8 + n) * 2 + 0] = M;
          part_ml[(ps * 8 + n) * 2 + 1] = lsum;
        }
      }
    }
    if (!whole) {
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const int ticket = atomicAdd(&counters[b * Hkv + h], 1);
        flag[0] = (ticket == i_last - i_first);
      }
      __syncthreads();
      if (flag[0]) {
        __threadfence();
        for (int idx = tid; idx < G * D; idx += kWarps * 32) {
          const int n = idx / D, d = idx % D;
          float M = -INFINITY;
          for (int i = i_first; i <= i_last; ++i) {
            const int si = (int)((long long)i * W / n_eff);
            const size_t ps = (size_t)i * 2 + ((si >= seg_start) ? 0 : 1);
            M = fmaxf(M, __ldcg(part_ml + (ps * 8 + n) * 2));
          }
          const float Mu = (M == -INFINITY) ? 0.0f : M;
          float sum = 0.0f, lsum = 0.0f;
          for (int i = i_first; i <= i_last; ++i) {
            const int si = (int)((long long)i * W / n_eff);
            const size_t ps = (size_t)i * 2 + ((si >= seg_start) ? 0 : 1);
            const float sc = ex2(__ldcg(part_ml + (ps * 8 + n) * 2) - Mu);
            sum += __ldcg(partials + (ps * 8 + n) * D + d) * sc;
            lsum += __ldcg(part_ml + (ps * 8 + n) * 2 + 1) * sc;
          }
          const float o = (lsum > 0.0f) ? __fdiv_rn(sum, lsum) * v_scale : 0.0f;
          write_output(a, ((long long)qt * a.num_q_heads + h * G + n) * D + d, o, o_scale);
        }
        if (tid == 0) counters[b * Hkv + h] = 0;
      }
    }
    __syncthreads();
    seg_f0 = pe;
  }
}

// Per-device launch facts, looked up once (outside any stream capture: the
// first call on a device should be an eager one).
struct DeviceFacts {
  int sms = 0;
  bool smem_attr_set = false;
};

template <int D, int BS>
static cudaError_t launch_decode_t(const AttentionArgs& a, cudaStream_t stream) {
  using S = DecodeShape<D, BS>;
  static DeviceFacts facts[64];
  const size_t smem = S::smem_bytes(a.num_seqs);
  auto kern = decode_attention_kernel<D, BS>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  DeviceFacts& f = facts[dev & 63];
  if (!f.smem_attr_set) {
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
  }
  int per_sm = 1;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarps * 32, smem);
  if (err != cudaSuccess) return err;
  int grid = f.sms * max(1, per_sm);
  if (grid > kDecodeCtas) grid = kDecodeCtas;
  kern<<<grid, kWarps * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

size_t decode_smem_bytes(int head_size, int block_size, int num_seqs) {
  if (head_size == 64 && block_size == 16) return DecodeShape<64, 16>::smem_bytes(num_seqs);
  if (head_size == 64 && block_size == 32) return DecodeShape<64, 32>::smem_bytes(num_seqs);
  if (head_size == 128 && block_size == 16) return DecodeShape<128, 16>::smem_bytes(num_seqs);
  if (head_size == 128 && block_size == 32) return DecodeShape<128, 32>::smem_bytes(num_seqs);
  if (head_size == 256 && block_size == 16) return DecodeShape<256, 16>::smem_bytes(num_seqs);
  if (head_size == 256 && block_size == 32) return DecodeShape<256, 32>::smem_bytes(num_seqs);
  return 0;
}

cudaError_t launch_decode_attention(const AttentionArgs& a, cudaStream_t stream) {
#define NVFP4_DECODE_CASE(DD, BB) \
  if (a.head_size == DD && a.block_size == BB) return launch_decode_t<DD, BB>(a, stream);
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
