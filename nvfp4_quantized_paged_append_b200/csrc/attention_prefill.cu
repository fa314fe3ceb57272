// Chunked-prefill attention over the NVFP4 paged cache.
//
// ("FlashInfer backend adds end-to-end NVFP4 KV cache support",
// implementation breakdown items 2-3: the prefill wrapper reads the NVFP4
// pages plus FP8 block scales and writes FP8 output.) Each sequence with
// q_len > 1 query tokens: query row r sits at position L - q_len + r and
// attends causally to keys 0..L-q_len+r of its paged cache.
//
// CTA = 4 warps x 16 rows; a row is one (query token, query head of the kv
// head's GQA group) pair, so the 64 rows of a CTA share one kv head and every
// page is read and dequantized once for all of them. Per page: one bulk async
// copy each for the K and V page (double-buffered on mbarriers), a
// cooperative dequant into f16 tiles in shared memory (exact: E2M1 * E4M3 has
// at most 6 significant bits), then mma.m16n8k16 for S = Q K^T and O += P V
// with fp32 accumulators and an exp2-domain online softmax.
#include <mutex>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

namespace {
constexpr int kPWarps = 4;
constexpr int kRows = kPWarps * 16;
constexpr float kPLog2e = 1.4426950408889634f;

template <int D, int BS>
struct PrefillShape {
  static constexpr int F = D / 2 + D / 16;
  static constexpr int PAGE = BS * F;
  static constexpr int LD = D + 8;  // f16 row stride of the smem tiles (bank spread)
  static size_t smem_bytes() {
    return 2ull * 2 * PAGE            // raw K,V pages, two stages
           + 2ull * kRows * LD        // Q tile (f16)
           + 2ull * 2 * BS * LD       // dequantized K and V tiles (f16)
           + 64;                      // mbarriers + scratch
  }
};
}  // namespace

template <int D, int BS>
__global__ void __launch_bounds__(kPWarps * 32) prefill_attention_kernel(const AttentionArgs a) {
  using S = PrefillShape<D, BS>;
  constexpr int F = S::F, PAGE = S::PAGE, LD = S::LD;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* raw = smem;                                              // [2][2][PAGE]
  __half* Qs = reinterpret_cast<__half*>(raw + 2 * 2 * PAGE);        // [kRows][LD]
  __half* Ks = Qs + kRows * LD;                                      // [BS][LD]
  __half* Vs = Ks + BS * LD;                                         // [BS][LD]
  uint64_t* bars = reinterpret_cast<uint64_t*>(Vs + BS * LD);        // [2]
  float* red = reinterpret_cast<float*>(bars + 2);                   // [4]
  int* okf = reinterpret_cast<int*>(red + 4);                        // [2]

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int b = blockIdx.z, h = blockIdx.y;
  const int Hkv = a.num_kv_heads, G = a.num_q_heads / Hkv;
  const int tpt = kRows / G;  // query tokens per CTA
  const int q_begin = a.qo_indptr[b];
  const int q_len = a.qo_indptr[b + 1] - q_begin;
  if (q_len <= 1) return;  // decode rows are served by the decode kernel
  if (q_len > (int)gridDim.x * tpt && blockIdx.x == 0 && threadIdx.x == 0)
    atomicOr(reinterpret_cast<uint32_t*>(a.workspace), kDevBadQlen);  // rows beyond the grid
  const int qtok0 = blockIdx.x * tpt;
  if (qtok0 >= q_len) return;
  const int L = a.seq_lens[b];
  const int last_tok = min(q_len - 1, qtok0 + tpt - 1);
  const int kv_end = min(L, max(0, L - q_len + last_tok + 1));  // keys [0, kv_end) are needed
  uint32_t* status = reinterpret_cast<uint32_t*>(a.workspace);
  const float k_scale = __ldg(a.kv_scales), v_scale = __ldg(a.kv_scales + 1);
  const float o_scale = __ldg(a.o_scale);

  // ---- Q tile -> shared (bf16 first), max |q|, then f16 with a power-of-two scale
  float mx = 0.0f;
  for (int c = tid; c < kRows * (D / 8); c += kPWarps * 32) {
    const int r = c / (D / 8), j = c % (D / 8);
    const int qt = qtok0 + r / G;
    uint4 v4 = make_uint4(0, 0, 0, 0);
    if (r < tpt * G && qt < q_len) {
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                 (long long)(q_begin + qt) * a.q_token_stride +
                                 (long long)(h * G + r % G) * D + 8 * j;
      v4 = __ldg(reinterpret_cast<const uint4*>(src));
    }
    const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(wv[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(wv[i] & 0xFFFF0000u)));
    }
    *reinterpret_cast<uint4*>(Qs + r * LD + 8 * j) = v4;
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[w] = mx;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const int ex = (mx > 0.0f) ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126 : 1;
  const int sh = min(126, max(-126, 15 - ex));
  const float qs = __uint_as_float((uint32_t)(sh + 127) << 23);
  const float qmult = a.sm_scale * k_scale * kPLog2e * __uint_as_float((uint32_t)(127 - sh) << 23);
  for (int c = tid; c < kRows * (D / 8); c += kPWarps * 32) {
    const int r = c / (D / 8), j = c % (D / 8);
    uint4* p = reinterpret_cast<uint4*>(Qs + r * LD + 8 * j);
    uint4 v4 = *p;
    uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      wv[i] = pack_f16x2(__uint_as_float(wv[i] << 16) * qs, __uint_as_float(wv[i] & 0xFFFF0000u) * qs);
    *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }

  const int npages = min(a.max_blocks_per_seq, (kv_end + BS - 1) / BS);
  auto issue = [&](int pg) {  // thread 0 only
    long long blk = __ldg(a.block_table + (long long)b * a.max_blocks_per_seq + pg);
    int ok = 1;
    if (blk < 0 || blk >= a.num_blocks) {
      atomicOr(status, kDevBadBlock);
      ok = 0;
      blk = 0;
    }
    const int st = pg & 1;
    okf[st] = ok;
    const uint8_t* kp = a.cache + ((blk * 2) * Hkv + h) * (long long)PAGE;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[st], 2 * PAGE);
    bulk_g2s(raw + st * 2 * PAGE, kp, PAGE, &bars[st]);
    bulk_g2s(raw + st * 2 * PAGE + PAGE, kp + (long long)Hkv * PAGE, PAGE, &bars[st]);
  };
  if (tid == 0 && npages > 0) issue(0);

  // rows of this lane: warp row base + g8 and + 8
  const int rA = w * 16 + g8, rB = rA + 8;
  const int posA = L - q_len + qtok0 + rA / G;  // absolute query positions
  const int posB = L - q_len + qtok0 + rB / G;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float acc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  bool poisoned = false;

  for (int pg = 0; pg < npages; ++pg) {
    const int st = pg & 1;
    if (tid == 0 && pg + 1 < npages && !poisoned) issue(pg + 1);
    bool ok = false;
    if (!poisoned) {
      if (mbar_wait_bounded(&bars[st], (uint32_t)((pg >> 1) & 1))) {
        ok = okf[st] != 0;
      } else {
        poisoned = true;
        if (tid == 0) atomicOr(status, kDevTimeout);
      }
    }
    // ---- dequant K and V pages into f16 tiles (masked rows -> 0)
    for (int c = tid; c < 2 * BS * (D / 8); c += kPWarps * 32) {
      const int kv = c / (BS * (D / 8));
      const int rem = c % (BS * (D / 8));
      const int r = rem / (D / 8), j = rem % (D / 8);
      const uint8_t* row = raw + st * 2 * PAGE + kv * PAGE + r * F;
      const bool valid = ok && (pg * BS + r < kv_end);
      const uint32_t codes = ld_shared_u32(smem_u32(row + 4 * j));
      const uint32_t sb = valid ? row[D / 2 + j / 2] : 0u;
      const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = hmul2_u32(e2m1x2_to_f16x2((codes >> (8 * i)) & 0xFFu), s2);
      __half* dst = (kv == 0 ? Ks : Vs) + r * LD + 8 * j;
      *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();

#pragma unroll
    for (int sub = 0; sub < BS / 16; ++sub) {
      const int key0 = pg * BS + sub * 16;
      // ---- S = Q K^T (16 rows x 16 keys)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t af[4], bf[4];
        const int ar = w * 16 + (lane & 15), acol = c * 16 + (lane >> 4) * 8;
        ldmatrix_x4(af, smem_u32(Qs + ar * LD + acol));
        // matrices: (keys 0-7, d lo), (keys 0-7, d hi), (keys 8-15, d lo), (keys 8-15, d hi)
        const int kr = sub * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int kc = c * 16 + ((lane >> 3) & 1) * 8;
        ldmatrix_x4(bf, smem_u32(Ks + kr * LD + kc));
        const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
        mma_f16_16816(sc[0], af, b0);
        mma_f16_16816(sc[1], af, b1);
      }
      // ---- mask + online softmax (rows rA: c0,c1; rB: c2,c3)
      float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int key = key0 + nt * 8 + 2 * t4 + e2;
          const bool kin = ok && key < kv_end;
          sc[nt][e2] = (kin && key <= posA) ? sc[nt][e2] * qmult : -INFINITY;
          sc[nt][2 + e2] = (kin && key <= posB) ? sc[nt][2 + e2] * qmult : -INFINITY;
          mxA = fmaxf(mxA, sc[nt][e2]);
          mxB = fmaxf(mxB, sc[nt][2 + e2]);
        }
      }
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
      const float mnA = fmaxf(m_run[0], mxA), mnB = fmaxf(m_run[1], mxB);
      const float muA = (mnA == -INFINITY) ? 0.f : mnA, muB = (mnB == -INFINITY) ? 0.f : mnB;
      const float alA = ex2(m_run[0] - muA), alB = ex2(m_run[1] - muB);
      m_run[0] = mnA;
      m_run[1] = mnB;
      float pA[4], pB[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        pA[2 * nt] = ex2(sc[nt][0] - muA);
        pA[2 * nt + 1] = ex2(sc[nt][1] - muA);
        pB[2 * nt] = ex2(sc[nt][2] - muB);
        pB[2 * nt + 1] = ex2(sc[nt][3] - muB);
      }
      l_run[0] = l_run[0] * alA + pA[0] + pA[1] + pA[2] + pA[3];
      l_run[1] = l_run[1] * alB + pB[0] + pB[1] + pB[2] + pB[3];
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        acc[j][0] *= alA;
        acc[j][1] *= alA;
        acc[j][2] *= alB;
        acc[j][3] *= alB;
      }
      // P as the A operand: (rA, k 2t4..), (rB, k 2t4..), (rA, k 2t4+8..), (rB, k 2t4+8..),
      // split into f16 hi + lo parts (hi = f16(p), lo = f16(p - hi)) so P keeps ~22 bits
      const uint32_t pa[4] = {pack_f16x2(pA[0], pA[1]), pack_f16x2(pB[0], pB[1]),
                              pack_f16x2(pA[2], pA[3]), pack_f16x2(pB[2], pB[3])};
      float lA[4], lB[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lA[i] = pA[i] - __half2float(__float2half_rn(pA[i]));
        lB[i] = pB[i] - __half2float(__float2half_rn(pB[i]));
      }
      const uint32_t pl[4] = {pack_f16x2(lA[0], lA[1]), pack_f16x2(lB[0], lB[1]),
                              pack_f16x2(lA[2], lA[3]), pack_f16x2(lB[2], lB[3])};
      // ---- O += P V
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        uint32_t bf[4];
        // matrices: (keys 0-7, d 16j..), (keys 8-15, d 16j..), (keys 0-7, d 16j+8..), (keys 8-15, d 16j+8..)
        const int vr = sub * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int vc = j * 16 + (lane >> 4) * 8;
        ldmatrix_x4_trans(bf, smem_u32(Vs + vr * LD + vc));
        const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
        mma_f16_16816(acc[2 * j], pa, b0);
        mma_f16_16816(acc[2 * j + 1], pa, b1);
        mma_f16_16816(acc[2 * j], pl, b0);
        mma_f16_16816(acc[2 * j + 1], pl, b1);
      }
    }
    __syncthreads();
  }

  // ---- epilogue: o = acc / l * v_scale -> fp32 / E4M3 / bf16
  float lA = l_run[0], lB = l_run[1];
  lA += __shfl_xor_sync(0xffffffffu, lA, 1);
  lA += __shfl_xor_sync(0xffffffffu, lA, 2);
  lB += __shfl_xor_sync(0xffffffffu, lB, 1);
  lB += __shfl_xor_sync(0xffffffffu, lB, 2);
  const int rows[2] = {rA, rB};
  const float ls[2] = {lA, lB};
#pragma unroll
  for (int ri = 0; ri < 2; ++ri) {
    const int r = rows[ri];
    const int qt = qtok0 + r / G;
    if (r >= tpt * G || qt >= q_len) continue;
    const long long obase = ((long long)(q_begin + qt) * a.num_q_heads + h * G + r % G) * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int d = j * 8 + 2 * t4 + e2;
        const float o = (ls[ri] > 0.f) ? __fdiv_rn(acc[j][2 * ri + e2], ls[ri]) * v_scale : 0.f;
        const long long idx = obase + d;
        if (a.o_f32) a.o_f32[idx] = o;
        const uint32_t code = f32_to_e4m3(__fdiv_rn(o, o_scale));
        a.o_fp8[idx] = (uint8_t)code;
        if (a.o_bf16)
          reinterpret_cast<__nv_bfloat16*>(a.o_bf16)[idx] =
              __float2bfloat16_rn(__fmul_rn(e4m3_to_f32(code), o_scale));
      }
    }
  }
}

template <int D, int BS>
static cudaError_t launch_prefill_t(const AttentionArgs& a, cudaStream_t stream) {
  using S = PrefillShape<D, BS>;
  const size_t smem = S::smem_bytes();
  auto kern = prefill_attention_kernel<D, BS>;
  // the attribute is set once per (device, context), under a lock
  static std::mutex attr_mutex;
  static unsigned long long attr_ctx[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  unsigned long long ctx = 0;
  err = current_context_id(&ctx);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(attr_mutex);
    if (ctx == 0 || attr_ctx[dev] != ctx) {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
      attr_ctx[dev] = ctx;
    }
  }
  const int G = a.num_q_heads / a.num_kv_heads;
  const int tpt = kRows / G;
  dim3 grid((a.max_q_len + tpt - 1) / tpt, a.num_kv_heads, a.num_seqs);
  kern<<<grid, kPWarps * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const AttentionArgs& a, cudaStream_t stream) {
#define NVFP4_PREFILL_CASE(DD, BB) \
  if (a.head_size == DD && a.block_size == BB) return launch_prefill_t<DD, BB>(a, stream);
  NVFP4_PREFILL_CASE(64, 16)
  NVFP4_PREFILL_CASE(64, 32)
  NVFP4_PREFILL_CASE(128, 16)
  NVFP4_PREFILL_CASE(128, 32)
  NVFP4_PREFILL_CASE(256, 16)
  NVFP4_PREFILL_CASE(256, 32)
#undef NVFP4_PREFILL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace nvfp4kv
