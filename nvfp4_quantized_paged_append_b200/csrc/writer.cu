// Slot-mapped NVFP4 quantize-append and paged dequantize kernels.
//
// Writer: "FlashInfer backend adds end-to-end NVFP4 KV cache support",
// key source snippets (_create_nvfp4_hnd_kv_cache: reshape_and_cache_flash
// with kv_cache_dtype "nvfp4", k_scale, v_scale and a slot mapping into the
// HND cache); row format from get_kv_cache_shape (full_dim = head_size/2 +
// head_size/16) and "Move NVFP4 GEMM management into NvFp4LinearKernel",
// base.py (FP4 pairs per byte, E4M3 scale per 16, global scale).
// Dequant: "FlashInfer NVFP4 KV serving on pre-SM100 GPUs", quick answer (the
// paged NVFP4 dequantize helper).
//
// Mapping: one CTA per token, one thread per 8 consecutive elements of a row
// (one 16-byte bf16 load, one 4-byte packed store); the two threads of a
// 16-element group meet with one shuffle for the block amax.
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

// E2M1 codes of fl32(x_i / S) for 8 values (element 2j in the low nibble of
// byte j). Fast path: y = x * rcp.approx(S) is within 2^-21 (relative) of
// x / S (the reciprocal is within 1 ulp, the product rounds by half an ulp),
// and so is fl32(x / S). If y * (1 - 2^-20) and y * (1 + 2^-20) give the same
// code, no rounding threshold of the E2M1 grid lies between them, and the
// conversion is monotone, so fl32(x / S) has that code as well. Otherwise
// (x / S within ~1e-6 of a threshold, exact ties included) the quotient is
// formed with IEEE division. S must be a positive normal number.
__device__ __forceinline__ uint32_t e2m1_codes_div(const float (&x)[8], float S) {
  float r;
  asm("rcp.approx.f32 %0, %1;\n" : "=f"(r) : "f"(S));
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float y = x[i] * r;
    lo[i] = y * 0.99999904632568359375f;  // 1 - 2^-20
    hi[i] = y * 1.00000095367431640625f;  // 1 + 2^-20
  }
  const uint32_t c_lo = f32x8_to_e2m1x8(lo);
  const uint32_t c_hi = f32x8_to_e2m1x8(hi);
  if (c_lo == c_hi) return c_lo;
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], S);
  return f32x8_to_e2m1x8(q);
}

// One CTA per new token: its K and V rows of every kv head, one thread per 8
// elements. A skipped (slot < 0) or out-of-range token exits as a whole.
template <int D>
__global__ void __launch_bounds__(256) quantize_append_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int num_kv_heads, uint8_t* __restrict__ cache,
    int64_t num_blocks, int bs_log2, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
    uint32_t* __restrict__ status) {
  constexpr int TPR = D / 8;  // threads per row
  constexpr int F = D / 2 + D / 16;
  // a kernel launched after this one as a programmatic dependent (attention)
  // may be scheduled now; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int64_t t = blockIdx.x;
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= (num_blocks << bs_log2)) {
    if (threadIdx.x == 0 && status) atomicOr(status, kDevBadSlot);
    return;
  }
  const int64_t blk = slot >> bs_log2;
  const int off = (int)(slot & ((1 << bs_log2) - 1));
  const int block_size = 1 << bs_log2;
  const int nthr = 2 * num_kv_heads * TPR;
  const int nthr_w = (nthr + 31) & ~31;  // whole warps iterate together (pair shuffles)
  for (int idx = threadIdx.x; idx < nthr_w; idx += blockDim.x) {
    const bool act = idx < nthr;
    const int rr = idx / TPR, j = idx % TPR;
    const int kv = rr >= num_kv_heads ? 1 : 0;
    const int h = rr - kv * num_kv_heads;
    float x[8];
    if (act) {
      const __nv_bfloat16* src = (kv == 0 ? k + t * k_stride : v + t * v_stride) + h * D + j * 8;
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.0f;
    }
    // block amax over the 16 elements held by this thread and its partner
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    if (!act) continue;

    const float g = __ldg(kv == 0 ? k_scale : v_scale);
    const float s32 = __fdiv_rn(amax, __fmul_rn(6.0f, g));
    const uint32_t sb = f32_to_e4m3(s32);
    const float S = __fmul_rn(e4m3_to_f32(sb), g);
    uint32_t packed = 0u;  // S == 0: every code 0
    if (S >= 1.17549435e-38f) {
      packed = e2m1_codes_div(x, S);
    } else if (S > 0.0f) {  // subnormal effective scale: divide exactly
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], S);
      packed = f32x8_to_e2m1x8(q);
    }
    uint8_t* dst =
        cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * F;
    *reinterpret_cast<uint32_t*>(dst + 4 * j) = packed;
    if ((j & 1) == 0) dst[D / 2 + j / 2] = (uint8_t)sb;
  }
}

template <int D>
__global__ void __launch_bounds__(256) dequantize_paged_kernel(
    const uint8_t* __restrict__ cache, int64_t num_blocks, int block_size, int num_kv_heads,
    const int32_t* __restrict__ block_ids, int64_t num_ids, const float* __restrict__ kv_scales,
    __nv_bfloat16* __restrict__ out) {
  constexpr int TPR = D / 8;
  constexpr int F = D / 2 + D / 16;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gtid / TPR;  // row index in out: [id][kv][h][off]
  const int j = (int)(gtid % TPR);
  const int64_t rows_per_id = 2LL * num_kv_heads * block_size;
  if (row >= num_ids * rows_per_id) return;
  const int64_t id = row / rows_per_id;
  const int64_t in_id = row % rows_per_id;  // (kv, h, off) flattened
  const int kv = (int)(in_id / ((int64_t)num_kv_heads * block_size));
  const int64_t blk = __ldg(block_ids + id);
  if (blk < 0 || blk >= num_blocks) return;
  const uint8_t* src = cache + (blk * rows_per_id + in_id) * F;
  const uint32_t codes = *reinterpret_cast<const uint32_t*>(src + 4 * j);
  const uint32_t sb = src[D / 2 + j / 2];
  const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
  const float g = __ldg(kv_scales + kv);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h2 = hmul2_u32(e2m1x2_to_f16x2((codes >> (8 * i)) & 0xFFu), s2);  // exact
    const float lo = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF))), g);
    const float hi = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 >> 16))), g);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
    o[i] = *reinterpret_cast<uint32_t*>(&b2);
  }
  *reinterpret_cast<uint4*>(out + row * D + 8 * j) = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_quantize_append(const QuantizeAppendArgs& a, cudaStream_t stream) {
  const int bs_log2 = (a.block_size == 16) ? 4 : 5;  // validated: 16 or 32
  const int block = 256;
  if (a.num_tokens > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)a.num_tokens;
  const auto* k = static_cast<const __nv_bfloat16*>(a.k);
  const auto* v = static_cast<const __nv_bfloat16*>(a.v);
#define NVFP4_WRITER_CASE(DD)                                                                  \
  case DD:                                                                                     \
    quantize_append_kernel<DD><<<grid, block, 0, stream>>>(                                    \
        k, v, a.k_token_stride, a.v_token_stride, a.num_kv_heads, a.cache, a.num_blocks,       \
        bs_log2, a.slot_mapping, a.k_scale, a.v_scale, a.device_status);                       \
    break;
  switch (a.head_size) {
    NVFP4_WRITER_CASE(64)
    NVFP4_WRITER_CASE(128)
    NVFP4_WRITER_CASE(256)
    default:
      return cudaErrorInvalidValue;
  }
#undef NVFP4_WRITER_CASE
  return cudaGetLastError();
}

cudaError_t launch_dequantize_paged(const DequantArgs& a, cudaStream_t stream) {
  const int64_t threads = a.num_block_ids * 2 * a.num_kv_heads * a.block_size * (a.head_size / 8);
  const int block = 256;
  const int64_t grid = (threads + block - 1) / block;
  auto* out = static_cast<__nv_bfloat16*>(a.out_bf16);
#define NVFP4_DEQ_CASE(DD)                                                                  \
  case DD:                                                                                  \
    dequantize_paged_kernel<DD><<<(unsigned)grid, block, 0, stream>>>(                      \
        a.cache, a.num_blocks, a.block_size, a.num_kv_heads, a.block_ids, a.num_block_ids, \
        a.kv_scales, out);                                                                  \
    break;
  switch (a.head_size) {
    NVFP4_DEQ_CASE(64)
    NVFP4_DEQ_CASE(128)
    NVFP4_DEQ_CASE(256)
    default:
      return cudaErrorInvalidValue;
  }
#undef NVFP4_DEQ_CASE
  return cudaGetLastError();
}

}  // namespace nvfp4kv
