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
// Mapping: one thread per 8 consecutive elements of a row (one 16-byte bf16
// load, one 4-byte packed store); the two threads of a 16-element group meet
// with one shuffle for the block amax. Rows are ordered token-major, then K/V,
// then head, so a warp streams contiguous bf16 memory.
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

template <int D>
__global__ void __launch_bounds__(256) quantize_append_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int64_t num_tokens, int num_kv_heads,
    uint8_t* __restrict__ cache, int64_t num_blocks, int block_size,
    const int64_t* __restrict__ slot_mapping, const float* __restrict__ k_scale,
    const float* __restrict__ v_scale, uint32_t* __restrict__ status) {
  constexpr int TPR = D / 8;  // threads per row
  constexpr int F = D / 2 + D / 16;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gtid / TPR;
  const int j = (int)(gtid % TPR);  // this thread's 8-element chunk
  const int64_t rows = num_tokens * 2 * num_kv_heads;
  const bool in_range = row < rows;

  int64_t t = 0;
  int kv = 0, h = 0;
  int64_t slot = -1;
  if (in_range) {
    t = row / (2 * num_kv_heads);
    const int rem = (int)(row % (2 * num_kv_heads));
    kv = rem / num_kv_heads;
    h = rem % num_kv_heads;
    slot = __ldg(slot_mapping + t);
  }

  float x[8];
  if (in_range) {
    const __nv_bfloat16* src =
        (kv == 0 ? k + t * k_stride : v + t * v_stride) + (int64_t)h * D + j * 8;
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

  const float g = in_range ? __ldg(kv == 0 ? k_scale : v_scale) : 1.0f;
  const float s32 = __fdiv_rn(amax, __fmul_rn(6.0f, g));
  const uint32_t sb = f32_to_e4m3(s32);
  const float S = __fmul_rn(e4m3_to_f32(sb), g);

  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = (S == 0.0f) ? 0.0f : __fdiv_rn(x[i], S);
  const uint32_t packed = f32x8_to_e2m1x8(q);

  if (!in_range || slot < 0) return;
  if (slot >= num_blocks * (int64_t)block_size) {
    if (j == 0 && kv == 0 && h == 0 && status) atomicOr(status, kDevBadSlot);
    return;
  }
  const int64_t blk = slot / block_size;
  const int off = (int)(slot % block_size);
  uint8_t* dst = cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * F;
  *reinterpret_cast<uint32_t*>(dst + 4 * j) = packed;
  if ((j & 1) == 0) dst[D / 2 + j / 2] = (uint8_t)sb;
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
  const int64_t threads = a.num_tokens * 2 * a.num_kv_heads * (a.head_size / 8);
  const int block = 256;
  const int64_t grid = (threads + block - 1) / block;
  const auto* k = static_cast<const __nv_bfloat16*>(a.k);
  const auto* v = static_cast<const __nv_bfloat16*>(a.v);
#define NVFP4_WRITER_CASE(DD)                                                                \
  case DD:                                                                                   \
    quantize_append_kernel<DD><<<(unsigned)grid, block, 0, stream>>>(                        \
        k, v, a.k_token_stride, a.v_token_stride, a.num_tokens, a.num_kv_heads, a.cache,     \
        a.num_blocks, a.block_size, a.slot_mapping, a.k_scale, a.v_scale, a.device_status); \
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
