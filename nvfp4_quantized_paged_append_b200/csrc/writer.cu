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
// Mapping: grid-stride blocks over tokens, one thread per two adjacent
// 16-element blocks of a row (NVFP4 rows of head size 128 or 256 when the
// token's row groups come in multiples of 64), else one thread per 16-element
// block; one CTA per token when a token has more groups than a block holds.
#include <algorithm>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

// One CTA per new token: its K and V rows of every kv head, one thread per
// 16-element block (two 16-byte bf16 loads, one scale, 8 bytes of codes). A
// skipped (slot < 0) or out-of-range token exits as a whole.
template <int D>
__global__ void __launch_bounds__(256) quantize_append_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int num_kv_heads, uint8_t* __restrict__ cache,
    int64_t num_blocks, int bs_log2, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
    uint32_t* __restrict__ status) {
  constexpr int TPR = D / 16;  // threads per row
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
  const float gk = __ldg(k_scale), gv = __ldg(v_scale);
  const int nthr = 2 * num_kv_heads * TPR;
  for (int idx = threadIdx.x; idx < nthr; idx += blockDim.x) {
    const int rr = idx / TPR, j = idx % TPR;
    const int kv = rr >= num_kv_heads ? 1 : 0;
    const int h = rr - kv * num_kv_heads;
    const __nv_bfloat16* src = (kv == 0 ? k + t * k_stride : v + t * v_stride) + h * D + j * 16;
    const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float x[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = __uint_as_float(wv[i] << 16);
      x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
    const float g = kv == 0 ? gk : gv;
    uint32_t c0, c1;
    const uint32_t sb = quantize_group16(x, g, c0, c1);
    uint8_t* dst =
        cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * F;
    if constexpr (F % 8 == 0) {  // rows 8-byte aligned
      *reinterpret_cast<uint2*>(dst + 8 * j) = make_uint2(c0, c1);
    } else {
      reinterpret_cast<uint32_t*>(dst + 8 * j)[0] = c0;
      reinterpret_cast<uint32_t*>(dst + 8 * j)[1] = c1;
    }
    dst[D / 2 + j] = (uint8_t)sb;
  }
}

// Grid-stride writer: thread `idx` of a block owns group idx % TPR of row
// idx / TPR (K rows first, then V rows) of every token the block visits
// (blockDim.x == 2 * num_kv_heads * D / 16). The next token's slot and input
// words are loaded before the current token is quantized, so the two memory
// latencies of a token (its slot, then its rows) overlap with other work.
// FP8 = false: NVFP4 rows; true: FP8-E4M3 rows.
template <int D, bool FP8>
__global__ void __launch_bounds__(1024) quantize_append_stream_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int num_kv_heads, uint8_t* __restrict__ cache,
    int64_t num_tokens, int64_t num_blocks, int bs_log2, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
    uint32_t* __restrict__ status) {
  constexpr int TPR = D / 16;
  constexpr int F = FP8 ? D : D / 2 + D / 16;
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int idx = threadIdx.x;
  const int rr = idx / TPR, j = idx % TPR;
  const int kv = rr >= num_kv_heads ? 1 : 0;
  const int h = rr - kv * num_kv_heads;
  const __nv_bfloat16* src0 = (kv == 0 ? k : v) + h * D + j * 16;
  const int64_t stride = kv == 0 ? k_stride : v_stride;
  const float g = __ldg(kv == 0 ? k_scale : v_scale);
  const int block_size = 1 << bs_log2;
  int64_t t = blockIdx.x;
  int64_t slot = -1;
  uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0;
  if (t < num_tokens) {
    slot = __ldg(slot_mapping + t);
    r0 = __ldg(reinterpret_cast<const uint4*>(src0 + t * stride));
    r1 = __ldg(reinterpret_cast<const uint4*>(src0 + t * stride) + 1);
  }
  while (t < num_tokens) {
    const int64_t tn = t + gridDim.x;
    int64_t slot_n = -1;
    uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
    if (tn < num_tokens) {  // rows exist for every token: loaded before the slot is known
      slot_n = __ldg(slot_mapping + tn);
      n0 = __ldg(reinterpret_cast<const uint4*>(src0 + tn * stride));
      n1 = __ldg(reinterpret_cast<const uint4*>(src0 + tn * stride) + 1);
    }
    if (slot >= (num_blocks << bs_log2)) {
      if (idx == 0 && status) atomicOr(status, kDevBadSlot);
    } else if (slot >= 0) {
      const int64_t blk = slot >> bs_log2;
      const int off = (int)(slot & (block_size - 1));
      uint8_t* dst =
          cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * F;
      const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      if constexpr (FP8) {
        uint32_t out[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t b0 = e4m3_of_quotient(__uint_as_float(wv[2 * i] << 16), g);
          const uint32_t b1 = e4m3_of_quotient(__uint_as_float(wv[2 * i] & 0xFFFF0000u), g);
          const uint32_t b2 = e4m3_of_quotient(__uint_as_float(wv[2 * i + 1] << 16), g);
          const uint32_t b3 = e4m3_of_quotient(__uint_as_float(wv[2 * i + 1] & 0xFFFF0000u), g);
          out[i] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
        *reinterpret_cast<uint4*>(dst + 16 * j) = make_uint4(out[0], out[1], out[2], out[3]);
      } else {
        float x[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[2 * i] = __uint_as_float(wv[i] << 16);
          x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
        }
        uint32_t c0, c1;
        const uint32_t sb = quantize_group16(x, g, c0, c1);
        if constexpr (F % 8 == 0) {
          *reinterpret_cast<uint2*>(dst + 8 * j) = make_uint2(c0, c1);
        } else {
          reinterpret_cast<uint32_t*>(dst + 8 * j)[0] = c0;
          reinterpret_cast<uint32_t*>(dst + 8 * j)[1] = c1;
        }
        dst[D / 2 + j] = (uint8_t)sb;
      }
    }
    t = tn;
    slot = slot_n;
    r0 = n0;
    r1 = n1;
  }
}

// Grid-stride NVFP4 writer with two adjacent 16-element groups of a row per
// thread (blockDim.x == num_kv_heads * D / 16; D = 128 or 256, whose rows
// start on 8-byte boundaries): four 16-byte bf16 loads, 16
// bytes of packed codes and a 2-byte pair of scales per token, so the token's
// slot, address and loop work is shared by two groups. Same slot rules and
// next-token prefetch as quantize_append_stream_kernel.
template <int D>
__global__ void __launch_bounds__(512) quantize_append_pair_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int num_kv_heads, uint8_t* __restrict__ cache,
    int64_t num_tokens, int64_t num_blocks, int bs_log2, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
    uint32_t* __restrict__ status) {
  constexpr int TPR = D / 32;  // threads per row
  constexpr int F = D / 2 + D / 16;
  static_assert(F % 8 == 0, "rows must be 8-byte aligned (head size 128 or 256)");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int idx = threadIdx.x;
  const int rr = idx / TPR, j = idx % TPR;
  const int kv = rr >= num_kv_heads ? 1 : 0;
  const int h = rr - kv * num_kv_heads;
  const __nv_bfloat16* src0 = (kv == 0 ? k : v) + h * D + j * 32;
  const int64_t stride = kv == 0 ? k_stride : v_stride;
  const float g = __ldg(kv == 0 ? k_scale : v_scale);
  const int block_size = 1 << bs_log2;
  int64_t t = blockIdx.x;
  int64_t slot = -1;
  uint4 r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = make_uint4(0u, 0u, 0u, 0u);
  if (t < num_tokens) {
    slot = __ldg(slot_mapping + t);
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = __ldg(reinterpret_cast<const uint4*>(src0 + t * stride) + i);
  }
  while (t < num_tokens) {
    const int64_t tn = t + gridDim.x;
    int64_t slot_n = -1;
    uint4 n[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) n[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tn < num_tokens) {
      slot_n = __ldg(slot_mapping + tn);
#pragma unroll
      for (int i = 0; i < 4; ++i) n[i] = __ldg(reinterpret_cast<const uint4*>(src0 + tn * stride) + i);
    }
    if (slot >= (num_blocks << bs_log2)) {
      if (idx == 0 && status) atomicOr(status, kDevBadSlot);
    } else if (slot >= 0) {
      const int64_t blk = slot >> bs_log2;
      const int off = (int)(slot & (block_size - 1));
      uint8_t* dst =
          cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * F;
      uint32_t cw[4], sbv[2];
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const uint32_t wv[8] = {r[2 * gi].x,     r[2 * gi].y,     r[2 * gi].z,     r[2 * gi].w,
                                r[2 * gi + 1].x, r[2 * gi + 1].y, r[2 * gi + 1].z, r[2 * gi + 1].w};
        float x[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[2 * i] = __uint_as_float(wv[i] << 16);
          x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
        }
        sbv[gi] = quantize_group16(x, g, cw[2 * gi], cw[2 * gi + 1]);
      }
      if constexpr (F % 16 == 0) {
        *reinterpret_cast<uint4*>(dst + 16 * j) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      } else {  // rows 8-byte aligned
        reinterpret_cast<uint2*>(dst + 16 * j)[0] = make_uint2(cw[0], cw[1]);
        reinterpret_cast<uint2*>(dst + 16 * j)[1] = make_uint2(cw[2], cw[3]);
      }
      // D / 2 + 2 j and F are even: the scale pair is 2-byte aligned
      *reinterpret_cast<uint16_t*>(dst + D / 2 + 2 * j) = (uint16_t)(sbv[0] | (sbv[1] << 8));
    }
    t = tn;
    slot = slot_n;
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = n[i];
  }
}

// FP8-E4M3 rows (the comparison format): code = E4M3 RNE satfinite of
// fl32(x / g) per element (same bracketed reciprocal fast path, IEEE division
// near rounding thresholds), D bytes per row in the same HND page layout.
template <int D>
__global__ void __launch_bounds__(256) quantize_append_fp8_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int64_t k_stride, int64_t v_stride, int num_kv_heads, uint8_t* __restrict__ cache,
    int64_t num_blocks, int bs_log2, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
    uint32_t* __restrict__ status) {
  constexpr int TPR = D / 16;
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
  const float gk = __ldg(k_scale), gv = __ldg(v_scale);
  const int nthr = 2 * num_kv_heads * TPR;
  for (int idx = threadIdx.x; idx < nthr; idx += blockDim.x) {
    const int rr = idx / TPR, j = idx % TPR;
    const int kv = rr >= num_kv_heads ? 1 : 0;
    const int h = rr - kv * num_kv_heads;
    const __nv_bfloat16* src = (kv == 0 ? k + t * k_stride : v + t * v_stride) + h * D + j * 16;
    const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    const float g = kv == 0 ? gk : gv;
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t b0 = e4m3_of_quotient(__uint_as_float(wv[2 * i] << 16), g);
      const uint32_t b1 = e4m3_of_quotient(__uint_as_float(wv[2 * i] & 0xFFFF0000u), g);
      const uint32_t b2 = e4m3_of_quotient(__uint_as_float(wv[2 * i + 1] << 16), g);
      const uint32_t b3 = e4m3_of_quotient(__uint_as_float(wv[2 * i + 1] & 0xFFFF0000u), g);
      out[i] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
    uint8_t* dst = cache + (((blk * 2 + kv) * num_kv_heads + h) * (int64_t)block_size + off) * D;
    *reinterpret_cast<uint4*>(dst + 16 * j) = make_uint4(out[0], out[1], out[2], out[3]);
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
  // one thread per 16-element block of the token's 2 * num_kv_heads rows
  const int rows_threads = 2 * a.num_kv_heads * (a.head_size / 16);
  const auto* k = static_cast<const __nv_bfloat16*>(a.k);
  const auto* v = static_cast<const __nv_bfloat16*>(a.v);
  int dev = 0, sms = 0;
  if (rows_threads % 32 == 0 && rows_threads <= 1024) {
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
  }
  if (!a.kv_format && a.head_size >= 128 && rows_threads % 64 == 0 && rows_threads <= 1024) {
    // NVFP4 rows of 8-byte aligned length, two groups per thread: grid-stride
    // blocks, as many as are resident at once
    const int threads = rows_threads / 2;
    cudaError_t err = cudaSuccess;
#define NVFP4_PAIR_CASE(DD)                                                                    \
  case DD: {                                                                                   \
    auto kern = quantize_append_pair_kernel<DD>;                                               \
    int per_sm = 1;                                                                            \
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);            \
    if (err != cudaSuccess) return err;                                                        \
    const long long resident = (long long)sms * std::max(1, per_sm);                           \
    const unsigned grid = (unsigned)std::min<long long>(a.num_tokens, resident);               \
    kern<<<grid, threads, 0, stream>>>(k, v, a.k_token_stride, a.v_token_stride,               \
                                       a.num_kv_heads, a.cache, a.num_tokens, a.num_blocks,    \
                                       bs_log2, a.slot_mapping, a.k_scale, a.v_scale,          \
                                       a.device_status);                                       \
    break;                                                                                     \
  }
    switch (a.head_size) {
      NVFP4_PAIR_CASE(128)
      NVFP4_PAIR_CASE(256)
      default:
        return cudaErrorInvalidValue;
    }
#undef NVFP4_PAIR_CASE
    return cudaGetLastError();
  }
  if (rows_threads % 32 == 0 && rows_threads <= 1024) {
    // grid-stride blocks, as many as are resident at once (tokens per block
    // rise with the batch)
    cudaError_t err = cudaSuccess;
#define NVFP4_STREAM_CASE(DD)                                                                  \
  case DD: {                                                                                   \
    auto kern = a.kv_format ? quantize_append_stream_kernel<DD, true>                          \
                            : quantize_append_stream_kernel<DD, false>;                        \
    int per_sm = 1;                                                                            \
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, rows_threads, 0);       \
    if (err != cudaSuccess) return err;                                                        \
    const long long resident = (long long)sms * std::max(1, per_sm);                           \
    const unsigned grid = (unsigned)std::min<long long>(a.num_tokens, resident);               \
    kern<<<grid, rows_threads, 0, stream>>>(k, v, a.k_token_stride, a.v_token_stride,          \
                                            a.num_kv_heads, a.cache, a.num_tokens,             \
                                            a.num_blocks, bs_log2, a.slot_mapping, a.k_scale,  \
                                            a.v_scale, a.device_status);                       \
    break;                                                                                     \
  }
    switch (a.head_size) {
      NVFP4_STREAM_CASE(64)
      NVFP4_STREAM_CASE(128)
      NVFP4_STREAM_CASE(256)
      default:
        return cudaErrorInvalidValue;
    }
#undef NVFP4_STREAM_CASE
    return cudaGetLastError();
  }
  // many heads: one block per token, threads loop over the token's groups
  const int block = rows_threads <= 128 ? 128 : 256;
  if (a.num_tokens > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)a.num_tokens;
#define NVFP4_WRITER_CASE(DD)                                                                  \
  case DD:                                                                                     \
    if (a.kv_format)                                                                           \
      quantize_append_fp8_kernel<DD><<<grid, block, 0, stream>>>(                              \
          k, v, a.k_token_stride, a.v_token_stride, a.num_kv_heads, a.cache, a.num_blocks,     \
          bs_log2, a.slot_mapping, a.k_scale, a.v_scale, a.device_status);                     \
    else                                                                                       \
      quantize_append_kernel<DD><<<grid, block, 0, stream>>>(                                  \
          k, v, a.k_token_stride, a.v_token_stride, a.num_kv_heads, a.cache, a.num_blocks,     \
          bs_log2, a.slot_mapping, a.k_scale, a.v_scale, a.device_status);                     \
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

// Bounded-wait check: the barrier expects 16 bytes that no copy delivers, so
// the wait must give up after `polls` polls and report kDevTimeout. No copy is
// ever issued, so nothing is in flight when the block exits.
__global__ void wait_timeout_probe_kernel(uint32_t* status, int polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_arrive_expect_tx(&bar, 16);
  if (!mbar_wait_bounded(&bar, 0u, polls)) atomicOr(status, kDevTimeout);
}

cudaError_t launch_wait_timeout_probe(uint32_t* status, int polls, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status, polls);
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
