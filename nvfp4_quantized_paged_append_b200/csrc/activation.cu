// Activation NVFP4 quantizer with the block-scaled GEMM's scale layout.
//
// "Move NVFP4 GEMM management into NvFp4LinearKernel", flashinfer.py and the
// CUTLASS linear kernel: scaled_fp4_quant(x, input_global_scale_inv,
// is_sf_swizzled_layout=True) produces packed E2M1 pairs and one E4M3 scale per
// 16 values, laid out by swizzle_blockscale for the block-scaled GEMM. The
// group codec is the KV cache's (quantize_group16) with g = fl32(1 / inv).
//
// Scale layout (swizzled): rows padded to 128 and scale columns to 4, 512-byte
// tiles of 128 rows x 4 scale columns in row-band-major order; inside a tile,
// scale (r, c) at (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4. Padding
// entries are written as 0 by the kernel itself.
//
// Mapping: block (x = row, y = 256-group slice of the row), one thread per
// 16-element group (two 16-byte loads, 8 bytes of codes, one scale byte); a
// warp reads 1 KB and writes 256 contiguous bytes of codes.
#include "nvfp4kv_device.cuh"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {

template <bool SWZ>
__global__ void __launch_bounds__(256) quantize_activation_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t row_stride,
    const float* __restrict__ inv, uint8_t* __restrict__ fp4, uint8_t* __restrict__ sf) {
  const int64_t r = blockIdx.x;
  const int64_t c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;  // 16-element group
  const int64_t c16 = cols / 16;
  const int64_t pc = SWZ ? (c16 + 3) / 4 * 4 : c16;
  if (c >= pc) return;
  int64_t at = r * c16 + c;
  if constexpr (SWZ)
    at = ((r >> 7) * (pc >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
  if (r >= rows || c >= c16) {  // padding of the swizzled layout
    sf[at] = 0;
    return;
  }
  const __nv_bfloat16* src = x + r * row_stride + c * 16;
  const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(src));
  const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
  const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(wv[i] << 16);
    v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
  }
  const float g = __fdiv_rn(1.0f, __ldg(inv));
  uint32_t c0, c1;
  const uint32_t sb = quantize_group16(v, g, c0, c1);
  *reinterpret_cast<uint2*>(fp4 + r * (cols / 2) + c * 8) = make_uint2(c0, c1);
  sf[at] = (uint8_t)sb;
}

cudaError_t launch_quantize_activation(const ActivationArgs& a, cudaStream_t stream) {
  const int64_t c16 = a.cols / 16;
  const int64_t pc = a.swizzled ? (c16 + 3) / 4 * 4 : c16;
  const int64_t pr = a.swizzled ? (a.rows + 127) / 128 * 128 : a.rows;
  const int64_t gy = (pc + 255) / 256;
  if (pr > 0x7FFFFFFFLL || gy > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)pr, (unsigned)gy);
  const auto* x = static_cast<const __nv_bfloat16*>(a.x);
  if (a.swizzled)
    quantize_activation_kernel<true><<<grid, 256, 0, stream>>>(x, a.rows, a.cols, a.row_stride,
                                                               a.global_scale_inv, a.out_fp4,
                                                               a.out_sf);
  else
    quantize_activation_kernel<false><<<grid, 256, 0, stream>>>(x, a.rows, a.cols, a.row_stride,
                                                                a.global_scale_inv, a.out_fp4,
                                                                a.out_sf);
  return cudaGetLastError();
}

}  // namespace nvfp4kv
