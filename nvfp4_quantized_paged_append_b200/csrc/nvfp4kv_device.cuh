// Device-side building blocks for the NVFP4 paged KV cache kernels (sm_100a).
//
// Format conversions use the Blackwell PTX conversion instructions:
//   cvt.rn.satfinite.e2m1x2.f32   two fp32 -> two E2M1 nibbles (RNE, saturating)
//   cvt.rn.satfinite.e4m3x2.f32   two fp32 -> two E4M3 bytes (RNE, saturating)
//   cvt.rn.f16x2.e2m1x2           two E2M1 nibbles -> two f16 (exact)
//   cvt.rn.f16x2.e4m3x2           two E4M3 bytes -> two f16 (exact)
// Page movement uses the bulk async copy (cp.async.bulk) completed on an
// mbarrier; every wait on an mbarrier is bounded and reports a timeout.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace nvfp4kv {

constexpr uint32_t kDevBadSlot = 0x1u;
constexpr uint32_t kDevBadBlock = 0x2u;
constexpr uint32_t kDevTimeout = 0x4u;
constexpr uint32_t kDevBadQlen = 0x8u;
constexpr uint32_t kAttnMetadataReady = 0x1u;  // NVFP4_ATTN_METADATA_READY
constexpr uint32_t kAttnHistoryReady = 0x2u;   // NVFP4_ATTN_HISTORY_READY
constexpr uint32_t kAttnQfp4 = 0x4u;           // NVFP4_ATTN_QFP4

// Wait until the grids this one depends on (programmatic dependent launch)
// have completed and their writes are visible; returns at once otherwise.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// ~ seconds of polling before a wait gives up (each try_wait suspends briefly).
constexpr int kMaxWaitIters = 1 << 24;

// ------------------------------------------------------------ conversions
// (pure register-to-register asm, not volatile: the compiler may schedule
// and combine it like ordinary arithmetic)
// Pack 8 fp32 values into 8 E2M1 nibbles: x[2j] -> low nibble of byte j.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float x[8]) {
  uint32_t out;
  asm(
      "{\n"
      ".reg .b8 q0, q1, q2, q3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n"
      "mov.b32 %0, {q0, q1, q2, q3};\n"
      "}\n"
      : "=r"(out)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]),
        "f"(x[7]));
  return out;
}

// fp32 -> E4M3 byte (RNE, satfinite), returned in the low 8 bits.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// two fp32 -> two E4M3 bytes: lo in bits 0..7, hi in bits 8..15.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// E4M3 byte pair (lo in bits 0..7) -> f16x2 (lo half = lo byte); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t out;
  uint16_t in = (uint16_t)two_bytes;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(out) : "h"(in));
  return out;
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

// E2M1 pair in one byte (low nibble -> lo half) -> f16x2; exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm(
      "{\n"
      ".reg .b8 b;\n"
      "cvt.u8.u32 b, %1;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n"
      "}\n"
      : "=r"(out)
      : "r"(byte));
  return out;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2 = e4m3x2_to_f16x2(byte & 0xFFu);
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// ------------------------------------------------------------ NVFP4 encode
// Packed fp32 pairs (Blackwell mul.rn.f32x2: two correctly rounded fp32
// products per instruction; the low half is the first element).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t d, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(lo), "=f"(hi) : "l"(d));
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max(a, b, c) in one instruction; a NaN operand is ignored like fmaxf's.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The bracket around an approximate quotient: 1 -+ 2^-20.
constexpr float kBracketLo = 0.99999904632568359375f;
constexpr float kBracketHi = 1.00000095367431640625f;

// E2M1 codes of fl32(x_i / S) for 8 values (element 2j in the low nibble of
// byte j). Fast path: with r = rcp.approx(S) (within 1 ulp of 1/S) and
// r_lo = fl32(r (1 - 2^-20)), r_hi = fl32(r (1 + 2^-20)), the products
// fl32(x r_lo) and fl32(x r_hi) lie strictly on either side of fl32(x / S)
// (the errors of the reciprocal and the two roundings add up to less than
// 2^-21, while the bracket is 2^-20 wide on each side). If both ends give the
// same code, no rounding threshold of the E2M1 grid lies between them, and
// the conversion is monotone, so fl32(x / S) has that code as well.
// Otherwise (x / S within ~1e-6 of a threshold, exact ties included) the
// quotient is formed with IEEE division. S must be a positive normal number;
// above 2^100 the reciprocal nears the subnormal range, where its 1-ulp bound
// no longer holds, so such scales always divide.
__device__ __forceinline__ uint32_t e2m1_codes_div(const float (&x)[8], float S) {
  if (S > 1.2676506e30f) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], S);
    return f32x8_to_e2m1x8(q);
  }
  float r;
  asm("rcp.approx.f32 %0, %1;\n" : "=f"(r) : "f"(S));
  const uint64_t rr = pack_f32x2(r, r);
  const uint64_t r_lo = mul_f32x2(rr, pack_f32x2(kBracketLo, kBracketLo));
  const uint64_t r_hi = mul_f32x2(rr, pack_f32x2(kBracketHi, kBracketHi));
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t p = pack_f32x2(x[2 * i], x[2 * i + 1]);
    unpack_f32x2(mul_f32x2(p, r_lo), lo[2 * i], lo[2 * i + 1]);
    unpack_f32x2(mul_f32x2(p, r_hi), hi[2 * i], hi[2 * i + 1]);
  }
  const uint32_t c_lo = f32x8_to_e2m1x8(lo);
  const uint32_t c_hi = f32x8_to_e2m1x8(hi);
  if (c_lo == c_hi) return c_lo;
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], S);
  return f32x8_to_e2m1x8(q);
}

// E4M3 byte of fl32(a / b) (RNE, satfinite). Fast path as for the codes: the
// bracketed products a r_lo and a r_hi (one packed multiply) lie on either
// side of fl32(a / b); when both encode to the same byte, so does fl32(a / b).
// Otherwise, and for b outside [2^-100, 2^100] or a non-finite a, the
// quotient is formed with IEEE division.
__device__ __forceinline__ uint32_t e4m3_of_quotient(float a, float b) {
  if (b >= 7.8886091e-31f && b <= 1.2676506e30f && a <= 3.4028235e38f) {
    float r;
    asm("rcp.approx.f32 %0, %1;\n" : "=f"(r) : "f"(b));
    const uint64_t rb = mul_f32x2(pack_f32x2(r, r), pack_f32x2(kBracketLo, kBracketHi));
    float lo, hi;
    unpack_f32x2(mul_f32x2(pack_f32x2(a, a), rb), lo, hi);
    const uint32_t two = f32x2_to_e4m3x2(lo, hi);
    if ((two & 0xFFu) == (two >> 8)) return two & 0xFFu;
  }
  return f32_to_e4m3(__fdiv_rn(a, b));
}


// One group of 16 values (element 2j in the low nibble of byte j): the E4M3
// block scale sb = E4M3(fl32(amax / fl32(6 g))) (returned) and the E2M1 codes
// of fl32(x_i / fl32(E4M3(sb) g)) in c0 (elements 0..7) and c1 (8..15); every
// code is 0 when that effective scale is 0. Bit-exact with IEEE fp32 division.
// amax is the largest |x_i| with NaNs ignored (0 when all are NaN).
__device__ __forceinline__ uint32_t quantize_group16(const float (&x)[16], float g, uint32_t& c0,
                                                     uint32_t& c1) {
  const float m0 = max3f(fabsf(x[0]), fabsf(x[1]), fabsf(x[2]));
  const float m1 = max3f(fabsf(x[3]), fabsf(x[4]), fabsf(x[5]));
  const float m2 = max3f(fabsf(x[6]), fabsf(x[7]), fabsf(x[8]));
  const float m3 = max3f(fabsf(x[9]), fabsf(x[10]), fabsf(x[11]));
  const float m4 = max3f(fabsf(x[12]), fabsf(x[13]), fabsf(x[14]));
  const float amax = max3f(max3f(m0, m1, m2), max3f(m3, m4, fabsf(x[15])), 0.0f);
  const uint32_t sb = e4m3_of_quotient(amax, __fmul_rn(6.0f, g));
  const float S = __fmul_rn(e4m3_to_f32(sb), g);
  c0 = 0u;
  c1 = 0u;
  if (S >= 1.17549435e-38f) {
    c0 = e2m1_codes_div(*reinterpret_cast<const float(*)[8]>(x), S);
    c1 = e2m1_codes_div(*reinterpret_cast<const float(*)[8]>(x + 8), S);
  } else if (S > 0.0f) {  // subnormal effective scale: divide exactly
    float q0[8], q1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q0[i] = __fdiv_rn(x[i], S);
      q1[i] = __fdiv_rn(x[8 + i], S);
    }
    c0 = f32x8_to_e2m1x8(q0);
    c1 = f32x8_to_e2m1x8(q1);
  }
  return sb;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// ------------------------------------------------------------ tensor cores
// D = A(16x16, row) * B(16x8, col) + D, f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4],
                                              const uint32_t b[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t r[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

// ------------------------------------------------------------ bulk copies
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n"
      ".reg .b64 st;\n"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n"
      "}\n" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Four rows (y0..y3) of a 2-D tensor map, each one box row wide starting at
// column 0, gathered into consecutive rows at smem_dst; completes the bytes
// on `bar`. The tensor map must live in kernel parameter space.
__device__ __forceinline__ void tma_gather4(uint32_t smem_dst, const CUtensorMap* map, int y0,
                                            int y1, int y2, int y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];\n" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y0), "r"(y1), "r"(y2), "r"(y3),
      "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar` to complete. Returns false (and
// the caller reports NVFP4_DEV_TIMEOUT) if it did not complete in time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  int max_iters = kMaxWaitIters) {
  for (int i = 0; i < max_iters; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void lds_v2(uint32_t addr, uint32_t& x, uint32_t& y) {
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(x), "=r"(y) : "r"(addr));
}
__device__ __forceinline__ void lds_v4(uint32_t addr, uint32_t (&w)[4]) {
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t lds_b8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

}  // namespace nvfp4kv
