/*
 * NVFP4 paged KV cache -- CPU ORACLE (test infrastructure, not product code).
 *
 * Plain, slow, obviously-correct restatement of what the GPU path computes.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library. It shares no code, header, table or helper with the CUDA
 * path under nvfp4_quantized_paged_append_b200/csrc/.
 *
 * Sources (page title, section):
 *   [P1] "FlashInfer backend adds end-to-end NVFP4 KV cache support"
 *        (vLLM PR #40177 summary): "key source snippets" -- get_kv_cache_shape
 *        (last dim head_size/2 + head_size/16), _create_nvfp4_hnd_kv_cache
 *        (HND physical order (num_blocks, 2, num_kv_heads, block_size,
 *        full_dim); writer called with an arange slot mapping and
 *        k_scale = v_scale = kv_scale); "implementation breakdown" items 2-3
 *        (FP8 output dequantized to the model dtype; FP8 block scales split
 *        from the packed rows).
 *   [P3] "Move NVFP4 GEMM management into NvFp4LinearKernel" (vLLM PR #39129
 *        report), base.py, NvFp4LinearLayerConfig docstring: packed uint8
 *        holding two FP4 values per byte, one FP8-E4M3 scale per group of 16,
 *        plus a global scalar scale.
 *   Method statement: scale = E4M3(amax / (6 * global)), then
 *        round-to-nearest-even onto the E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6};
 *        attention in fp32 online softmax is defined here as plain fp64
 *        softmax attention over the dequantized cache.
 *
 * Readings where the pages are silent (the pages above fix only the shapes,
 * the packing and the scale formats; the method statement fixes the rounding):
 *   - element 2j sits in the LOW nibble of byte j, 2j+1 in the high nibble;
 *   - a row is [head_size/2 data bytes][head_size/16 scale bytes];
 *   - s32 = fl32(amax / fl32(6*g)); sb = E4M3_RNE_satfinite(s32);
 *     S = fl32(dec(sb) * g); code = E2M1_RNE_satfinite(fl32(x / S)),
 *     with IEEE fp32 division; if S == 0 every code of the group is 0x0;
 *   - rounding keeps the sign of x (a small negative value gives -0, 0x8);
 *   - dequant: xhat = E2M1(code) * E4M3(sb) * g;
 *   - attention: query row r of a sequence with q_len rows and L keys sits at
 *     absolute position L - q_len + r and sees keys 0..L-q_len+r; q head hq
 *     reads kv head hq / (Hq/Hkv); an empty window gives a zero output row;
 *   - o_fp8 = E4M3_RNE_satfinite(o / o_scale) from the fp64 value;
 *     o_bf16 = bf16_RNE(fl32(dec(o_fp8) * o_scale)).
 *
 * Floating point: compiled with -fno-fast-math -ffp-contract=off on x86-64
 * (SSE, FLT_EVAL_METHOD == 0), so every `float` operation below is one IEEE
 * binary32 operation with round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Element formats                                                           */
/* ------------------------------------------------------------------------ */

/* E2M1: sign(1) | exponent(2, bias 1) | mantissa(1). Exponent 0 is
 * subnormal: magnitude = mantissa * 0.5. No Inf, no NaN. */
double nvo_e2m1_decode(uint8_t code) {
  int sign = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

/* E4M3 ("fn" variant): sign(1) | exponent(4, bias 7) | mantissa(3).
 * Exponent 0 is subnormal: (m/8) * 2^-6. S.1111.111 is NaN; there is no Inf,
 * so the largest finite magnitude is 1.75 * 2^8 = 448. */
double nvo_e4m3_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 15;
  int m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Round a non-negative, non-NaN magnitude to the nearest entry of a grid
 * whose code i has magnitude grid(i), increasing in i for i = 0..n-1.
 * Ties go to the even code (for both formats the code's lowest bit is the
 * mantissa's lowest bit). Values at or above the top entry saturate to it
 * ("satfinite"). Midpoints of two grid values are exact in double, so every
 * comparison below is exact. */
static uint8_t rne_onto_grid(double ax, double (*grid)(uint8_t), int n) {
  if (ax >= grid((uint8_t)(n - 1))) return (uint8_t)(n - 1);
  for (int i = 0; i + 1 < n; ++i) {
    double lo = grid((uint8_t)i), hi = grid((uint8_t)(i + 1));
    if (ax <= hi) {
      double mid = 0.5 * (lo + hi);
      if (ax < mid) return (uint8_t)i;
      if (ax > mid) return (uint8_t)(i + 1);
      return (uint8_t)((i % 2 == 0) ? i : i + 1);
    }
  }
  return (uint8_t)(n - 1); /* not reached */
}

/* E4M3 round-to-nearest-even with saturation to +-448; NaN -> 0x7F. */
uint8_t nvo_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  return (uint8_t)(sign | rne_onto_grid(fabs(x), nvo_e4m3_decode, 127));
}

/* E2M1 round-to-nearest-even with saturation to +-6. NaN has no E2M1
 * encoding; it is mapped to +6 here (inputs with NaN are undefined). */
uint8_t nvo_e2m1_encode(double x) {
  if (isnan(x)) return 0x7;
  uint8_t sign = signbit(x) ? 0x8 : 0x0;
  return (uint8_t)(sign | rne_onto_grid(fabs(x), nvo_e2m1_decode, 8));
}

/* bfloat16 <-> binary32. bf16 is the upper half of a binary32, so widening
 * is exact. Narrowing rounds to nearest, ties to even, on the dropped 16
 * bits; NaN stays a quiet NaN. */
float nvo_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

uint16_t nvo_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040);
  uint32_t upper = u >> 16, lower = u & 0xFFFFu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
  return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* Cache geometry [P1, get_kv_cache_shape / _create_nvfp4_hnd_kv_cache]      */
/* ------------------------------------------------------------------------ */

int64_t nvo_full_dim(int64_t head_size) {
  if (head_size <= 0 || head_size % 16 != 0) return -1;
  return head_size / 2 + head_size / 16;
}

/* Byte offset of row (block, kv, head, offset) in the HND cache
 * uint8[num_blocks][2][num_kv_heads][block_size][full_dim]. */
static int64_t row_offset(int64_t block, int kv, int head, int off,
                          int num_kv_heads, int block_size, int64_t full_dim) {
  return (((block * 2 + kv) * num_kv_heads + head) * (int64_t)block_size + off) *
         full_dim;
}

/* ------------------------------------------------------------------------ */
/* Writer: quantize one row of head_size bf16 values                         */
/* ------------------------------------------------------------------------ */

void nvo_quantize_row(const uint16_t* x, int head_size, float g,
                      uint8_t* row) {
  int ngroups = head_size / 16;
  float six_g = 6.0f * g; /* fl32(6 * g) */
  for (int j = 0; j < ngroups; ++j) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float a = fabsf(nvo_bf16_to_f32(x[16 * j + i]));
      if (a > amax) amax = a;
    }
    float s32 = amax / six_g;                  /* IEEE fp32 division */
    uint8_t sb = nvo_e4m3_encode((double)s32); /* E4M3 RNE satfinite */
    float S = (float)nvo_e4m3_decode(sb) * g;  /* fl32(dec(sb) * g) */
    row[head_size / 2 + j] = sb;
    uint8_t code[16];
    for (int i = 0; i < 16; ++i) {
      if (S == 0.0f) {
        code[i] = 0x0;
      } else {
        float v = nvo_bf16_to_f32(x[16 * j + i]) / S; /* IEEE fp32 division */
        code[i] = nvo_e2m1_encode((double)v);
      }
    }
    for (int p = 0; p < 8; ++p)
      row[8 * j + p] = (uint8_t)(code[2 * p] | (code[2 * p + 1] << 4));
  }
}

/* Slot-mapped quantize-append [P1, _create_nvfp4_hnd_kv_cache and the
 * reshape_and_cache_flash call]: token t goes to slot slot_mapping[t]
 * (block = slot / block_size, offset = slot % block_size); slot < 0 skips
 * the token. k/v are bf16 [num_tokens][num_kv_heads][head_size] with the
 * given token strides (in elements). Returns the number of tokens whose slot
 * was >= num_blocks*block_size (those are not written). */
int64_t nvo_quantize_append_paged(const uint16_t* k, const uint16_t* v,
                                  int64_t k_token_stride,
                                  int64_t v_token_stride, int64_t num_tokens,
                                  int num_kv_heads, int head_size,
                                  uint8_t* cache, int64_t num_blocks,
                                  int block_size, const int64_t* slot_mapping,
                                  float k_scale, float v_scale) {
  int64_t full_dim = nvo_full_dim(head_size);
  int64_t bad = 0;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_blocks * block_size) {
      ++bad;
      continue;
    }
    int64_t block = slot / block_size;
    int off = (int)(slot % block_size);
    for (int h = 0; h < num_kv_heads; ++h) {
      nvo_quantize_row(k + t * k_token_stride + (int64_t)h * head_size,
                       head_size, k_scale,
                       cache + row_offset(block, 0, h, off, num_kv_heads,
                                          block_size, full_dim));
      nvo_quantize_row(v + t * v_token_stride + (int64_t)h * head_size,
                       head_size, v_scale,
                       cache + row_offset(block, 1, h, off, num_kv_heads,
                                          block_size, full_dim));
    }
  }
  return bad;
}

/* ------------------------------------------------------------------------ */
/* Dequantization                                                            */
/* ------------------------------------------------------------------------ */

/* xhat = E2M1(code) * E4M3(scale) for element d of a row (without g). The
 * product has at most 6 significant bits, so it is exact in double. */
static double row_elem(const uint8_t* row, int head_size, int d) {
  uint8_t byte = row[d / 2];
  uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  return nvo_e2m1_decode(code) * nvo_e4m3_decode(row[head_size / 2 + d / 16]);
}

/* Row formats of the paged cache: NVFP4 (E2M1 pairs + E4M3 block scales,
 * head_size/2 + head_size/16 bytes) or FP8 (one E4M3 byte per element,
 * head_size bytes; the per-tensor k_scale / v_scale multiplies it). */
enum { NVO_KV_NVFP4 = 0, NVO_KV_FP8 = 1 };

static int64_t kv_row_bytes(int kv_format, int head_size) {
  return kv_format == NVO_KV_FP8 ? (int64_t)head_size : nvo_full_dim(head_size);
}

/* Element d of a row without the global scale (exact in double). */
static double kv_elem(int kv_format, const uint8_t* row, int head_size, int d) {
  if (kv_format == NVO_KV_FP8) return nvo_e4m3_decode(row[d]);
  return row_elem(row, head_size, d);
}

/* Standalone dequant of listed blocks: out[i] = bf16 pages of block
 * block_ids[i], layout bf16[num_block_ids][2][num_kv_heads][block_size]
 * [head_size]; value bf16_RNE(fl32(xhat * g)), g = k_scale for K pages and
 * v_scale for V pages. */
void nvo_dequantize_paged(const uint8_t* cache, int64_t num_blocks,
                          int block_size, int num_kv_heads, int head_size,
                          const int32_t* block_ids, int64_t num_block_ids,
                          float k_scale, float v_scale, uint16_t* out) {
  (void)num_blocks;
  int64_t full_dim = nvo_full_dim(head_size);
  for (int64_t i = 0; i < num_block_ids; ++i) {
    int64_t block = block_ids[i];
    for (int kv = 0; kv < 2; ++kv) {
      float g = kv == 0 ? k_scale : v_scale;
      for (int h = 0; h < num_kv_heads; ++h)
        for (int off = 0; off < block_size; ++off) {
          const uint8_t* row =
              cache + row_offset(block, kv, h, off, num_kv_heads, block_size,
                                 full_dim);
          uint16_t* dst =
              out + (((i * 2 + kv) * num_kv_heads + h) * (int64_t)block_size +
                     off) * head_size;
          for (int d = 0; d < head_size; ++d) {
            float x = (float)row_elem(row, head_size, d) * g;
            dst[d] = nvo_f32_to_bf16(x);
          }
        }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Paged attention (fp64) with FP8-E4M3 output                               */
/* ------------------------------------------------------------------------ */

/* q: bf16 [num_q_tokens][num_q_heads][head_size].
 * block_table: int32 [num_seqs][max_blocks_per_seq]; seq_lens: int32
 * [num_seqs] = number of keys of the sequence (cached + new).
 * qo_indptr: int32 [num_seqs+1] query-token ranges, or NULL for decode (one
 * query token per sequence, token b for sequence b).
 * sm_scale <= 0 selects 1/sqrt(head_size).
 * Outputs (each may be NULL): o_f64 [num_q_tokens][num_q_heads][head_size],
 * o_fp8 (E4M3 bytes), o_bf16 (bf16 bits), same shape.
 * Rows are independent; the loop over them is split across threads. */
/* NVFP4 queries for a block-scaled QK^T (operand format of "Move NVFP4 GEMM
 * management into NvFp4LinearKernel", base.py): the global scale of a query
 * row is the smallest power of two g with amax(row) / (6 g) <= 448, i.e.
 * g = 2^ceil(log2(amax / 2688)) (1 for an all-zero row). Reading taken: the
 * pages quantize activations with a per-tensor global scale but fix none for
 * the query of a block-scaled QK^T; a per-row power of two keeps every block
 * scale in E4M3's range and folds exactly into the logit scale. */
float nvo_q_row_global(const uint16_t* x, int head_size) {
  float amax = 0.0f;
  for (int d = 0; d < head_size; ++d) {
    float a = fabsf(nvo_bf16_to_f32(x[d]));
    if (a > amax) amax = a;
  }
  if (!(amax > 0.0f)) return 1.0f;
  int E;
  frexpf(amax, &E);      /* amax in [2^(E-1), 2^E) */
  int k = (E - 1) - 11;  /* 2688 = 1.3125 * 2^11: ceil(log2(amax/2688)) is k or k+1 */
  if (ldexpf(2688.0f, k) >= amax) return ldexpf(1.0f, k);
  return ldexpf(1.0f, k + 1);
}

static void attention_impl(const uint16_t* q, int64_t num_q_tokens,
                           int num_q_heads, const uint8_t* cache,
                           int64_t num_blocks, int block_size, int num_kv_heads,
                           int head_size, const int32_t* block_table,
                           int max_blocks_per_seq, const int32_t* seq_lens,
                           const int32_t* qo_indptr, int num_seqs, float k_scale,
                           float v_scale, double sm_scale, float o_scale,
                           double* o_f64, uint8_t* o_fp8, uint16_t* o_bf16,
                           int kv_format, int q_fp4) {
  (void)num_blocks;
  (void)num_q_tokens;
  int64_t full_dim = kv_row_bytes(kv_format, head_size);
  int group = num_q_heads / num_kv_heads;
  if (sm_scale <= 0.0) sm_scale = 1.0 / sqrt((double)head_size);

  /* One task per (sequence, query row, query head); list the rows first. */
  int64_t num_rows = 0;
  for (int b = 0; b < num_seqs; ++b)
    num_rows += qo_indptr ? (qo_indptr[b + 1] - qo_indptr[b]) : 1;
  int32_t* row_seq = (int32_t*)malloc(sizeof(int32_t) * (num_rows + 1));
  int64_t* row_idx = (int64_t*)malloc(sizeof(int64_t) * (num_rows + 1));
  {
    int64_t k = 0;
    for (int b = 0; b < num_seqs; ++b) {
      int64_t q_len = qo_indptr ? (qo_indptr[b + 1] - qo_indptr[b]) : 1;
      for (int64_t r = 0; r < q_len; ++r, ++k) {
        row_seq[k] = b;
        row_idx[k] = r;
      }
    }
  }

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t task = 0; task < num_rows * num_q_heads; ++task) {
    int64_t row = task / num_q_heads;
    int hq = (int)(task % num_q_heads);
    int b = row_seq[row];
    int64_t r = row_idx[row];
    int64_t L = seq_lens[b];
    int64_t q_begin = qo_indptr ? qo_indptr[b] : b;
    int64_t q_len = qo_indptr ? (qo_indptr[b + 1] - qo_indptr[b]) : 1;
    int h = hq / group;
    int64_t tok = q_begin + r;
    int64_t last = L - q_len + r; /* keys 0..last are visible */
    int64_t nkeys = last + 1 > 0 ? last + 1 : 0;
    if (nkeys > L) nkeys = L;
    const uint16_t* qrow = q + (tok * num_q_heads + hq) * (int64_t)head_size;
    /* the query as the dot products see it: bf16, or (q_fp4, rows of
     * sequences with more than one query) its NVFP4 round trip under the
     * row's global scale */
    double* qv = (double*)malloc(sizeof(double) * (size_t)head_size);
    if (q_fp4 && q_len > 1) {
      float g = nvo_q_row_global(qrow, head_size);
      uint8_t* qq = (uint8_t*)malloc((size_t)(head_size / 2 + head_size / 16));
      nvo_quantize_row(qrow, head_size, g, qq);
      for (int d = 0; d < head_size; ++d)
        qv[d] = row_elem(qq, head_size, d) * (double)g;
      free(qq);
    } else {
      for (int d = 0; d < head_size; ++d) qv[d] = (double)nvo_bf16_to_f32(qrow[d]);
    }
    double* z = (double*)malloc(sizeof(double) * (nkeys > 0 ? nkeys : 1));
    double* o = (double*)calloc((size_t)head_size, sizeof(double));
    double m = -INFINITY;
    for (int64_t n = 0; n < nkeys; ++n) {
      int64_t block =
          block_table[(int64_t)b * max_blocks_per_seq + n / block_size];
      const uint8_t* krow =
          cache + row_offset(block, 0, h, (int)(n % block_size), num_kv_heads,
                             block_size, full_dim);
      double dot = 0.0;
      for (int d = 0; d < head_size; ++d)
        dot += qv[d] * (kv_elem(kv_format, krow, head_size, d) * (double)k_scale);
      z[n] = sm_scale * dot;
      if (z[n] > m) m = z[n];
    }
    double l = 0.0;
    for (int64_t n = 0; n < nkeys; ++n) {
      double w = exp(z[n] - m);
      l += w;
      int64_t block =
          block_table[(int64_t)b * max_blocks_per_seq + n / block_size];
      const uint8_t* vrow =
          cache + row_offset(block, 1, h, (int)(n % block_size), num_kv_heads,
                             block_size, full_dim);
      for (int d = 0; d < head_size; ++d)
        o[d] += w * (kv_elem(kv_format, vrow, head_size, d) * (double)v_scale);
    }
    int64_t out_base = (tok * num_q_heads + hq) * (int64_t)head_size;
    for (int d = 0; d < head_size; ++d) {
      double od = (l > 0.0) ? o[d] / l : 0.0;
      if (o_f64) o_f64[out_base + d] = od;
      uint8_t c = nvo_e4m3_encode(od / (double)o_scale);
      if (o_fp8) o_fp8[out_base + d] = c;
      if (o_bf16)
        o_bf16[out_base + d] =
            nvo_f32_to_bf16((float)nvo_e4m3_decode(c) * o_scale);
    }
    free(z);
    free(o);
    free(qv);
  }
  free(row_seq);
  free(row_idx);
}

void nvo_paged_attention_fmt(const uint16_t* q, int64_t num_q_tokens,
                             int num_q_heads, const uint8_t* cache,
                             int64_t num_blocks, int block_size, int num_kv_heads,
                             int head_size, const int32_t* block_table,
                             int max_blocks_per_seq, const int32_t* seq_lens,
                             const int32_t* qo_indptr, int num_seqs, float k_scale,
                             float v_scale, double sm_scale, float o_scale,
                             double* o_f64, uint8_t* o_fp8, uint16_t* o_bf16,
                             int kv_format) {
  attention_impl(q, num_q_tokens, num_q_heads, cache, num_blocks, block_size,
                 num_kv_heads, head_size, block_table, max_blocks_per_seq,
                 seq_lens, qo_indptr, num_seqs, k_scale, v_scale, sm_scale,
                 o_scale, o_f64, o_fp8, o_bf16, kv_format, 0);
}

/* NVFP4 cache, NVFP4-quantized queries in prefill rows (see nvo_q_row_global). */
void nvo_paged_attention_qfp4(const uint16_t* q, int64_t num_q_tokens,
                              int num_q_heads, const uint8_t* cache,
                              int64_t num_blocks, int block_size, int num_kv_heads,
                              int head_size, const int32_t* block_table,
                              int max_blocks_per_seq, const int32_t* seq_lens,
                              const int32_t* qo_indptr, int num_seqs, float k_scale,
                              float v_scale, double sm_scale, float o_scale,
                              double* o_f64, uint8_t* o_fp8, uint16_t* o_bf16) {
  attention_impl(q, num_q_tokens, num_q_heads, cache, num_blocks, block_size,
                 num_kv_heads, head_size, block_table, max_blocks_per_seq,
                 seq_lens, qo_indptr, num_seqs, k_scale, v_scale, sm_scale,
                 o_scale, o_f64, o_fp8, o_bf16, NVO_KV_NVFP4, 1);
}

/* NVFP4 cache (the format above). */
void nvo_paged_attention(const uint16_t* q, int64_t num_q_tokens,
                         int num_q_heads, const uint8_t* cache,
                         int64_t num_blocks, int block_size, int num_kv_heads,
                         int head_size, const int32_t* block_table,
                         int max_blocks_per_seq, const int32_t* seq_lens,
                         const int32_t* qo_indptr, int num_seqs, float k_scale,
                         float v_scale, double sm_scale, float o_scale,
                         double* o_f64, uint8_t* o_fp8, uint16_t* o_bf16) {
  nvo_paged_attention_fmt(q, num_q_tokens, num_q_heads, cache, num_blocks,
                          block_size, num_kv_heads, head_size, block_table,
                          max_blocks_per_seq, seq_lens, qo_indptr, num_seqs,
                          k_scale, v_scale, sm_scale, o_scale, o_f64, o_fp8,
                          o_bf16, NVO_KV_NVFP4);
}

/* ------------------------------------------------------------------------ */
/* FP8-E4M3 KV cache (the comparison format)                                 */
/* ------------------------------------------------------------------------ */

/* [P1] review highlights and risks: the FP8 KV cache is the format NVFP4 is
 * compared with (TPOT at batch 256). Reading taken: the FP8 cache has the same
 * HND page layout with head_size-byte rows of E4M3 codes; the writer stores
 * E4M3_RNE_satfinite(fl32(x / g)) (IEEE fp32 division, g = k_scale or
 * v_scale) and the attention reads xhat = E4M3(code) * g. */
int64_t nvo_fp8kv_quantize_append_paged(const uint16_t* k, const uint16_t* v,
                                        int64_t k_token_stride,
                                        int64_t v_token_stride,
                                        int64_t num_tokens, int num_kv_heads,
                                        int head_size, uint8_t* cache,
                                        int64_t num_blocks, int block_size,
                                        const int64_t* slot_mapping,
                                        float k_scale, float v_scale) {
  int64_t bad = 0;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_blocks * block_size) {
      ++bad;
      continue;
    }
    int64_t block = slot / block_size;
    int off = (int)(slot % block_size);
    for (int kv = 0; kv < 2; ++kv) {
      const uint16_t* src = kv == 0 ? k + t * k_token_stride : v + t * v_token_stride;
      float g = kv == 0 ? k_scale : v_scale;
      for (int h = 0; h < num_kv_heads; ++h) {
        uint8_t* row = cache + row_offset(block, kv, h, off, num_kv_heads,
                                          block_size, head_size);
        for (int d = 0; d < head_size; ++d) {
          float x = nvo_bf16_to_f32(src[(int64_t)h * head_size + d]) / g;
          row[d] = nvo_e4m3_encode((double)x);
        }
      }
    }
  }
  return bad;
}

/* ------------------------------------------------------------------------ */
/* Activation quantizer with the block-scaled GEMM's scale-factor layout      */
/* ------------------------------------------------------------------------ */

/* [P3] "Move NVFP4 GEMM management into NvFp4LinearKernel", flashinfer.py and
 * the CUTLASS linear kernel: scaled_fp4_quant(x, input_global_scale_inv,
 * is_sf_swizzled_layout=True) turns the activations into packed E2M1 pairs
 * plus one E4M3 scale per 16 values, and swizzle_blockscale rearranges scales
 * for the block-scaled GEMM. The pages name both helpers without defining
 * them; the readings taken here:
 *   - the argument is the inverse global scale; g = fl32(1 / inv) (IEEE
 *     division), and every row is then quantized exactly like a KV-cache row
 *     (nvo_quantize_row): scale E4M3(amax / (6 g)), codes RNE onto E2M1;
 *   - packed data: uint8 [rows][cols/2], element 2j in the low nibble;
 *   - plain scales: uint8 [rows][cols/16];
 *   - swizzled scales: rows padded to a multiple of 128 and scale columns to
 *     a multiple of 4 (padding bytes 0); 512-byte tiles of 128 rows x 4 scale
 *     columns, tile (r/128, c/4) at ((r/128) * (padded cols / 4) + c/4) * 512,
 *     and inside a tile entry (r, c) at (r % 32) * 16 + ((r % 128) / 32) * 4
 *     + c % 4 (the 32 x 4 x 4 interleave of the block-scaled MMA). */
int64_t nvo_act_sf_bytes(int64_t rows, int64_t cols, int swizzled) {
  int64_t c16 = cols / 16;
  if (!swizzled) return rows * c16;
  int64_t pr = (rows + 127) / 128 * 128, pc = (c16 + 3) / 4 * 4;
  return pr * pc;
}

int64_t nvo_act_sf_index(int64_t r, int64_t c, int64_t cols) {
  int64_t pc = (cols / 16 + 3) / 4 * 4;
  int64_t tile = (r / 128) * (pc / 4) + c / 4;
  return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4;
}

void nvo_quantize_activation(const uint16_t* x, int64_t rows, int64_t cols,
                             int64_t row_stride, float global_scale_inv,
                             uint8_t* out_fp4, uint8_t* out_sf, int swizzled) {
  float g = 1.0f / global_scale_inv; /* IEEE fp32 division */
  int64_t c16 = cols / 16;
  uint8_t* row = (uint8_t*)malloc((size_t)(cols / 2 + c16));
  memset(out_sf, 0, (size_t)nvo_act_sf_bytes(rows, cols, swizzled));
  for (int64_t r = 0; r < rows; ++r) {
    nvo_quantize_row(x + r * row_stride, (int)cols, g, row);
    memcpy(out_fp4 + r * (cols / 2), row, (size_t)(cols / 2));
    for (int64_t c = 0; c < c16; ++c) {
      int64_t at = swizzled ? nvo_act_sf_index(r, c, cols) : r * c16 + c;
      out_sf[at] = row[cols / 2 + c];
    }
  }
  free(row);
}
