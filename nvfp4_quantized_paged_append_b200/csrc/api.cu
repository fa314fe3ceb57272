// C ABI of libnvfp4kv: host-side validation, then kernel launches on the
// caller's stream. See include/nvfp4kv.h for the contract of each call.
#include <cudaTypedefs.h>
#include <math.h>

#include "../../include/nvfp4kv.h"
#include "nvfp4kv_host.h"

namespace {

bool head_size_ok(int64_t d) { return d == 64 || d == 128 || d == 256; }
bool block_size_ok(int64_t bs) { return bs == 16 || bs == 32; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

thread_local const char* g_last_error = "no error";

}  // namespace

namespace nvfp4kv {

cudaError_t current_context_id(unsigned long long* id) {
  struct Fns {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
  };
  static const Fns fns = [] {
    Fns f;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    return f;
  }();
  *id = 0;
  if (!fns.get_current || !fns.get_id) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (fns.get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  if (!ctx) return cudaSuccess;
  return fns.get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorUnknown;
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  g_last_error = cudaGetErrorString(e);
  return NVFP4_ERR_CUDA;
}

AttentionArgs attention_args(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                             int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                             int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                             const int32_t* block_table, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, const int32_t* qo_indptr,
                             int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                             float sm_scale, uint8_t* o_fp8, const float* o_scale, void* o_bf16,
                             float* o_f32) {
  AttentionArgs a{};
  a.q = q;
  a.q_token_stride = q_token_stride;
  a.num_q_tokens = num_q_tokens;
  a.num_q_heads = num_q_heads;
  a.cache = cache;
  a.num_blocks = num_blocks;
  a.block_size = block_size;
  a.num_kv_heads = num_kv_heads;
  a.head_size = head_size;
  a.block_table = block_table;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.seq_lens = seq_lens;
  a.qo_indptr = qo_indptr;
  a.num_seqs = num_seqs;
  a.max_q_len = max_q_len;
  a.kv_scales = kv_scales;
  a.sm_scale = (sm_scale > 0.0f || head_size <= 0) ? sm_scale : 1.0f / sqrtf((float)head_size);
  a.o_fp8 = o_fp8;
  a.o_scale = o_scale;
  a.o_bf16 = o_bf16;
  a.o_f32 = o_f32;
  return a;
}

int check_attention(const AttentionArgs& a, bool* nothing_to_do) {
  *nothing_to_do = false;
  if (a.num_q_tokens < 0 || a.num_seqs < 0 || a.num_q_heads <= 0 || a.num_kv_heads <= 0 ||
      a.head_size <= 0 || a.block_size <= 0 || a.num_blocks <= 0 || a.max_blocks_per_seq <= 0 ||
      a.max_q_len < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (a.head_size % 16 != 0 || a.num_q_heads % a.num_kv_heads != 0) return NVFP4_ERR_INVALID_ARG;
  if (!head_size_ok(a.head_size) || !block_size_ok(a.block_size)) return NVFP4_ERR_UNSUPPORTED;
  const int G = a.num_q_heads / a.num_kv_heads;
  if (G > 8) return NVFP4_ERR_UNSUPPORTED;
  if (!a.qo_indptr && a.num_q_tokens < a.num_seqs) return NVFP4_ERR_INVALID_ARG;
  if (!a.qo_indptr && a.max_q_len > 1) return NVFP4_ERR_INVALID_ARG;
  if (a.num_seqs == 0 || a.num_q_tokens == 0) {
    *nothing_to_do = true;
    return NVFP4_OK;
  }
  if (!a.q || !a.cache || !a.block_table || !a.seq_lens || !a.kv_scales || !a.o_fp8 ||
      !a.o_scale)
    return NVFP4_ERR_INVALID_ARG;
  if (a.q_token_stride < (int64_t)a.num_q_heads * a.head_size || a.q_token_stride % 8 != 0)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(a.q, 16) || !aligned(a.cache, 16) || !aligned(a.o_fp8, 2) ||
      (a.o_bf16 && !aligned(a.o_bf16, 4)) || (a.o_f32 && !aligned(a.o_f32, 8)))
    return NVFP4_ERR_INVALID_ARG;
  // flattened page indices and cache page rows are int32 on the device
  if ((int64_t)a.num_seqs * a.max_blocks_per_seq * a.num_kv_heads >= (int64_t)1 << 30 ||
      a.num_blocks * 2 * a.num_kv_heads >= (int64_t)1 << 31)
    return NVFP4_ERR_UNSUPPORTED;
  if (decode_warps(a.head_size, a.block_size, a.num_seqs, G, a.kv_format) < 1)
    return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

int launch_attention(const AttentionArgs& a, cudaStream_t s) {
  const int st = cuda_status(launch_decode_attention(a, s));
  if (st != NVFP4_OK) return st;
  if (a.qo_indptr && a.max_q_len > 1) return cuda_status(launch_prefill_attention(a, s));
  return NVFP4_OK;
}

}  // namespace nvfp4kv

using nvfp4kv::cuda_status;

extern "C" {

int64_t nvfp4_kv_full_dim(int64_t head_size) {
  if (head_size <= 0 || head_size % 16 != 0) return -1;
  return head_size / 2 + head_size / 16;
}

const char* nvfp4_last_cuda_error(void) { return g_last_error; }

const char* nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK:
      return "ok";
    case NVFP4_ERR_INVALID_ARG:
      return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case NVFP4_ERR_CUDA:
      return "CUDA error";
    case NVFP4_ERR_WORKSPACE:
      return "workspace missing or too small";
    case NVFP4_ERR_DEVICE_BOUNDS:
      return "a kernel skipped an out-of-range slot, block id or query range";
    case NVFP4_ERR_DEVICE_TIMEOUT:
      return "a kernel's bounded pipeline wait gave up";
    default:
      return "unknown status";
  }
}

static int quantize_append_fmt(const void* k, const void* v, int64_t k_token_stride,
                               int64_t v_token_stride, int64_t num_tokens, int32_t num_kv_heads,
                               int32_t head_size, uint8_t* cache, int64_t num_blocks,
                               int32_t block_size, const int64_t* slot_mapping,
                               const float* k_scale, const float* v_scale,
                               uint32_t* device_status, nvfp4_stream_t stream, int kv_format) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_size <= 0 || num_blocks <= 0 ||
      block_size <= 0)
    return NVFP4_ERR_INVALID_ARG;
  if (head_size % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!head_size_ok(head_size) || !block_size_ok(block_size)) return NVFP4_ERR_UNSUPPORTED;
  if (num_tokens == 0) return NVFP4_OK;
  if (!k || !v || !cache || !slot_mapping || !k_scale || !v_scale) return NVFP4_ERR_INVALID_ARG;
  const int64_t row = (int64_t)num_kv_heads * head_size;
  if (k_token_stride < row || v_token_stride < row || k_token_stride % 8 != 0 ||
      v_token_stride % 8 != 0)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(cache, 16) || !aligned(slot_mapping, 8))
    return NVFP4_ERR_INVALID_ARG;
  nvfp4kv::QuantizeAppendArgs a{k,           v,          k_token_stride, v_token_stride,
                                num_tokens,  num_kv_heads, head_size,    cache,
                                num_blocks,  block_size, slot_mapping,   k_scale,
                                v_scale,     device_status, kv_format};
  return cuda_status(nvfp4kv::launch_quantize_append(a, (cudaStream_t)stream));
}

int nvfp4_quantize_append_paged(const void* k, const void* v, int64_t k_token_stride,
                                int64_t v_token_stride, int64_t num_tokens,
                                int32_t num_kv_heads, int32_t head_size, uint8_t* cache,
                                int64_t num_blocks, int32_t block_size,
                                const int64_t* slot_mapping, const float* k_scale,
                                const float* v_scale, uint32_t* device_status,
                                nvfp4_stream_t stream) {
  return quantize_append_fmt(k, v, k_token_stride, v_token_stride, num_tokens, num_kv_heads,
                             head_size, cache, num_blocks, block_size, slot_mapping, k_scale,
                             v_scale, device_status, stream, 0);
}

int nvfp4_fp8kv_quantize_append_paged(const void* k, const void* v, int64_t k_token_stride,
                                      int64_t v_token_stride, int64_t num_tokens,
                                      int32_t num_kv_heads, int32_t head_size, uint8_t* cache,
                                      int64_t num_blocks, int32_t block_size,
                                      const int64_t* slot_mapping, const float* k_scale,
                                      const float* v_scale, uint32_t* device_status,
                                      nvfp4_stream_t stream) {
  return quantize_append_fmt(k, v, k_token_stride, v_token_stride, num_tokens, num_kv_heads,
                             head_size, cache, num_blocks, block_size, slot_mapping, k_scale,
                             v_scale, device_status, stream, 1);
}

size_t nvfp4_paged_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                            int32_t num_kv_heads, int32_t head_size) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_size <= 0) return 0;
  if (num_q_heads % num_kv_heads != 0) return 0;
  return nvfp4kv::workspace_layout(num_seqs, num_kv_heads, head_size,
                                   num_q_heads / num_kv_heads).total;
}

int nvfp4_paged_attention(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                          int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                          int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                          const int32_t* block_table, int32_t max_blocks_per_seq,
                          const int32_t* seq_lens, const int32_t* qo_indptr,
                          int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                          float sm_scale, uint8_t* o_fp8, const float* o_scale,
                          void* o_bf16, float* o_f32, void* workspace,
                          size_t workspace_bytes, nvfp4_stream_t stream) {
  return nvfp4_paged_attention_ex(q, q_token_stride, num_q_tokens, num_q_heads, cache,
                                  num_blocks, block_size, num_kv_heads, head_size, block_table,
                                  max_blocks_per_seq, seq_lens, qo_indptr, num_seqs, max_q_len,
                                  kv_scales, sm_scale, o_fp8, o_scale, o_bf16, o_f32, workspace,
                                  workspace_bytes, 0u, stream);
}

static int paged_attention_fmt(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                               int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                               int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                               const int32_t* block_table, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, const int32_t* qo_indptr,
                               int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                               float sm_scale, uint8_t* o_fp8, const float* o_scale,
                               void* o_bf16, float* o_f32, void* workspace,
                               size_t workspace_bytes, uint32_t flags, nvfp4_stream_t stream,
                               int kv_format) {
  if (flags & ~(NVFP4_ATTN_METADATA_READY | NVFP4_ATTN_HISTORY_READY | NVFP4_ATTN_QFP4))
    return NVFP4_ERR_INVALID_ARG;
  // NVFP4 queries (block-scaled QK^T in prefill rows): head size 256, NVFP4 cache
  if ((flags & NVFP4_ATTN_QFP4) && (head_size != 256 || kv_format != 0))
    return NVFP4_ERR_UNSUPPORTED;
  nvfp4kv::AttentionArgs a = nvfp4kv::attention_args(
      q, q_token_stride, num_q_tokens, num_q_heads, cache, num_blocks, block_size, num_kv_heads,
      head_size, block_table, max_blocks_per_seq, seq_lens, qo_indptr, num_seqs, max_q_len,
      kv_scales, sm_scale, o_fp8, o_scale, o_bf16, o_f32);
  a.kv_format = kv_format;
  bool nothing_to_do = false;
  const int st = nvfp4kv::check_attention(a, &nothing_to_do);
  if (st != NVFP4_OK || nothing_to_do) return st;
  const size_t need = nvfp4_paged_attention_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                           head_size);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return NVFP4_ERR_WORKSPACE;
  a.workspace = workspace;
  a.flags = flags;
  return nvfp4kv::launch_attention(a, (cudaStream_t)stream);
}

int nvfp4_paged_attention_ex(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                             int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                             int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                             const int32_t* block_table, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, const int32_t* qo_indptr,
                             int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                             float sm_scale, uint8_t* o_fp8, const float* o_scale,
                             void* o_bf16, float* o_f32, void* workspace,
                             size_t workspace_bytes, uint32_t flags, nvfp4_stream_t stream) {
  return paged_attention_fmt(q, q_token_stride, num_q_tokens, num_q_heads, cache, num_blocks,
                             block_size, num_kv_heads, head_size, block_table, max_blocks_per_seq,
                             seq_lens, qo_indptr, num_seqs, max_q_len, kv_scales, sm_scale, o_fp8,
                             o_scale, o_bf16, o_f32, workspace, workspace_bytes, flags, stream, 0);
}

int nvfp4_fp8kv_paged_attention(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                                int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                                int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* qo_indptr,
                                int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                                float sm_scale, uint8_t* o_fp8, const float* o_scale,
                                void* o_bf16, float* o_f32, void* workspace,
                                size_t workspace_bytes, uint32_t flags, nvfp4_stream_t stream) {
  return paged_attention_fmt(q, q_token_stride, num_q_tokens, num_q_heads, cache, num_blocks,
                             block_size, num_kv_heads, head_size, block_table, max_blocks_per_seq,
                             seq_lens, qo_indptr, num_seqs, max_q_len, kv_scales, sm_scale, o_fp8,
                             o_scale, o_bf16, o_f32, workspace, workspace_bytes, flags, stream, 1);
}

int nvfp4_status_from_bits(uint32_t bits) {
  if (bits & NVFP4_DEV_TIMEOUT) return NVFP4_ERR_DEVICE_TIMEOUT;
  if (bits & (NVFP4_DEV_BAD_SLOT | NVFP4_DEV_BAD_BLOCK | NVFP4_DEV_BAD_QLEN))
    return NVFP4_ERR_DEVICE_BOUNDS;
  return NVFP4_OK;
}

int nvfp4_read_device_status(const uint32_t* status_word, uint32_t* host_bits, int clear,
                             nvfp4_stream_t stream) {
  if (!status_word || !aligned(status_word, 4)) return NVFP4_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t bits = 0;
  int st = cuda_status(cudaMemcpyAsync(&bits, status_word, sizeof(bits), cudaMemcpyDeviceToHost, s));
  if (st != NVFP4_OK) return st;
  st = cuda_status(cudaStreamSynchronize(s));
  if (st != NVFP4_OK) return st;
  if (clear && bits) {
    st = cuda_status(cudaMemsetAsync(const_cast<uint32_t*>(status_word), 0, sizeof(bits), s));
    if (st != NVFP4_OK) return st;
  }
  if (host_bits) *host_bits = bits;
  return nvfp4_status_from_bits(bits);
}

int nvfp4_wait_timeout_probe(uint32_t* status_word, int32_t polls, nvfp4_stream_t stream) {
  if (!status_word || !aligned(status_word, 4) || polls < 1 || polls > (1 << 24))
    return NVFP4_ERR_INVALID_ARG;
  return cuda_status(nvfp4kv::launch_wait_timeout_probe(status_word, polls, (cudaStream_t)stream));
}

int nvfp4_paged_decode_append(const void* q, int64_t q_token_stride, int32_t num_q_heads,
                              const void* k_new, const void* v_new, int64_t k_token_stride,
                              int64_t v_token_stride, uint8_t* cache, int64_t num_blocks,
                              int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                              const int32_t* block_table, int32_t max_blocks_per_seq,
                              const int32_t* seq_lens, int32_t num_seqs, const float* kv_scales,
                              float sm_scale, uint8_t* o_fp8, const float* o_scale, void* o_bf16,
                              float* o_f32, void* workspace, size_t workspace_bytes,
                              uint32_t flags, nvfp4_stream_t stream) {
  if (flags & ~(NVFP4_ATTN_METADATA_READY | NVFP4_ATTN_HISTORY_READY))
    return NVFP4_ERR_INVALID_ARG;
  nvfp4kv::AttentionArgs a = nvfp4kv::attention_args(
      q, q_token_stride, num_seqs, num_q_heads, cache, num_blocks, block_size, num_kv_heads,
      head_size, block_table, max_blocks_per_seq, seq_lens, nullptr, num_seqs, 1, kv_scales,
      sm_scale, o_fp8, o_scale, o_bf16, o_f32);
  bool nothing_to_do = false;
  const int st = nvfp4kv::check_attention(a, &nothing_to_do);
  if (st != NVFP4_OK || nothing_to_do) return st;
  if (!k_new || !v_new) return NVFP4_ERR_INVALID_ARG;
  const int64_t row = (int64_t)num_kv_heads * head_size;
  if (k_token_stride < row || v_token_stride < row || k_token_stride % 8 != 0 ||
      v_token_stride % 8 != 0 || !aligned(k_new, 16) || !aligned(v_new, 16))
    return NVFP4_ERR_INVALID_ARG;
  const size_t need = nvfp4_paged_attention_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                           head_size);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return NVFP4_ERR_WORKSPACE;
  a.workspace = workspace;
  a.flags = flags;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_new_stride = k_token_stride;
  a.v_new_stride = v_token_stride;
  return nvfp4kv::launch_attention(a, (cudaStream_t)stream);
}

size_t nvfp4_activation_sf_bytes(int64_t rows, int64_t cols, int swizzled) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return 0;
  const int64_t c16 = cols / 16;
  if (!swizzled) return (size_t)(rows * c16);
  return (size_t)(((rows + 127) / 128 * 128) * ((c16 + 3) / 4 * 4));
}

int nvfp4_quantize_activation(const void* x, int64_t rows, int64_t cols, int64_t row_stride,
                              const float* global_scale_inv, uint8_t* out_fp4, uint8_t* out_sf,
                              int swizzled, nvfp4_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0 || row_stride < cols || row_stride % 8 != 0)
    return NVFP4_ERR_INVALID_ARG;
  if (rows == 0) return NVFP4_OK;
  if (!x || !global_scale_inv || !out_fp4 || !out_sf) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out_fp4, 8)) return NVFP4_ERR_INVALID_ARG;
  nvfp4kv::ActivationArgs a{x, rows, cols, row_stride, global_scale_inv, out_fp4, out_sf,
                            swizzled != 0};
  return cuda_status(nvfp4kv::launch_quantize_activation(a, (cudaStream_t)stream));
}

int nvfp4_dequantize_paged(const uint8_t* cache, int64_t num_blocks, int32_t block_size,
                           int32_t num_kv_heads, int32_t head_size,
                           const int32_t* block_ids, int64_t num_block_ids,
                           const float* kv_scales, void* out_bf16, nvfp4_stream_t stream) {
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_size <= 0 ||
      num_block_ids < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (head_size % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!head_size_ok(head_size) || !block_size_ok(block_size)) return NVFP4_ERR_UNSUPPORTED;
  if (num_block_ids == 0) return NVFP4_OK;
  if (!cache || !block_ids || !kv_scales || !out_bf16) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(cache, 16) || !aligned(out_bf16, 16)) return NVFP4_ERR_INVALID_ARG;
  nvfp4kv::DequantArgs a{cache, num_blocks, block_size, num_kv_heads, head_size,
                         block_ids, num_block_ids, kv_scales, out_bf16};
  return cuda_status(nvfp4kv::launch_dequantize_paged(a, (cudaStream_t)stream));
}

}  // extern "C"
