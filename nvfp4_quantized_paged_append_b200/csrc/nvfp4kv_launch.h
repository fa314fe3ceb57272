// Host-side launch interface between the C ABI (api.cu) and the kernels.
// Arguments arrive here already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace nvfp4kv {

struct QuantizeAppendArgs {
  const void* k;
  const void* v;
  int64_t k_token_stride, v_token_stride, num_tokens;
  int num_kv_heads, head_size;
  uint8_t* cache;
  int64_t num_blocks;
  int block_size;
  const int64_t* slot_mapping;
  const float* k_scale;
  const float* v_scale;
  uint32_t* device_status;
  int kv_format;  // 0: NVFP4 rows, 1: FP8-E4M3 rows
};

struct ActivationArgs {
  const void* x;  // bf16 [rows][row_stride]
  int64_t rows, cols, row_stride;
  const float* global_scale_inv;
  uint8_t* out_fp4;  // [rows][cols / 2]
  uint8_t* out_sf;   // swizzled or [rows][cols / 16]
  bool swizzled;
};

struct DequantArgs {
  const uint8_t* cache;
  int64_t num_blocks;
  int block_size, num_kv_heads, head_size;
  const int32_t* block_ids;
  int64_t num_block_ids;
  const float* kv_scales;
  void* out_bf16;
};

struct AttentionArgs {
  // the cache as a 2-D tensor of page rows (row r = (block, K|V, head) page,
  // PAGE / 8 eight-byte elements), for gather4 page loads; encoded by the
  // launcher when the configuration uses them
  CUtensorMap kv_pages;
  const void* q;
  int64_t q_token_stride, num_q_tokens;
  int num_q_heads;
  const uint8_t* cache;
  int64_t num_blocks;
  int block_size, num_kv_heads, head_size;
  const int32_t* block_table;
  int max_blocks_per_seq;
  const int32_t* seq_lens;
  const int32_t* qo_indptr;  // may be null (decode)
  int num_seqs, max_q_len;
  const float* kv_scales;
  float sm_scale;  // resolved (> 0)
  uint8_t* o_fp8;
  const float* o_scale;
  void* o_bf16;   // may be null
  float* o_f32;   // may be null
  void* workspace;
  uint32_t flags;  // NVFP4_ATTN_* launch flags (0: none)
  // fused append (decode only; k_new == nullptr: none): bf16 [num_seqs][Hkv][D]
  // rows of every sequence's newest token, quantized and written to position
  // seq_lens[b] - 1 of the cache by the decode kernel itself
  const void* k_new;
  const void* v_new;
  int64_t k_new_stride, v_new_stride;  // token strides in elements
  int kv_format;  // 0: NVFP4 rows (D/2 + D/16 bytes), 1: FP8-E4M3 rows (D bytes)
};

// Decode split-KV: at most kDecodeWarps warps in the whole grid; every warp
// owns a contiguous piece of the flattened key range and has two
// partial-state slots in the workspace (the segment holding its first unit,
// and the one holding its last).
constexpr int kDecodeCtas = 148 * 4;
constexpr int kDecodeWarps = kDecodeCtas * 4;

// Workspace layout (bytes from the start, all 256-byte aligned):
//   [0, 256)   uint32 device status word (+ padding)
//   counters:  int32 [num_seqs * num_kv_heads] arrival counts of the blocks
//              that hold pieces of a cut segment (back to 0 after each call)
//   partials:  float [kDecodeWarps * 2][group][head_size] accumulators
//   partial m/l: float [kDecodeWarps * 2][group][2]
struct WorkspaceLayout {
  size_t counters_off, partials_off, ml_off, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WorkspaceLayout workspace_layout(int num_seqs, int num_kv_heads,
                                                            int head_size, int group) {
  WorkspaceLayout w;
  w.counters_off = 256;
  w.partials_off = align256(w.counters_off + sizeof(int32_t) * (size_t)num_seqs * num_kv_heads);
  w.ml_off = align256(w.partials_off +
                      sizeof(float) * (size_t)kDecodeWarps * 2 * group * head_size);
  w.total = align256(w.ml_off + sizeof(float) * (size_t)kDecodeWarps * 2 * group * 2);
  return w;
}

// Unique id of the CUDA context current on the calling thread (0 if none is
// current yet). Per-device launch caches are keyed on it, so set-up done for a
// context that was since destroyed (cudaDeviceReset) is done again.
cudaError_t current_context_id(unsigned long long* id);

cudaError_t launch_quantize_append(const QuantizeAppendArgs& a, cudaStream_t stream);
cudaError_t launch_dequantize_paged(const DequantArgs& a, cudaStream_t stream);
cudaError_t launch_quantize_activation(const ActivationArgs& a, cudaStream_t stream);
cudaError_t launch_decode_attention(const AttentionArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_attention(const AttentionArgs& a, cudaStream_t stream);
// A one-block kernel that arms an mbarrier for 16 bytes no copy will deliver,
// waits on it with at most `polls` polls and ORs kDevTimeout into *status when
// the wait gives up (nothing is in flight when it returns).
cudaError_t launch_wait_timeout_probe(uint32_t* status, int polls, cudaStream_t stream);

}  // namespace nvfp4kv
