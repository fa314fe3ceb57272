// Host side shared by the attention entry points (api.cu, noalloc.cu): the
// argument block, the checks every entry point makes (nothing launched;
// NVFP4_OK with *nothing_to_do set for an empty batch), the launches (decode,
// then chunked prefill when the batch has multi-token query ranges) and the
// recording of a CUDA error for nvfp4_last_cuda_error. Status values are the
// NVFP4_* codes of include/nvfp4kv.h.
#pragma once

#include "nvfp4kv_launch.h"

namespace nvfp4kv {

AttentionArgs attention_args(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                             int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                             int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                             const int32_t* block_table, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, const int32_t* qo_indptr,
                             int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                             float sm_scale, uint8_t* o_fp8, const float* o_scale, void* o_bf16,
                             float* o_f32);
int check_attention(const AttentionArgs& a, bool* nothing_to_do);
int launch_attention(const AttentionArgs& a, cudaStream_t stream);
int cuda_status(cudaError_t e);
int decode_warps(int head_size, int block_size, int num_seqs, int group, int kv_format);

}  // namespace nvfp4kv
