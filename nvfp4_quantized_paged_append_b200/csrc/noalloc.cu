// Paged attention without a caller-provided workspace.
//
// nvfp4_paged_attention needs scratch memory for its split-KV partial
// results, completion tickets and status word, and takes it from the caller.
// Some callers have no way to supply it: code handed only its input and
// output buffers by a host framework (a plugin or callback interface with no
// workspace hook), or code running while the device memory is owned by
// another allocator that does not let it reserve more. For them this file
// keeps one fixed scratch array in device memory, declared at file scope, so
// the call itself allocates nothing.
//
// The array is a `static __device__` object of kNoAllocScratchBytes bytes:
// every GPU that loads this library holds that much memory until the process
// exits. Host code cannot use the array's name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it; do that first call outside any
// stream capture. All calls on a device share the array and the array keeps
// whatever the previous call left in it, so each call clears the part that
// must start at zero (status word and completion tickets) on its stream
// before the kernels run. Calls that overlap on the GPU (different streams,
// no ordering between them) race on the array and must not be issued.
#include <math.h>

#include <mutex>

#include "../../include/nvfp4kv.h"
#include "nvfp4kv_launch.h"

namespace nvfp4kv {
int decode_warps(int head_size, int block_size, int num_seqs, int group);

// Largest workspace this entry point can serve (NVFP4_NOALLOC_SCRATCH_BYTES,
// 12 MiB): partial-result slots take 4736 * G * head_size * 4 bytes (4.9 MB
// for G = 2, head_size 128), plus 4 bytes per (sequence, kv head).
constexpr size_t kNoAllocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;
}  // namespace nvfp4kv

static __device__ __align__(256) uint8_t g_nvfp4_scratch[nvfp4kv::kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_nvfp4_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

int nvfp4_paged_attention_noalloc(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                                  int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                                  int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                                  const int32_t* block_table, int32_t max_blocks_per_seq,
                                  const int32_t* seq_lens, const int32_t* qo_indptr,
                                  int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                                  float sm_scale, uint8_t* o_fp8, const float* o_scale,
                                  void* o_bf16, float* o_f32, nvfp4_stream_t stream) {
  if (num_q_tokens < 0 || num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      head_size <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
      max_q_len < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (head_size % 16 != 0 || num_q_heads % num_kv_heads != 0) return NVFP4_ERR_INVALID_ARG;
  if (!(head_size == 64 || head_size == 128 || head_size == 256) ||
      !(block_size == 16 || block_size == 32))
    return NVFP4_ERR_UNSUPPORTED;
  if (num_q_heads / num_kv_heads > 8) return NVFP4_ERR_UNSUPPORTED;
  if (!qo_indptr && (num_q_tokens < num_seqs || max_q_len > 1)) return NVFP4_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_q_tokens == 0) return NVFP4_OK;
  if (!q || !cache || !block_table || !seq_lens || !kv_scales || !o_fp8 || !o_scale)
    return NVFP4_ERR_INVALID_ARG;
  if (q_token_stride < (int64_t)num_q_heads * head_size || q_token_stride % 8 != 0)
    return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) % 16) || (reinterpret_cast<uintptr_t>(cache) % 16) ||
      (reinterpret_cast<uintptr_t>(o_fp8) % 2) ||
      (o_bf16 && reinterpret_cast<uintptr_t>(o_bf16) % 4) ||
      (o_f32 && reinterpret_cast<uintptr_t>(o_f32) % 8))
    return NVFP4_ERR_INVALID_ARG;
  if ((int64_t)num_seqs * max_blocks_per_seq * num_kv_heads >= (int64_t)1 << 30 ||
      num_blocks * 2 * num_kv_heads >= (int64_t)1 << 31)
    return NVFP4_ERR_UNSUPPORTED;
  if (nvfp4kv::decode_warps(head_size, block_size, num_seqs, num_q_heads / num_kv_heads) < 1)
    return NVFP4_ERR_UNSUPPORTED;
  const nvfp4kv::WorkspaceLayout wl = nvfp4kv::workspace_layout(
      num_seqs, num_kv_heads, head_size, num_q_heads / num_kv_heads);
  if (wl.total > nvfp4kv::kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;

  void* scratch = nullptr;
  cudaError_t err = scratch_address(&scratch);
  if (err != cudaSuccess) return NVFP4_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // status word + completion tickets must start at zero; partial slots are
  // always written before they are read
  err = cudaMemsetAsync(scratch, 0, wl.partials_off, s);
  if (err != cudaSuccess) return NVFP4_ERR_CUDA;

  nvfp4kv::AttentionArgs a{};
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
  a.sm_scale = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)head_size);
  a.o_fp8 = o_fp8;
  a.o_scale = o_scale;
  a.o_bf16 = o_bf16;
  a.o_f32 = o_f32;
  a.workspace = scratch;
  err = nvfp4kv::launch_decode_attention(a, s);
  if (err == cudaSuccess && qo_indptr && max_q_len > 1)
    err = nvfp4kv::launch_prefill_attention(a, s);
  if (err != cudaSuccess) return NVFP4_ERR_CUDA;
  return NVFP4_OK;
}

}  // extern "C"
