// Paged attention without a caller-provided workspace.
//
// nvfp4_paged_attention needs scratch memory for its split-KV partial
// results, arrival counters and status word, and takes it from the caller.
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
// (with that device current) and keeps it for that device's context; do that
// first call outside any stream capture. If the context is re-created (after
// cudaDeviceReset), the next call looks the address up again. All calls on a
// device share the array and the array keeps whatever the previous call left
// in it, so each call clears the part that must start at zero (the arrival
// counters) on its stream before the kernels run. The status word is sticky,
// as in a caller's workspace: nvfp4_paged_attention_noalloc_status reads and
// optionally clears it. Calls that overlap on the GPU (different streams, no
// ordering between them) race on the array and must not be issued.
#include <mutex>

#include "../../include/nvfp4kv.h"
#include "nvfp4kv_host.h"

namespace nvfp4kv {

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
unsigned long long g_scratch_ctx[kMaxDevices] = {0};

// Device address of the scratch array on the current device, looked up once
// per (device, context).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long ctx = 0;
  err = nvfp4kv::current_context_id(&ctx);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_nvfp4_scratch);
    if (err != cudaSuccess) return err;
    // the look-up makes the context current if none was
    if (ctx == 0 && nvfp4kv::current_context_id(&ctx) != cudaSuccess) ctx = 0;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
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
  nvfp4kv::AttentionArgs a = nvfp4kv::attention_args(
      q, q_token_stride, num_q_tokens, num_q_heads, cache, num_blocks, block_size, num_kv_heads,
      head_size, block_table, max_blocks_per_seq, seq_lens, qo_indptr, num_seqs, max_q_len,
      kv_scales, sm_scale, o_fp8, o_scale, o_bf16, o_f32);
  bool nothing_to_do = false;
  const int st = nvfp4kv::check_attention(a, &nothing_to_do);
  if (st != NVFP4_OK || nothing_to_do) return st;
  const nvfp4kv::WorkspaceLayout wl = nvfp4kv::workspace_layout(
      num_seqs, num_kv_heads, head_size, num_q_heads / num_kv_heads);
  if (wl.total > nvfp4kv::kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;

  void* scratch = nullptr;
  int cst = nvfp4kv::cuda_status(scratch_address(&scratch));
  if (cst != NVFP4_OK) return cst;
  cudaStream_t s = (cudaStream_t)stream;
  // the arrival counters must start at zero; partial slots are always written
  // before they are read; the status word (bytes 0..3) is left as it is
  cst = nvfp4kv::cuda_status(cudaMemsetAsync(static_cast<uint8_t*>(scratch) + wl.counters_off, 0,
                                             wl.partials_off - wl.counters_off, s));
  if (cst != NVFP4_OK) return cst;
  a.workspace = scratch;
  return nvfp4kv::launch_attention(a, s);
}

int nvfp4_paged_attention_noalloc_status(uint32_t* host_bits, int clear, nvfp4_stream_t stream) {
  void* scratch = nullptr;
  const int cst = nvfp4kv::cuda_status(scratch_address(&scratch));
  if (cst != NVFP4_OK) return cst;
  return nvfp4_read_device_status(static_cast<const uint32_t*>(scratch), host_bits, clear, stream);
}

}  // extern "C"
