/*
 * nvfp4kv -- NVFP4 paged KV cache for B200 (sm_100a): C ABI.
 *
 * Two hot operations and two helpers, after the pages on NVFP4 KV caches:
 *   - "FlashInfer backend adds end-to-end NVFP4 KV cache support" (vLLM PR
 *     #40177 summary), key source snippets: get_kv_cache_shape gives the
 *     cache shape (num_blocks, 2, block_size, num_kv_heads, full_dim) with
 *     full_dim = head_size/2 + head_size/16; _create_nvfp4_hnd_kv_cache stores
 *     it in HND order (num_blocks, 2, num_kv_heads, block_size, full_dim) and
 *     fills it with reshape_and_cache_flash(k, v, ..., slot_mapping, "nvfp4",
 *     k_scale, v_scale); implementation breakdown items 2-3: the attention
 *     kernel reads the packed data plus the FP8 block scales and writes FP8
 *     output that is dequantized back to the model dtype.
 *   - "FlashInfer NVFP4 KV serving on pre-SM100 GPUs" (vLLM RFC #47684),
 *     quick answer: the slot-mapped NVFP4 append helper and the paged NVFP4
 *     dequantize helper.
 *   - "Move NVFP4 GEMM management into NvFp4LinearKernel" (vLLM PR #39129),
 *     base.py, NvFp4LinearLayerConfig: two FP4 (E2M1) values per byte, one
 *     FP8-E4M3 scale per 16 values, one global scale.
 *
 * Cache row (per token, per kv head, K or V): full_dim bytes =
 *   [head_size/2 bytes: E2M1 pairs, element 2j in the low nibble of byte j]
 *   [head_size/16 bytes: E4M3 block scales, one per 16 elements]
 * Physical cache layout (HND): uint8 [num_blocks][2][num_kv_heads][block_size]
 * [full_dim]; index 0 of the second dim is K, 1 is V. A page (block, K|V,
 * head) is block_size*full_dim contiguous bytes.
 *
 * Quantization (bit-exact contract, g = k_scale or v_scale, fp32):
 *   per group of 16: s32 = fl32(amax / fl32(6*g)); sb = E4M3 RNE satfinite(s32);
 *   S = fl32(E4M3(sb) * g); code = E2M1 RNE satfinite(fl32(x / S)) (IEEE
 *   division; sign kept, so small negatives give 0x8); S == 0 -> all codes 0.
 * Dequantization: xhat = E2M1(code) * E4M3(sb) * g.
 *
 * Conventions for every entry point:
 *   - All pointers are caller-owned DEVICE memory unless stated; the library
 *     never allocates device memory and never synchronizes the stream (the
 *     status read-back calls excepted, which say so).
 *   - Work is enqueued on `stream` (cudaStream_t; NULL = legacy default).
 *   - Host-side validation failures return a negative status and launch
 *     nothing. A CUDA launch error returns NVFP4_ERR_CUDA. Device-side faults
 *     that the kernels detect (out-of-range block ids, a pipeline wait that
 *     timed out) skip the bad access and raise bits in a device status word.
 *   - bf16 tensors are passed as `const void*` (IEEE bfloat16 bit patterns).
 *   - Supported: head_size in {64, 128, 256}; block_size in {16, 32};
 *     num_q_heads / num_kv_heads in 1..8 (attention).
 */
#ifndef NVFP4KV_H_
#define NVFP4KV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NVFP4KV_API __attribute__((visibility("default")))
#else
#define NVFP4KV_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = -1, /* null pointer, negative size, bad shape */
  NVFP4_ERR_UNSUPPORTED = -2, /* valid but not built: head_size, block_size, GQA group */
  NVFP4_ERR_CUDA = -3,        /* kernel launch / CUDA runtime error */
  NVFP4_ERR_WORKSPACE = -4,   /* workspace null or smaller than required */
  NVFP4_ERR_DEVICE_BOUNDS = -5, /* read back: a kernel skipped an out-of-range
                                   slot, block id or query range */
  NVFP4_ERR_DEVICE_TIMEOUT = -6 /* read back: a bounded pipeline wait gave up */
} nvfp4_status;

/* Bits of the device status word (see nvfp4_paged_attention's workspace and
 * nvfp4_quantize_append_paged's `device_status`). */
#define NVFP4_DEV_BAD_SLOT 0x1u    /* slot >= num_blocks*block_size (token skipped) */
#define NVFP4_DEV_BAD_BLOCK 0x2u   /* block id outside [0, num_blocks) (page skipped) */
#define NVFP4_DEV_TIMEOUT 0x4u     /* a bounded pipeline wait gave up */
#define NVFP4_DEV_BAD_QLEN 0x8u    /* a query range longer than max_q_len (rows
                                      past max_q_len left unwritten) */

/* Row width in bytes, head_size/2 + head_size/16 ("FlashInfer backend adds
 * end-to-end NVFP4 KV cache support", get_kv_cache_shape, the
 * nvfp4_kv_cache_full_dim helper). Returns -1 if head_size <= 0 or
 * head_size % 16 != 0. Pure host function. */
NVFP4KV_API int64_t nvfp4_kv_full_dim(int64_t head_size);

/* Slot-mapped quantize-append ("FlashInfer backend adds end-to-end NVFP4 KV
 * cache support", reshape_and_cache_flash with kv_cache_dtype "nvfp4";
 * "FlashInfer NVFP4 KV serving on pre-SM100 GPUs", the slot-mapping append
 * helper).
 *   k, v            bf16 [num_tokens][num_kv_heads][head_size]; heads and
 *                   elements contiguous, token stride given in ELEMENTS
 *                   (>= num_kv_heads*head_size; allows views into a fused
 *                   qkv buffer). 16-byte aligned rows required.
 *   cache           uint8 HND cache, num_blocks*2*num_kv_heads*block_size*
 *                   full_dim bytes, 16-byte aligned.
 *   slot_mapping    int64 [num_tokens]; token t goes to block slot/block_size,
 *                   offset slot%block_size; slot < 0 skips the token; a slot
 *                   >= num_blocks*block_size is skipped and flagged.
 *   k_scale,v_scale device fp32 scalars (global scales g; finite, > 0).
 *   device_status   optional (NULL allowed) device uint32 word; the kernel
 *                   ORs NVFP4_DEV_BAD_SLOT into it. Never cleared here.
 * Rows not named by a slot are never touched. Duplicate slots: undefined
 * which token wins. num_tokens == 0 is a no-op returning NVFP4_OK. */
NVFP4KV_API int nvfp4_quantize_append_paged(const void* k, const void* v, int64_t k_token_stride,
                                int64_t v_token_stride, int64_t num_tokens,
                                int32_t num_kv_heads, int32_t head_size, uint8_t* cache,
                                int64_t num_blocks, int32_t block_size,
                                const int64_t* slot_mapping, const float* k_scale,
                                const float* v_scale, uint32_t* device_status,
                                nvfp4_stream_t stream);

/* Bytes of workspace nvfp4_paged_attention needs for these sizes (a pure host
 * function of its arguments). Returns 0 for invalid arguments. */
NVFP4KV_API size_t nvfp4_paged_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                            int32_t num_kv_heads, int32_t head_size);

/* Paged decode and chunked-prefill attention over the NVFP4 cache ("FlashInfer
 * backend adds end-to-end NVFP4 KV cache support", implementation breakdown
 * items 2-3: FP8 output, dequantized back to the model dtype; the pages read
 * through a block table with the split-out FP8 block scales).
 *   q               bf16 [num_q_tokens][num_q_heads][head_size], token stride
 *                   q_token_stride in elements, 16-byte aligned rows.
 *   cache           HND cache as above.
 *   block_table     int32 [num_seqs][max_blocks_per_seq]: logical block i of
 *                   sequence b lives in cache block block_table[b][i].
 *   seq_lens        int32 [num_seqs]: keys of sequence b (cached + new), >= 1.
 *   qo_indptr       int32 [num_seqs+1] query-token ranges (chunked prefill and
 *                   mixed batches), or NULL: one query token per sequence
 *                   (token b of q belongs to sequence b; decode).
 *                   Query row r of a sequence with q_len = qo_indptr[b+1] -
 *                   qo_indptr[b] sits at position seq_lens[b]-q_len+r and sees
 *                   keys 0..seq_lens[b]-q_len+r (causal); an empty window
 *                   writes zeros.
 *   max_q_len       host upper bound on every q_len (1 for pure decode).
 *   kv_scales       device fp32 [2] = {k_scale, v_scale}.
 *   sm_scale        softmax scale; <= 0 selects 1/sqrt(head_size).
 *   o_fp8           uint8 E4M3 [num_q_tokens][num_q_heads][head_size]:
 *                   E4M3 RNE satfinite(o / o_scale), 2-byte aligned.
 *   o_scale         device fp32 scalar (> 0).
 *   o_bf16          optional bf16 output, same shape: bf16(E4M3(o_fp8)*o_scale),
 *                   4-byte aligned.
 *   o_f32           optional fp32 output of o before the FP8 cast (testing),
 *                   8-byte aligned. (Adjacent pairs of d are stored together.)
 *   workspace       device scratch of >= nvfp4_paged_attention_workspace_size
 *                   bytes, 256-byte aligned, ZERO-FILLED before its first use;
 *                   every call that completes leaves it ready for the next
 *                   one. Its first 4 bytes are the device status word
 *                   (NVFP4_DEV_* bits, sticky until the caller clears them).
 *                   Calls that share a workspace must not overlap on the GPU.
 * The GQA group G = num_q_heads/num_kv_heads maps q head hq to kv head hq/G. */
NVFP4KV_API int nvfp4_paged_attention(const void* q, int64_t q_token_stride, int64_t num_q_tokens,
                          int32_t num_q_heads, const uint8_t* cache, int64_t num_blocks,
                          int32_t block_size, int32_t num_kv_heads, int32_t head_size,
                          const int32_t* block_table, int32_t max_blocks_per_seq,
                          const int32_t* seq_lens, const int32_t* qo_indptr,
                          int32_t num_seqs, int32_t max_q_len, const float* kv_scales,
                          float sm_scale, uint8_t* o_fp8, const float* o_scale,
                          void* o_bf16, float* o_f32, void* workspace,
                          size_t workspace_bytes, nvfp4_stream_t stream);

/* nvfp4_paged_attention with launch flags (no counterpart in the pages; a
 * B200 launch option). The decode kernel is always launched as a programmatic
 * dependent of the kernel before it on `stream`: its blocks may become
 * resident while that kernel finishes, and by default they read nothing until
 * it has completed. With NVFP4_ATTN_METADATA_READY the caller promises that
 * the preceding kernel writes none of block_table, seq_lens, qo_indptr,
 * kv_scales, o_scale and the workspace (they were made ready earlier, e.g.
 * copied from the host before it); the kernel then reads them, builds its
 * work split, fetches block ids (setting NVFP4_DEV_BAD_BLOCK in the status
 * word for bad ones) before waiting, and reads q and the cache only after.
 * With NVFP4_ATTN_HISTORY_READY (which implies NVFP4_ATTN_METADATA_READY) the
 * caller further promises that the preceding kernel writes no cache page this
 * call reads (for nvfp4_paged_decode_append: none of each sequence's keys
 * before position seq_len - 1, the row the call writes itself), as when that
 * kernel is the projection producing q; the first page copies then start
 * before the wait as well, overlapping that kernel's tail.
 * flags = 0 is nvfp4_paged_attention. Unknown bits: NVFP4_ERR_INVALID_ARG. */
#define NVFP4_ATTN_METADATA_READY 0x1u
#define NVFP4_ATTN_HISTORY_READY 0x2u
/* NVFP4_ATTN_QFP4 (nvfp4_paged_attention_ex only; head size 256 over the NVFP4
 * cache, else NVFP4_ERR_UNSUPPORTED): the rows of sequences with more than one
 * query compute q K^T on the block-scaled tensor-core path
 * (tcgen05 kind::mxf4nvf4), with each query row quantized to NVFP4 by the KV
 * row codec under its own power-of-two global scale, the smallest g with
 * max|q| / (6 g) <= 448, and K read as the cache's own codes and block scales.
 * It changes the results (a variant measured against the same tolerance over
 * the quantized queries); decode rows are unchanged. */
#define NVFP4_ATTN_QFP4 0x4u
NVFP4KV_API int nvfp4_paged_attention_ex(
    const void* q, int64_t q_token_stride, int64_t num_q_tokens, int32_t num_q_heads,
    const uint8_t* cache, int64_t num_blocks, int32_t block_size, int32_t num_kv_heads,
    int32_t head_size, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, const int32_t* qo_indptr, int32_t num_seqs, int32_t max_q_len,
    const float* kv_scales, float sm_scale, uint8_t* o_fp8, const float* o_scale,
    void* o_bf16, float* o_f32, void* workspace, size_t workspace_bytes, uint32_t flags,
    nvfp4_stream_t stream);

/* Decode step with the append fused in: one launch that quantizes and writes
 * every sequence's newest K and V rows into the cache and runs decode
 * attention over all of each sequence's keys, the new ones included
 * ("FlashInfer backend adds end-to-end NVFP4 KV cache support", key source
 * snippets: the forward pass calls reshape_and_cache_flash with the nvfp4
 * dtype and then the attention kernel; here they are one kernel).
 * Results equal those of nvfp4_quantize_append_paged (same bytes) followed by
 * nvfp4_paged_attention on the same stream, with:
 *   q               bf16 [num_seqs][num_q_heads][head_size] (token b = the
 *                   query of sequence b), token stride q_token_stride.
 *   k_new, v_new    bf16 [num_seqs][num_kv_heads][head_size], token strides
 *                   in elements, 16-byte aligned rows: the newest token of
 *                   sequence b, written to position seq_lens[b] - 1, i.e. slot
 *                   block_table[b][(L-1)/block_size]*block_size +
 *                   (L-1)%block_size with L = seq_lens[b] (>= 1).
 *   kv_scales       {k_scale, v_scale}: the global scales of the writer and of
 *                   the attention.
 * Every other argument, the workspace contract and `flags` are those of
 * nvfp4_paged_attention_ex (no query ranges: decode only). A new row whose
 * block id is out of range is neither written nor attended to
 * (NVFP4_DEV_BAD_BLOCK). */
NVFP4KV_API int nvfp4_paged_decode_append(
    const void* q, int64_t q_token_stride, int32_t num_q_heads, const void* k_new,
    const void* v_new, int64_t k_token_stride, int64_t v_token_stride, uint8_t* cache,
    int64_t num_blocks, int32_t block_size, int32_t num_kv_heads, int32_t head_size,
    const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
    int32_t num_seqs, const float* kv_scales, float sm_scale, uint8_t* o_fp8,
    const float* o_scale, void* o_bf16, float* o_f32, void* workspace, size_t workspace_bytes,
    uint32_t flags, nvfp4_stream_t stream);

/* Dequantize listed cache blocks to bf16 ("FlashInfer NVFP4 KV serving on
 * pre-SM100 GPUs", quick answer: the paged NVFP4 dequantize helper).
 *   block_ids       int32 [num_block_ids]: cache blocks to expand.
 *   kv_scales       device fp32 [2] = {k_scale, v_scale}.
 *   out_bf16        bf16 [num_block_ids][2][num_kv_heads][block_size][head_size]:
 *                   out[i] = bf16_RNE(fl32(xhat * g)) of block block_ids[i].
 * Out-of-range block ids are skipped (output left untouched). */
NVFP4KV_API int nvfp4_dequantize_paged(const uint8_t* cache, int64_t num_blocks, int32_t block_size,
                           int32_t num_kv_heads, int32_t head_size,
                           const int32_t* block_ids, int64_t num_block_ids,
                           const float* kv_scales, void* out_bf16, nvfp4_stream_t stream);

/* FP8-E4M3 KV cache: the comparison format of "FlashInfer backend adds
 * end-to-end NVFP4 KV cache support", review highlights (TPOT of NVFP4 versus
 * FP8 KV at batch 256). Same HND page layout with head_size-byte rows of E4M3
 * codes (one per element, no block scales).
 * nvfp4_fp8kv_quantize_append_paged: arguments, slot rules, status bits and
 * errors of nvfp4_quantize_append_paged; each element is stored as
 * E4M3 RNE satfinite(fl32(x / g)), g = *k_scale or *v_scale.
 * nvfp4_fp8kv_paged_attention: arguments, workspace (the same
 * nvfp4_paged_attention_workspace_size), flags, outputs and errors of
 * nvfp4_paged_attention_ex, reading the FP8 cache with xhat = E4M3(code) * g. */
NVFP4KV_API int nvfp4_fp8kv_quantize_append_paged(
    const void* k, const void* v, int64_t k_token_stride, int64_t v_token_stride,
    int64_t num_tokens, int32_t num_kv_heads, int32_t head_size, uint8_t* cache,
    int64_t num_blocks, int32_t block_size, const int64_t* slot_mapping, const float* k_scale,
    const float* v_scale, uint32_t* device_status, nvfp4_stream_t stream);
NVFP4KV_API int nvfp4_fp8kv_paged_attention(
    const void* q, int64_t q_token_stride, int64_t num_q_tokens, int32_t num_q_heads,
    const uint8_t* cache, int64_t num_blocks, int32_t block_size, int32_t num_kv_heads,
    int32_t head_size, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, const int32_t* qo_indptr, int32_t num_seqs, int32_t max_q_len,
    const float* kv_scales, float sm_scale, uint8_t* o_fp8, const float* o_scale,
    void* o_bf16, float* o_f32, void* workspace, size_t workspace_bytes, uint32_t flags,
    nvfp4_stream_t stream);

/* Activation quantizer for NVFP4 GEMMs ("Move NVFP4 GEMM management into
 * NvFp4LinearKernel", flashinfer.py and the CUTLASS linear kernel:
 * scaled_fp4_quant(x, input_global_scale_inv, is_sf_swizzled_layout=True),
 * swizzle_blockscale). Same group codec as the KV cache rows with the global
 * scale g = fl32(1 / *global_scale_inv).
 *   x               bf16 [rows][cols] with row stride row_stride (elements,
 *                   a multiple of 8, >= cols), 16-byte aligned; cols % 16 == 0.
 *   global_scale_inv device fp32 scalar (finite, > 0).
 *   out_fp4         uint8 [rows][cols/2]: E2M1 pairs, element 2j in the low
 *                   nibble of byte j; 8-byte aligned.
 *   out_sf          E4M3 scales, nvfp4_activation_sf_bytes(rows, cols,
 *                   swizzled) bytes. swizzled == 0: [rows][cols/16]. Else rows
 *                   padded to a multiple of 128 and scale columns to a multiple
 *                   of 4, 512-byte tiles of 128 rows x 4 scale columns, tile
 *                   (r/128, c/4) at ((r/128)*(padded columns/4) + c/4)*512,
 *                   scale (r, c) inside it at (r%32)*16 + ((r%128)/32)*4 + c%4;
 *                   padding bytes are written as 0.
 * rows == 0 is a no-op returning NVFP4_OK. */
NVFP4KV_API size_t nvfp4_activation_sf_bytes(int64_t rows, int64_t cols, int swizzled);
NVFP4KV_API int nvfp4_quantize_activation(const void* x, int64_t rows, int64_t cols,
                                          int64_t row_stride, const float* global_scale_inv,
                                          uint8_t* out_fp4, uint8_t* out_sf, int swizzled,
                                          nvfp4_stream_t stream);

/* Paged attention that allocates nothing and takes no workspace. The pages
 * this library follows have no counterpart: it exists for callers that
 * cannot provide the scratch memory nvfp4_paged_attention asks for, such as
 * code handed only its input and output buffers by a host framework (a
 * plugin or callback interface with no workspace hook), or code running
 * while all device memory is owned by an allocator it may not draw from.
 * Arguments and results are those of nvfp4_paged_attention without
 * `workspace` / `workspace_bytes`; the caller still provides every input and
 * output buffer.
 * Scratch: one fixed array of NVFP4_NOALLOC_SCRATCH_BYTES bytes in device
 * memory, defined inside the library; every GPU that loads the library keeps
 * it until the process exits. Sizes whose workspace
 * (nvfp4_paged_attention_workspace_size) exceeds it return
 * NVFP4_ERR_WORKSPACE. The first call on a device looks up the array's
 * device address on that device (make that first call before any stream
 * capture; the look-up is repeated if the device's context is ever
 * re-created). Each call clears the array's arrival counters on `stream`
 * first; its status word is sticky across calls, like a workspace's, and is
 * read (and optionally cleared) with nvfp4_paged_attention_noalloc_status.
 * All calls share the one array, so calls that may overlap on the GPU
 * (unordered streams) race and must not be made. The call never calls
 * cudaMalloc, cudaFree or any allocating routine. */
#define NVFP4_NOALLOC_SCRATCH_BYTES ((size_t)12 << 20)
NVFP4KV_API int nvfp4_paged_attention_noalloc(
    const void* q, int64_t q_token_stride, int64_t num_q_tokens, int32_t num_q_heads,
    const uint8_t* cache, int64_t num_blocks, int32_t block_size, int32_t num_kv_heads,
    int32_t head_size, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, const int32_t* qo_indptr, int32_t num_seqs, int32_t max_q_len,
    const float* kv_scales, float sm_scale, uint8_t* o_fp8, const float* o_scale,
    void* o_bf16, float* o_f32, nvfp4_stream_t stream);

/* nvfp4_read_device_status for the status word of the allocation-free
 * entry point's scratch array on the current device (same synchronization,
 * clearing and return codes). */
NVFP4KV_API int nvfp4_paged_attention_noalloc_status(uint32_t* host_bits, int clear,
                                                     nvfp4_stream_t stream);

/* Device status read-back (the status reporting of the method statement's
 * C ABI; the pages raise errors at start-up only). Copies the 4-byte device
 * status word at `status_word` (a workspace's first 4 bytes, or the word given
 * to nvfp4_quantize_append_paged as device_status) to the host after the work
 * already enqueued on `stream`, SYNCHRONIZES the stream, optionally clears the
 * word (clear != 0, enqueued on `stream`), and stores the bits in *host_bits
 * (may be NULL). Returns NVFP4_ERR_DEVICE_TIMEOUT if NVFP4_DEV_TIMEOUT is set,
 * else NVFP4_ERR_DEVICE_BOUNDS if any of NVFP4_DEV_BAD_SLOT / _BAD_BLOCK /
 * _BAD_QLEN is set, else NVFP4_OK (or a CUDA / argument error). Not for use
 * inside stream capture. */
NVFP4KV_API int nvfp4_read_device_status(const uint32_t* status_word, uint32_t* host_bits,
                                         int clear, nvfp4_stream_t stream);

/* The status code nvfp4_read_device_status returns for a set of NVFP4_DEV_*
 * bits. Pure host function. */
NVFP4KV_API int nvfp4_status_from_bits(uint32_t bits);

/* Self-test of the kernels' bounded waits (no counterpart in the pages; the
 * failure-detection contract above). Launches one block that arms a
 * shared-memory barrier for 16 bytes that no copy will deliver and waits on it
 * with at most `polls` polls (1 .. 2^24); when the wait gives up it ORs
 * NVFP4_DEV_TIMEOUT into the device word *status_word and returns. Nothing is
 * in flight when the block exits, so the context stays usable. */
NVFP4KV_API int nvfp4_wait_timeout_probe(uint32_t* status_word, int32_t polls,
                                         nvfp4_stream_t stream);

/* Static description of a status code. */
NVFP4KV_API const char* nvfp4_status_string(int status);

/* Text of the CUDA error behind the calling thread's most recent
 * NVFP4_ERR_CUDA ("no error" if none). Static string, not owned by caller. */
NVFP4KV_API const char* nvfp4_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4KV_H_ */
