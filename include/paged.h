/*
 * libpaged -- PagedAttention decode and KV-cache append for NVIDIA B200
 * (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 * Operations (page titles as published):
 *  - pa_reshape_and_cache: the append step -- "the current token's K/V are
 *    appended at the end of the cache" ("PagedAttention：KV Cache 的分页革命",
 *    section 为什么 KV Cache 会爆显存; "【infra之路】10-PagedAttention 与
 *    KV Cache 管理", section 1.2), with the slot of each token given by the
 *    block table (same tutorial, section 3.3).
 *  - pa_decode: single-query attention softmax(q K^T * scale) V of each
 *    sequence over its cached tokens (tutorial section 1.1), where K/V are
 *    read block by block through the per-sequence block table (tutorial
 *    sections 3.2-3.4), split over the context and merged by log-sum-exp
 *    (the FlashDecoding-style split named in the tutorial's section 8, Q2).
 *
 * Layouts (row-major, element = fp16 or bf16 as given by `dtype`):
 *   k_cache, v_cache : [num_blocks][num_kv_heads][block_size][head_dim]
 *   key, value       : [num_tokens][num_kv_heads][head_dim]
 *   q, out           : [num_seqs][num_heads][head_dim]
 *   block_tables     : int32 [num_seqs][max_blocks_per_seq]; logical block i
 *                      of sequence s is physical block block_tables[s][i]
 *   context_lens     : int32 [num_seqs]; tokens of sequence s INCLUDING the
 *                      one appended in this step (its position is ctx-1)
 *   slot_mapping     : int64 [num_tokens]; slot = block_id*block_size + offset
 * q-head h reads kv-head h / (num_heads / num_kv_heads).
 *
 * Ownership: the caller allocates every buffer (device memory unless noted)
 * and keeps ownership; the library allocates nothing and retains no pointer
 * after a call returns.  All calls are asynchronous on `stream` (NULL = the
 * legacy default stream) and never synchronize.
 *
 * Errors: host-side argument checks return PA_ERR_INVALID /
 * PA_ERR_UNSUPPORTED / PA_ERR_WORKSPACE before anything is launched; a
 * launch failure returns PA_ERR_CUDA.  Bad values that only the device sees
 * (an out-of-range slot or block id, a context length that does not fit)
 * never fault: the access is skipped and a PA_ERRF_* bit is OR-ed into
 * *err_flags (when err_flags is non-NULL; the caller zeroes it and reads it
 * after synchronizing).
 */
#ifndef LIBPAGED_PAGED_H
#define LIBPAGED_PAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef struct CUstream_st* pa_stream_t; /* same type as cudaStream_t */

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,     /* null pointer, negative size, bad head ratio, misaligned pointer */
  PA_ERR_UNSUPPORTED = 2, /* head_dim/block_size/group size/num_seqs outside what is compiled */
  PA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  PA_ERR_WORKSPACE = 4    /* workspace missing or smaller than pa_decode_workspace_size() */
} pa_status;

/* Device-side error bits (OR-ed into *err_flags). */
#define PA_ERRF_SLOT_RANGE (1u << 0)  /* append: slot >= num_blocks*block_size; token skipped */
#define PA_ERRF_BLOCK_RANGE (1u << 1) /* decode: table entry outside [0, num_blocks); that chunk of 16 tokens is skipped */
#define PA_ERRF_CONTEXT (1u << 2)     /* decode: context_lens[s] < 0, > max_context_len or > max_blocks_per_seq*block_size; clamped */
#define PA_ERRF_TIMEOUT (1u << 3)     /* decode: a pipeline wait gave up after ~1 s; that warp's outputs are not written */

/*
 * pa_reshape_and_cache -- write the K/V of `num_tokens` new tokens into the
 * paged caches.  For token n with s = slot_mapping[n] >= 0, and every kv-head
 * h:  k_cache[s / block_size][h][s % block_size][:] = key[n][h][:]  (same for
 * value/v_cache).  s < 0 marks a padding token and is skipped; s >=
 * num_blocks*block_size is skipped and sets PA_ERRF_SLOT_RANGE.  The copy is
 * bit-exact.  Two tokens with the same slot in one call: undefined which wins.
 * head_dim in {64, 128}; block_size in {8, 16, 32, 64}; all data pointers
 * 16-byte aligned.
 */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                               int32_t* err_flags, pa_stream_t stream);

/*
 * Bytes of device workspace pa_decode needs on the CURRENT device for this
 * shape (it depends on the device's SM count, not on the context lengths).
 * Returns 0 for invalid or unsupported arguments.
 */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                int max_context_len);

/*
 * pa_decode -- out[s][h][:] = softmax(scale * q[s][h] . K_s^T) V_s, where K_s,
 * V_s are the first context_lens[s] tokens of sequence s gathered through
 * block_tables[s] from kv-head h / (num_heads/num_kv_heads).  Only the first
 * ceil(ctx/block_size) table entries of a row are read; the rest may hold
 * anything.  context_lens[s] == 0 writes zeros.  Accumulation is fp32; the
 * result is rounded to `dtype`.
 *
 * max_context_len: an upper bound on context_lens (used to size the launch).
 * workspace: device buffer of at least pa_decode_workspace_size() bytes,
 *   16-byte aligned, owned by the caller; its contents need no
 *   initialisation and are scratch after the call.  Calls that overlap on the
 *   GPU must use different workspaces.
 * max_ctas: 0 = one CTA per SM (default); n > 0 caps the grid at n CTAs
 *   (fewer, longer per-warp runs -> fewer split partitions).  The result is
 *   the same attention for every choice, up to fp32 rounding order.
 * Supported: head_dim in {64, 128}; block_size in {8, 16, 32, 64};
 *   num_heads/num_kv_heads in {1, 2, 4, 8}; 1 <= num_seqs <= 2048;
 *   num_seqs * num_kv_heads * ceil(max_context_len/16) < 2^31.
 */
PA_API pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                    int num_seqs, int max_context_len, float scale, int num_heads, int num_kv_heads,
                    int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype, void* workspace,
                    size_t workspace_bytes, int max_ctas, int32_t* err_flags, pa_stream_t stream);

/*
 * pa_step_inputs_layout -- where each per-step input sits in the packed
 * staging buffer of pa_decode_step_host.  Writes the byte offsets of q, key,
 * value, slot_mapping, block_tables and context_lens (in that order, each
 * 256-byte aligned, layouts as above, one new token per sequence) to
 * offsets[0..5] and returns the buffer's total size (0 for bad arguments).
 */
PA_API size_t pa_step_inputs_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                    int max_blocks_per_seq, size_t offsets[6]);

/*
 * pa_decode_step_host -- one decode step whose per-step inputs live in host
 * memory.  h_inputs holds q, key, value, slot_mapping, block_tables and
 * context_lens packed as pa_step_inputs_layout describes; it is copied in one
 * piece into the caller's device staging buffer d_inputs (same size,
 * 256-byte aligned), then pa_reshape_and_cache and pa_decode run on the
 * resident caches (output in d_out, [num_seqs][num_heads][head_dim]) and the
 * output is copied back into h_out.  Everything is enqueued on `stream` in
 * that order; h_out is valid after the stream is synchronized.  Host buffers
 * should be pinned (page-locked) for the copies to be asynchronous.  Errors
 * are those of the two calls it makes, plus PA_ERR_CUDA for a failed copy.
 */
PA_API pa_status pa_decode_step_host(const void* h_inputs, void* d_inputs, void* h_out, void* d_out, void* k_cache,
                              void* v_cache, int num_seqs, int max_blocks_per_seq, int max_context_len,
                              float scale, int num_heads, int num_kv_heads, int head_dim, int block_size,
                              int64_t num_blocks, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                              int32_t* err_flags, pa_stream_t stream);

/*
 * pa_decode_static -- pa_decode for callers that cannot allocate device
 * memory (code where cudaMalloc is not allowed or not available, such as a
 * host callback, a thread that must never block on an allocator, or a host
 * application that hands a plugin only its input and output buffers).  The
 * pages have no counterpart of this entry point; it exists for such callers.
 *
 * Same arguments and result as pa_decode, minus the workspace: the scratch
 * is a 10 MiB array inside the library's device image, reserved on every
 * GPU that uses this call until the process exits.  A shape that needs more
 * scratch than that (pa_decode_workspace_size) returns PA_ERR_WORKSPACE; on
 * a 148-SM B200 every supported shape fits.  All calls on one GPU share the
 * array: calls that can run at the same time on that GPU race and give wrong
 * results, so serialise them.  The array needs no clearing between calls.
 * The first call on a device looks up the array's address
 * (cudaGetSymbolAddress); make it before any stream capture on that device.
 * Nothing is allocated or freed.
 */
PA_API pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int num_seqs, int max_context_len, float scale, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype, int max_ctas,
                           int32_t* err_flags, pa_stream_t stream);

/* Static, human-readable name of a status code. */
PA_API const char* pa_status_string(pa_status status);

/* Library version, major*10000 + minor*100 + patch. */
PA_API int pa_version(void);

/* Detail of the last PA_ERR_CUDA / PA_ERR_UNSUPPORTED raised on this thread
 * by a failing CUDA step (static thread-local storage; never NULL). */
PA_API const char* pa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBPAGED_PAGED_H */
