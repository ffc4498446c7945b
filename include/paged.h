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
typedef struct CUevent_st* pa_event_t;   /* same type as cudaEvent_t */

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,     /* null pointer, negative size, bad head ratio, misaligned pointer */
  PA_ERR_UNSUPPORTED = 2, /* head_dim/block_size/group size/num_seqs outside what is compiled */
  PA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  PA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than pa_decode_workspace_size() */
  PA_ERR_OUT_OF_BLOCKS = 5 /* block manager: not enough free blocks (nothing was changed) */
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
 * shape with the largest grid (one CTA per SM; it depends on the device's SM
 * count, not on the context lengths).  A call with max_ctas > 0 needs less:
 * the workspace of a grid of n CTAs is enough for it.  Returns 0 for invalid
 * or unsupported arguments.
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
 * One kernel launch: every (sequence, kv-head) context is cut into 16-token
 * chunks that are spread evenly over a persistent grid; a context split
 * across warps is merged by log-sum-exp inside the same launch (the last
 * warp to finish its part merges; no warp waits for another).
 *
 * max_context_len: an upper bound on context_lens (used to size the launch).
 * workspace: device buffer, 16-byte aligned, owned by the caller, of at
 *   least pa_decode_workspace_size() bytes (or the size for the capped grid
 *   when max_ctas > 0; PA_ERR_WORKSPACE if smaller).  It must be ZERO-FILLED
 *   before its first use (cudaMemset once): it holds the merge's ticket
 *   counters, which every call leaves at zero again, also when a wait gave
 *   up (PA_ERRF_TIMEOUT).  The rest is scratch.  Calls that overlap on the
 *   GPU must use different workspaces.
 * max_ctas: 0 = one CTA per SM (default); n > 0 caps the grid at n CTAs
 *   (fewer, longer per-warp runs -> fewer split partitions).  The result is
 *   the same attention for every choice, up to fp32 rounding order.
 * Supported: head_dim in {64, 128}; block_size in {8, 16, 32, 64};
 *   num_heads/num_kv_heads in {1, 2, 4, 8}; num_kv_heads < 32768.  One
 *   launch takes at most 16384 sequences (its per-sequence prefix table, 4
 *   bytes a sequence, lives in shared memory); a larger batch runs as
 *   several launches of up to 16384 sequences, in order on `stream`, sharing
 *   the workspace.  Per launch, sequences * num_kv_heads *
 *   ceil(max_context_len/16) < 2^31 (PA_ERR_UNSUPPORTED otherwise).
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
 * pa_decode_step_host_pipelined -- pa_decode_step_host for a loop of decode
 * steps, with each step's copies overlapping the neighbouring steps' kernels.
 * Three streams take part:
 *   in_stream   the copy h_inputs -> d_inputs, then event inputs_ready;
 *   stream      append and decode into d_out, after inputs_ready and after
 *               output_free (the previous copy out of this d_out); then
 *               events inputs_free and output_ready;
 *   out_stream  the copy d_out -> h_out after output_ready, then event
 *               output_free.
 * The caller keeps two sets of {d_inputs (256-byte aligned,
 * pa_step_inputs_layout() bytes), d_out, inputs_ready, inputs_free,
 * output_ready, output_free} and passes them in turn: step i uses set i % 2.
 * A set's input copy waits only until the kernels that last read its
 * d_inputs (two steps earlier) are done, so it runs while step i-1 computes;
 * its output copy runs while step i+1 computes.  The events are the
 * caller's (e.g. cudaEventCreateWithFlags(..., cudaEventDisableTiming)); a
 * never-recorded event counts as complete, so the first steps start at once.
 * The copies overlap the kernels only when the three streams are distinct;
 * the results are the same either way.  h_out holds step i's output once
 * output_free of step i has completed (cudaEventSynchronize, or a
 * cudaStreamWaitEvent before a consumer); h_inputs must stay unchanged until
 * inputs_ready has completed, so alternate two host buffers as well when they
 * are refilled every step.  Errors as for pa_decode_step_host; PA_ERR_INVALID
 * for a NULL event.
 */
PA_API pa_status pa_decode_step_host_pipelined(const void* h_inputs, void* d_inputs, void* h_out, void* d_out,
                                               void* k_cache, void* v_cache, int num_seqs, int max_blocks_per_seq,
                                               int max_context_len, float scale, int num_heads, int num_kv_heads,
                                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                                               void* workspace, size_t workspace_bytes, int32_t* err_flags,
                                               pa_stream_t stream, pa_stream_t in_stream, pa_stream_t out_stream,
                                               pa_event_t inputs_ready, pa_event_t inputs_free,
                                               pa_event_t output_ready, pa_event_t output_free);

/*
 * pa_decode_static -- pa_decode for callers that cannot allocate device
 * memory: a plugin whose host application owns every device allocation and
 * hands it only input and output buffers, code under an allocation policy
 * that forbids cudaMalloc on its path (a thread that must never block on an
 * allocator, a fixed memory budget), or a binding with no device allocator.
 * The pages have no counterpart of this entry point; it exists for such
 * callers.  It enqueues kernels, so call it from an ordinary host thread
 * (never from a host function enqueued on a stream, where CUDA calls are
 * not allowed).
 *
 * Same arguments and result as pa_decode, minus the workspace: the scratch
 * is a 10 MiB array inside the library's device image, reserved on every
 * GPU where the library's module is loaded, until the process exits.  The
 * scratch a call needs is that of the grid it launches: every supported
 * shape fits on a GPU of up to 148 SMs (a B200); on a larger GPU a shape
 * that does not fit returns PA_ERR_WORKSPACE (see pa_last_error), and
 * max_ctas > 0 shrinks the grid and its scratch.  Argument errors return
 * PA_ERR_INVALID / PA_ERR_UNSUPPORTED before any CUDA call.  All calls on one
 * GPU share the array, which keeps what the last call left: calls that can
 * run at the same time on that GPU race and give wrong results, so
 * serialise them.  The first call in a CUDA context sets the array up: it
 * looks up its device address (cudaGetSymbolAddress) and zeroes the merge's
 * ticket counters with cudaMemsetAsync on `stream` (every call leaves them
 * at zero again).  Make that first call before any stream capture on that
 * device.  Nothing is allocated or freed.
 */
PA_API pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int num_seqs, int max_context_len, float scale, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype, int max_ctas,
                           int32_t* err_flags, pa_stream_t stream);

/*
 * pa_prefill -- multi-token paged attention: several new tokens per sequence
 * (a prompt, a chunk of one, or speculative tokens) attend causally over the
 * paged cache (the ops-transformer page's call with a [batch, heads, seq_len,
 * head_dim] query).  Sequence s owns query rows cu_q_lens[s] ..
 * cu_q_lens[s+1]-1 of q/out [total_q][num_heads][head_dim]; those n tokens
 * are the LAST n of its context_lens[s] cached tokens (append them with
 * pa_reshape_and_cache first), so row i (position ctx-n+i) attends to cached
 * positions 0..ctx-n+i.  cu_q_lens: int32 device array [num_seqs+1],
 * non-decreasing, cu_q_lens[0] = 0.  max_q_len bounds the per-sequence n
 * (sizes the launch).  n > ctx or a context above the bound is clamped and
 * flags PA_ERRF_CONTEXT; offsets outside [0, total_q] skip the sequence and
 * flag it.  No workspace.  Same head_dim / block_size support as pa_decode;
 * num_seqs and num_heads <= 65535.  scale must be positive (else
 * PA_ERR_UNSUPPORTED: the kernel takes row maxima on unscaled scores).  Runs
 * on the tcgen05 tensor cores with tensor-memory accumulators.
 */
PA_API pa_status pa_prefill(void* out, const void* q, const int32_t* cu_q_lens, int total_q, int max_q_len,
                     const void* k_cache, const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                     const int32_t* context_lens, int num_seqs, int max_context_len, float scale, int num_heads,
                     int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                     int32_t* err_flags, pa_stream_t stream);

/* The same operation on the legacy mma.sync tensor-core path (kept as the
 * reference point the tcgen05 kernel is measured against). */
PA_API pa_status pa_prefill_mma(void* out, const void* q, const int32_t* cu_q_lens, int total_q, int max_q_len,
                         const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int max_context_len,
                         float scale, int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int64_t num_blocks, pa_dtype dtype, int32_t* err_flags, pa_stream_t stream);

/*
 * pa_copy_blocks -- copy-on-write copies inside the paged pools ("【infra之路】10-
 * PagedAttention 与 KV Cache 管理", section 4.3: shared prefixes and beams share
 * physical blocks until one writes).  For every pair i, block
 * block_pairs[2i+1] of k_cache and of v_cache becomes a bit-exact copy of
 * block block_pairs[2i] (all kv-heads, all rows).  block_pairs: int64 device
 * array of 2*num_pairs ids.  A block may not be both a source and a
 * destination in one call.  An id outside [0, num_blocks) skips that pair and
 * sets PA_ERRF_BLOCK_RANGE.
 */
PA_API pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_pairs, int64_t num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                         int32_t* err_flags, pa_stream_t stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools with the same block
 * size in bytes (block_bytes = num_kv_heads*block_size*head_dim*2), e.g. a
 * device pool and a pinned host pool (the tutorial's section 4.3 preemption:
 * swap a request's blocks out to CPU memory and back).  For every pair i,
 * dst_pool block block_pairs[2i+1] = src_pool block block_pairs[2i].  Call once
 * for the K pool and once for the V pool.  Each pool, and block_pairs, must be
 * device memory or pinned (page-locked) host memory; anything else returns
 * PA_ERR_INVALID without launching.  Out-of-range ids are skipped and flagged
 * (PA_ERRF_BLOCK_RANGE).
 */
PA_API pa_status pa_swap_blocks(const void* src_pool, int64_t src_num_blocks, void* dst_pool, int64_t dst_num_blocks,
                         int64_t block_bytes, const int64_t* block_pairs, int64_t num_pairs, int32_t* err_flags,
                         pa_stream_t stream);

/*
 * Block manager (host memory, not thread-safe): the pool lifecycle of
 * "PagedAttention：KV Cache 的分页革命" (section Runtime 如何管理 KV Block: a pool
 * of fixed-size blocks, a free block taken when a step needs space, the page
 * table updated, blocks returned when a request ends) with the per-request
 * block tables of the tutorial (section 3.3) and shared, copy-on-write blocks
 * (section 4.3).  Free blocks are handed out lowest id first.  All functions
 * return PA_ERR_INVALID for an unknown or duplicate sequence id.
 */
typedef struct pa_block_manager pa_block_manager;

/* A manager of blocks 0..num_blocks-1, all free; NULL on bad arguments or no memory. */
PA_API pa_block_manager* pa_bm_create(int64_t num_blocks, int block_size);
PA_API void pa_bm_destroy(pa_block_manager* m);
PA_API int64_t pa_bm_num_free_blocks(const pa_block_manager* m);

/* A new sequence holding num_tokens tokens (positions 0..num_tokens-1). */
PA_API pa_status pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id, int64_t num_tokens);

/* child shares all of parent's blocks (beam search / shared prefix): the
 * table is copied, the KV is not. */
PA_API pa_status pa_bm_fork(pa_block_manager* m, int64_t parent, int64_t child);

/* Room for one more token: returns its slot (block_id*block_size + offset).
 * A new block is taken when the last one is full; if the last block is shared,
 * it is replaced by a fresh block and (*cow_src, *cow_dst) name the copy the
 * caller must make with pa_copy_blocks before writing (else both are -1). */
PA_API pa_status pa_bm_append_slot(pa_block_manager* m, int64_t seq_id, int64_t* slot, int64_t* cow_src,
                            int64_t* cow_dst);

/* Release a sequence; blocks no other sequence holds become free. */
PA_API pa_status pa_bm_free_sequence(pa_block_manager* m, int64_t seq_id);

/* Tokens held by the sequence, or -1 if unknown. */
PA_API int64_t pa_bm_context_len(const pa_block_manager* m, int64_t seq_id);

/* The sequence's block table into table[0..max_blocks) (-1 after the last
 * block); *num_blocks gets its length (PA_ERR_INVALID if it exceeds max_blocks). */
PA_API pa_status pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* table, int max_blocks,
                            int* num_blocks);

/* Free blocks that appending one more token to each listed sequence takes
 * (admission control, the tutorial's section 6 scheduler): one per sequence
 * whose last block is full, plus, for a partly filled last block held by r
 * sequences of which k are listed, min(k, r-1) copies (the last writer keeps
 * the block).  Exactly what pa_bm_prepare_decode on the same batch takes;
 * -1 on bad ids. */
PA_API int64_t pa_bm_blocks_needed_to_append(const pa_block_manager* m, const int64_t* seq_ids, int num_seqs);

/* One decode step for a batch: appends one token to each sequence and writes
 * the kernels' inputs (host arrays): block_tables [num_seqs][max_blocks_per_seq],
 * context_lens [num_seqs] (counting the new token), slot_mapping [num_seqs],
 * and the copy-on-write pairs cow_pairs [2*num_seqs] (*num_cow_pairs of them).
 * All-or-nothing: PA_ERR_OUT_OF_BLOCKS or PA_ERR_INVALID leaves the manager
 * unchanged. */
PA_API pa_status pa_bm_prepare_decode(pa_block_manager* m, const int64_t* seq_ids, int num_seqs, int max_blocks_per_seq,
                               int32_t* block_tables, int32_t* context_lens, int64_t* slot_mapping, int64_t* cow_pairs,
                               int64_t* num_cow_pairs);

/* Move a sequence from manager `from` to manager `to` (e.g. device pool ->
 * host pool on preemption, and back): fresh blocks are taken in `to`, the
 * blocks in `from` are released, and pairs[2i], pairs[2i+1] = (block in
 * `from`, block in `to`) for pa_swap_blocks.  Shared blocks are copied, not
 * shared, in `to`. */
PA_API pa_status pa_bm_swap_sequence(pa_block_manager* from, pa_block_manager* to, int64_t seq_id, int64_t* pairs,
                              int64_t max_pairs, int64_t* num_pairs);

/*
 * pa_selftest_wait_timeout -- checks, on the device, the bounded barrier wait
 * that every kernel above relies on (the pages have no counterpart).  One
 * CTA waits on two shared-memory barriers that nothing ever completes, one
 * with each wait flavour the kernels use (plain probe loop; suspending
 * probe), each limited to `limit_ns` nanoseconds (1 .. 1e8).  Each wait must
 * give up, after which PA_ERRF_TIMEOUT is OR-ed into err_flags[0] (plain)
 * and err_flags[1] (suspending), int32 device words owned by the caller, and
 * the kernel returns: no trap, the context stays usable.  Asynchronous on
 * `stream`; PA_ERR_INVALID for a NULL err_flags or a limit out of range.
 */
PA_API pa_status pa_selftest_wait_timeout(uint64_t limit_ns, int32_t* err_flags, pa_stream_t stream);

/*
 * pa_selftest_exp2 -- evaluates, on the device, the polynomial 2^x that the
 * multi-token kernel runs on the FMA pipe for part of its softmax
 * exponentials, beside CUDA's exp2f on the same inputs (the pages have no
 * counterpart): y_poly[i] = polynomial 2^x[i] (the scalar form for even i,
 * the packed two-input form for odd i), y_ref[i] = exp2f(x[i]) for i < n;
 * float32 device arrays owned by the caller.  The polynomial is
 * specified for x < 127 with relative error below 1.0e-4, and returns 2^-125
 * for x <= -125 (including -inf).  Asynchronous on `stream`; PA_ERR_INVALID
 * for n < 0 or a NULL array.
 */
PA_API pa_status pa_selftest_exp2(const float* x, float* y_poly, float* y_ref, int64_t n, pa_stream_t stream);

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
