// One whole decode step driven from host memory: the step's inputs are
// copied host -> device, the new tokens' K/V are appended to the paged
// caches, paged decode attention runs, and the output is copied back --
// all enqueued on one stream, in the order of the tutorial's section 1.2
// ("【infra之路】10-PagedAttention 与 KV Cache 管理": append, then attend).
//
// The KV caches and the workspace stay resident on the device; only the
// per-step tensors cross PCIe.  They travel packed in one staging buffer
// (layout from pa_step_inputs_layout), so a step costs one host-to-device
// and one device-to-host copy.
//
// pa_decode_step_host_pipelined is the same step for a serving loop: its
// host-to-device copy runs on a second stream, into one of two staging
// buffers used in turn, so that it overlaps the previous step's kernels
// instead of preceding them; its device-to-host copy runs on a third, out of
// one of two output buffers, so that it overlaps the next step's kernels.
// A copy between two kernels on one stream also ends the programmatic-launch
// overlap of their start and end, which costs more than the copy itself.
#include "pa_device.cuh"
#include "pa_host.h"

namespace {
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

extern "C" size_t pa_step_inputs_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                        int max_blocks_per_seq, size_t offsets[6]) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0 || !offsets)
    return 0;
  const size_t S = static_cast<size_t>(num_seqs);
  const size_t sizes[6] = {
      S * num_heads * head_dim * 2,           // q
      S * num_kv_heads * head_dim * 2,        // key
      S * num_kv_heads * head_dim * 2,        // value
      S * sizeof(int64_t),                    // slot_mapping
      S * max_blocks_per_seq * sizeof(int32_t),  // block_tables
      S * sizeof(int32_t),                    // context_lens
  };
  size_t off = 0;
  for (int i = 0; i < 6; ++i) {
    offsets[i] = off;
    off = align256(off + sizes[i]);
  }
  return off;
}

namespace {

// Append and decode from a staging buffer already on the device (both on `stream`).
pa_status step_kernels(void* d_inputs, const size_t off[6], void* d_out, void* k_cache, void* v_cache, int num_seqs,
                       int max_blocks_per_seq, int max_context_len, float scale, int num_heads, int num_kv_heads,
                       int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype, void* workspace,
                       size_t workspace_bytes, int32_t* err_flags, pa_stream_t stream) {
  uint8_t* d = static_cast<uint8_t*>(d_inputs);
  const void* d_q = d + off[0];
  const void* d_key = d + off[1];
  const void* d_value = d + off[2];
  const int64_t* d_slots = reinterpret_cast<const int64_t*>(d + off[3]);
  const int32_t* d_tables = reinterpret_cast<const int32_t*>(d + off[4]);
  const int32_t* d_ctx = reinterpret_cast<const int32_t*>(d + off[5]);
  pa_status st = pa_reshape_and_cache(d_key, d_value, k_cache, v_cache, d_slots, num_seqs, num_kv_heads, head_dim,
                                      block_size, num_blocks, dtype, err_flags, stream);
  if (st != PA_OK) return st;
  return pa_decode(d_out, d_q, k_cache, v_cache, d_tables, max_blocks_per_seq, d_ctx, num_seqs, max_context_len,
                   scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype, workspace,
                   workspace_bytes, 0, err_flags, stream);
}

}  // namespace

extern "C" pa_status pa_decode_step_host(const void* h_inputs, void* d_inputs, void* h_out, void* d_out,
                                         void* k_cache, void* v_cache, int num_seqs, int max_blocks_per_seq,
                                         int max_context_len, float scale, int num_heads, int num_kv_heads,
                                         int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                                         void* workspace, size_t workspace_bytes, int32_t* err_flags,
                                         pa_stream_t stream) {
  pa::DecodePlan plan;  // the decode's argument checks, before anything is enqueued
  const pa_status pst = pa::plan_decode(num_seqs, max_blocks_per_seq, max_context_len, scale, num_heads,
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype, 0, &plan);
  if (pst != PA_OK) return pst;
  if (num_seqs == 0) return PA_OK;
  size_t off[6];
  const size_t total = pa_step_inputs_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq, off);
  if (total == 0) return PA_ERR_INVALID;
  if (!h_inputs || !d_inputs || !h_out || !d_out) return PA_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(d_inputs) & 255u) return PA_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(d_inputs, h_inputs, total, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host: host-to-device copy", e);
  const pa_status st = step_kernels(d_inputs, off, d_out, k_cache, v_cache, num_seqs, max_blocks_per_seq,
                                    max_context_len, scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                    dtype, workspace, workspace_bytes, err_flags, stream);
  if (st != PA_OK) return st;
  const size_t out_bytes = static_cast<size_t>(num_seqs) * num_heads * head_dim * 2;
  e = cudaMemcpyAsync(h_out, d_out, out_bytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host: device-to-host copy", e);
  return PA_OK;
}

extern "C" pa_status pa_decode_step_host_pipelined(const void* h_inputs, void* d_inputs, void* h_out, void* d_out,
                                                   void* k_cache, void* v_cache, int num_seqs, int max_blocks_per_seq,
                                                   int max_context_len, float scale, int num_heads, int num_kv_heads,
                                                   int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                                                   void* workspace, size_t workspace_bytes, int32_t* err_flags,
                                                   pa_stream_t stream, pa_stream_t in_stream, pa_stream_t out_stream,
                                                   pa_event_t inputs_ready, pa_event_t inputs_free,
                                                   pa_event_t output_ready, pa_event_t output_free) {
  pa::DecodePlan plan;  // the decode's argument checks, before anything is enqueued
  const pa_status pst = pa::plan_decode(num_seqs, max_blocks_per_seq, max_context_len, scale, num_heads,
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype, 0, &plan);
  if (pst != PA_OK) return pst;
  if (num_seqs == 0) return PA_OK;
  size_t off[6];
  const size_t total = pa_step_inputs_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq, off);
  if (total == 0) return PA_ERR_INVALID;
  if (!h_inputs || !d_inputs || !h_out || !d_out) return PA_ERR_INVALID;
  if (!inputs_ready || !inputs_free || !output_ready || !output_free) return PA_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(d_inputs) & 255u) return PA_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t is = reinterpret_cast<cudaStream_t>(in_stream);
  cudaStream_t os = reinterpret_cast<cudaStream_t>(out_stream);
  cudaEvent_t in_ready = reinterpret_cast<cudaEvent_t>(inputs_ready);
  cudaEvent_t in_free = reinterpret_cast<cudaEvent_t>(inputs_free);
  cudaEvent_t out_ready = reinterpret_cast<cudaEvent_t>(output_ready);
  cudaEvent_t out_free = reinterpret_cast<cudaEvent_t>(output_free);
  // Input copy: once the kernels of the last step that read this staging
  // buffer are done (not the previous step's: it overlaps them).
  cudaError_t e = cudaStreamWaitEvent(is, in_free, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d_inputs, h_inputs, total, cudaMemcpyHostToDevice, is);
  if (e == cudaSuccess) e = cudaEventRecord(in_ready, is);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host_pipelined: host-to-device copy", e);
  // Kernels: after this step's inputs and after the copy out of this d_out
  // two steps back.  Both waits come before the append, so nothing sits
  // between the append and the decode, which overlap through the
  // programmatic launch.
  e = cudaStreamWaitEvent(s, in_ready, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, out_free, 0);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host_pipelined: stream wait", e);
  const pa_status st = step_kernels(d_inputs, off, d_out, k_cache, v_cache, num_seqs, max_blocks_per_seq,
                                    max_context_len, scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                    dtype, workspace, workspace_bytes, err_flags, stream);
  if (st != PA_OK) return st;
  e = cudaEventRecord(in_free, s);  // this buffer's inputs are consumed
  if (e == cudaSuccess) e = cudaEventRecord(out_ready, s);
  // Output copy, off the compute stream: the next step's kernels start
  // without waiting for it.
  if (e == cudaSuccess) e = cudaStreamWaitEvent(os, out_ready, 0);
  if (e == cudaSuccess) {
    const size_t out_bytes = static_cast<size_t>(num_seqs) * num_heads * head_dim * 2;
    e = cudaMemcpyAsync(h_out, d_out, out_bytes, cudaMemcpyDeviceToHost, os);
  }
  if (e == cudaSuccess) e = cudaEventRecord(out_free, os);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host_pipelined: device-to-host copy", e);
  return PA_OK;
}
