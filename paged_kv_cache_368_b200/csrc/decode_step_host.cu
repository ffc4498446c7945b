// One whole decode step driven from host memory: the step's inputs are
// copied host -> device, the new tokens' K/V are appended to the paged
// caches, paged decode attention runs, and the output is copied back --
// all enqueued on one stream, in the order of the tutorial's section 1.2
// ("【infra之路】10-PagedAttention 与 KV Cache 管理": append, then attend).
//
// The KV caches and the workspace stay resident on the device; only the
// per-step tensors cross PCIe.  One cudaMemcpyAsync per tensor (host buffers
// should be pinned for the copies to be asynchronous).
#include "pa_device.cuh"

extern "C" pa_status pa_decode_step_host(const void* h_q, const void* h_key, const void* h_value,
                                         const int64_t* h_slot_mapping, const int32_t* h_block_tables,
                                         const int32_t* h_context_lens, void* h_out, void* d_q, void* d_key,
                                         void* d_value, int64_t* d_slot_mapping, int32_t* d_block_tables,
                                         int32_t* d_context_lens, void* d_out, void* k_cache, void* v_cache,
                                         int num_seqs, int max_blocks_per_seq, int max_context_len, float scale,
                                         int num_heads, int num_kv_heads, int head_dim, int block_size,
                                         int64_t num_blocks, pa_dtype dtype, void* workspace,
                                         size_t workspace_bytes, int32_t* err_flags, pa_stream_t stream) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0)
    return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!h_q || !h_key || !h_value || !h_slot_mapping || !h_block_tables || !h_context_lens || !h_out || !d_q ||
      !d_key || !d_value || !d_slot_mapping || !d_block_tables || !d_context_lens || !d_out)
    return PA_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t S = static_cast<size_t>(num_seqs);
  const size_t q_bytes = S * num_heads * head_dim * 2;
  const size_t kv_bytes = S * num_kv_heads * head_dim * 2;
  struct Copy {
    void* dst;
    const void* src;
    size_t bytes;
  } in[] = {
      {d_key, h_key, kv_bytes},
      {d_value, h_value, kv_bytes},
      {d_slot_mapping, h_slot_mapping, S * sizeof(int64_t)},
      {d_q, h_q, q_bytes},
      {d_block_tables, h_block_tables, S * max_blocks_per_seq * sizeof(int32_t)},
      {d_context_lens, h_context_lens, S * sizeof(int32_t)},
  };
  for (const Copy& c : in) {
    const cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host: host-to-device copy", e);
  }
  pa_status st = pa_reshape_and_cache(d_key, d_value, k_cache, v_cache, d_slot_mapping, num_seqs, num_kv_heads,
                                      head_dim, block_size, num_blocks, dtype, err_flags, stream);
  if (st != PA_OK) return st;
  st = pa_decode(d_out, d_q, k_cache, v_cache, d_block_tables, max_blocks_per_seq, d_context_lens, num_seqs,
                 max_context_len, scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype, workspace,
                 workspace_bytes, 0, err_flags, stream);
  if (st != PA_OK) return st;
  const cudaError_t e = cudaMemcpyAsync(h_out, d_out, q_bytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step_host: device-to-host copy", e);
  return PA_OK;
}
