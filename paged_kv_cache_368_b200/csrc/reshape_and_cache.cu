// Cache append: each new token's K/V row goes to its slot in the paged pools.
//
// "PagedAttention：KV Cache 的分页革命" (section 为什么 KV Cache 会爆显存) and
// "【infra之路】10-PagedAttention 与 KV Cache 管理" (section 1.2) append the
// current token's K/V to the cache every decode step; the tutorial's section
// 3.3 places logical token i in physical block table[i / block_size] at
// offset i % block_size, which the caller folds into a flat slot id.
//
// The operation is a scatter of 16-byte vectors: thread t copies one vector
// of one (token, kv-head, K-or-V) row.  It moves 2 * num_tokens *
// num_kv_heads * head_dim * 2 bytes and is latency bound at decode sizes.
#include "pa_device.cuh"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4* __restrict__ key,
                                                                 const uint4* __restrict__ value,
                                                                 uint4* __restrict__ k_cache,
                                                                 uint4* __restrict__ v_cache,
                                                                 const int64_t* __restrict__ slot_mapping,
                                                                 int64_t num_tokens, int num_kv_heads,
                                                                 int vec_per_row, int block_size,
                                                                 int64_t num_slots, int32_t* err_flags) {
  // Launched with programmatic serialization: wait for the previous grid
  // (which may still read the cache) before writing.
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per_tensor = num_tokens * num_kv_heads * vec_per_row;
  const int64_t total = 2 * per_tensor;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const int64_t r = is_v ? i - per_tensor : i;
    const int v = static_cast<int>(r % vec_per_row);
    const int64_t row = r / vec_per_row;  // token * num_kv_heads + head
    const int h = static_cast<int>(row % num_kv_heads);
    const int64_t n = row / num_kv_heads;
    const int64_t slot = slot_mapping[n];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (v == 0 && h == 0 && !is_v) set_err(err_flags, PA_ERRF_SLOT_RANGE);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * vec_per_row + v;
    if (is_v)
      v_cache[dst] = value[r];
    else
      k_cache[dst] = key[r];
  }
}

}  // namespace pa

namespace {
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                                          const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                                          int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                                          int32_t* err_flags, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID;
  const int vec_per_row = head_dim / 8;
  const int64_t total = 2 * num_tokens * num_kv_heads * vec_per_row;
  const int threads = 256;
  const int64_t blocks64 = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(blocks64 < 65535 ? blocks64 : 65535);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, pa::reshape_and_cache_kernel, static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens, num_kv_heads,
      vec_per_row, block_size, num_blocks * block_size, err_flags);
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching reshape_and_cache_kernel", e);
}
