// Whole-block copies between physical blocks of the paged pools.
//
// "【infra之路】10-PagedAttention 与 KV Cache 管理", section 4.3: requests that
// share a prompt prefix (or beams of one request) point their block tables at
// the same physical blocks and copy a block only when one of them writes to
// it (copy on write); preempted requests have their blocks swapped out to CPU
// memory and back, like an OS swap.  pa_copy_blocks is the copy-on-write copy
// inside the device pools; pa_swap_blocks moves blocks between a device pool
// and a pinned host pool (either direction).
//
// One kernel serves both: for every (src, dst) pair, copy block_bytes from
// src_pool + src*block_bytes to dst_pool + dst*block_bytes with 16-byte
// vectors, a grid-stride over (pair, slab of the block).  HBM-bound for
// device pools (read + write), PCIe-bound when one pool is host memory.
#include <algorithm>

#include "pa_device.cuh"

namespace pa {

__global__ void __launch_bounds__(256) block_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         const int64_t* __restrict__ pairs, int64_t num_pairs,
                                                         int64_t vec_per_block, int64_t src_blocks,
                                                         int64_t dst_blocks, int slabs, int32_t* err_flags) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per_slab = (vec_per_block + slabs - 1) / slabs;
  for (int64_t job = blockIdx.x; job < num_pairs * slabs; job += gridDim.x) {
    const int64_t pair = job / slabs;
    const int slab = static_cast<int>(job - pair * slabs);
    const int64_t s = pairs[2 * pair], d = pairs[2 * pair + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
      if (slab == 0 && threadIdx.x == 0) set_err(err_flags, PA_ERRF_BLOCK_RANGE);
      continue;
    }
    const uint4* from = src + s * vec_per_block;
    uint4* to = dst + d * vec_per_block;
    const int64_t lo = slab * per_slab;
    const int64_t hi = min(vec_per_block, lo + per_slab);
    int64_t i = lo + threadIdx.x;
    for (; i + 3 * 256 < hi; i += 4 * 256) {  // four independent loads in flight
      const uint4 a = from[i], b = from[i + 256], c = from[i + 512], e = from[i + 768];
      to[i] = a;
      to[i + 256] = b;
      to[i + 512] = c;
      to[i + 768] = e;
    }
    for (; i < hi; i += 256) to[i] = from[i];
  }
}

}  // namespace pa

namespace {

// A device-usable address for `p`: device memory, managed memory, or pinned
// (registered) host memory.  Pageable host memory is rejected: a kernel must
// never dereference it.
bool device_view(const void* p, size_t bytes, const void** out) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeUnregistered || a.devicePointer == nullptr) return false;
  if (bytes > 1) {  // the whole range must belong to usable memory
    cudaPointerAttributes b;
    const void* last = static_cast<const char*>(p) + bytes - 1;
    if (cudaPointerGetAttributes(&b, last) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    if (b.type == cudaMemoryTypeUnregistered || b.devicePointer == nullptr) return false;
  }
  *out = a.devicePointer;
  return true;
}

pa_status launch_copy(const void* src, void* dst, const int64_t* pairs, int64_t num_pairs, int64_t block_bytes,
                      int64_t src_blocks, int64_t dst_blocks, int32_t* err_flags, cudaStream_t stream) {
  const int64_t vec = block_bytes / 16;
  const int slabs = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(64, vec / 1024)));
  const int64_t jobs = num_pairs * slabs;
  const int blocks = static_cast<int>(std::min<int64_t>(jobs, 148 * 16));
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, pa::block_copy_kernel, static_cast<const uint4*>(src),
                                           static_cast<uint4*>(dst), pairs, num_pairs, vec, src_blocks, dst_blocks,
                                           slabs, err_flags);
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching block_copy_kernel", e);
}

}  // namespace

extern "C" pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_pairs, int64_t num_pairs,
                                    int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                                    pa_dtype dtype, int32_t* err_flags, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0) return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_pairs) return PA_ERR_INVALID;
  const int64_t block_bytes = int64_t(num_kv_heads) * block_size * head_dim * 2;
  if (block_bytes % 16 || (reinterpret_cast<uintptr_t>(k_cache) & 15) || (reinterpret_cast<uintptr_t>(v_cache) & 15) ||
      (reinterpret_cast<uintptr_t>(block_pairs) & 7))
    return PA_ERR_INVALID;
  // The pair list is usually built on the host: make sure the kernel can read it.
  const void* pairs_d;
  if (!device_view(block_pairs, size_t(num_pairs) * 2 * sizeof(int64_t), &pairs_d))
    return pa::fail(PA_ERR_INVALID, "pa_copy_blocks: block_pairs is not device-accessible memory", cudaSuccess);
  const int64_t* pp = static_cast<const int64_t*>(pairs_d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  pa_status st = launch_copy(k_cache, k_cache, pp, num_pairs, block_bytes, num_blocks, num_blocks, err_flags, s);
  if (st != PA_OK) return st;
  return launch_copy(v_cache, v_cache, pp, num_pairs, block_bytes, num_blocks, num_blocks, err_flags, s);
}

extern "C" pa_status pa_swap_blocks(const void* src_pool, int64_t src_num_blocks, void* dst_pool,
                                    int64_t dst_num_blocks, int64_t block_bytes, const int64_t* block_pairs,
                                    int64_t num_pairs, int32_t* err_flags, pa_stream_t stream) {
  if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || block_bytes <= 0 || block_bytes % 16)
    return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!src_pool || !dst_pool || !block_pairs || src_pool == dst_pool) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(src_pool) & 15) || (reinterpret_cast<uintptr_t>(dst_pool) & 15) ||
      (reinterpret_cast<uintptr_t>(block_pairs) & 7))
    return PA_ERR_INVALID;
  const void *src_d, *dst_d, *pairs_d;
  if (!device_view(src_pool, size_t(src_num_blocks) * block_bytes, &src_d) ||
      !device_view(dst_pool, size_t(dst_num_blocks) * block_bytes, &dst_d) ||
      !device_view(block_pairs, size_t(num_pairs) * 2 * sizeof(int64_t), &pairs_d))
    return pa::fail(PA_ERR_INVALID, "pa_swap_blocks: a pool or the pair list is not device-accessible memory",
                    cudaSuccess);
  return launch_copy(src_d, const_cast<void*>(dst_d), static_cast<const int64_t*>(pairs_d), num_pairs, block_bytes,
                     src_num_blocks, dst_num_blocks, err_flags, reinterpret_cast<cudaStream_t>(stream));
}
