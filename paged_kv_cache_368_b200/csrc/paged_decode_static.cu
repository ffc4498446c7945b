// pa_decode_static: paged decode attention for callers that cannot allocate
// device memory.
//
// pa_decode needs a caller-provided workspace for the partial results of
// units split across warps.  Some callers have no way to provide one: code
// running where cudaMalloc is forbidden or unavailable (for example inside a
// host callback, a real-time thread that must not block on the allocator,
// or a plugin host that owns every device allocation and hands out only
// input/output buffers).  For them this entry point uses a scratch area that
// is part of the library image itself: a fixed-size array in device global
// memory, reserved when the library's module is loaded on a GPU.
//
// Properties a user must know:
//  * The scratch holds kStaticScratchBytes (10 MiB).  Every GPU on which this
//    entry point is used keeps that memory reserved until the process exits.
//    The shapes the library supports need at most 9.5 MiB on a 148-SM B200;
//    a request that needs more (a GPU with more SMs) is rejected with
//    PA_ERR_WORKSPACE and a pa_last_error() message -- pass max_ctas to
//    shrink the grid (and the scratch it needs) in that case.
//  * All calls share the one array per GPU.  Calls whose kernels may run at
//    the same time on one GPU (different streams, different host threads)
//    race on it and produce wrong results: serialise them.
//  * The kernel writes every scratch word before reading it in the same
//    call, so nothing has to start at zero and the contents a previous call
//    left behind are harmless.
//  * The first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (which may load the module).  Make that first call
//    before any stream capture begins on that device.
//  * No device memory is allocated or freed: no cudaMalloc/cudaFree and no
//    allocating library routine is called.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "pa_device.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(10) << 20;
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char pa_static_scratch[kStaticScratchBytes];

namespace {

// Device address of pa_static_scratch on device `dev` (the current device),
// looked up once per device.  The host-side name of the array is only a
// stand-in: a kernel must be given this address, never &pa_static_scratch.
void* static_scratch_address(int dev, cudaError_t* err) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  *err = cudaSuccess;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, pa_static_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int max_context_len, float scale,
                                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                                      int64_t num_blocks, pa_dtype dtype, int max_ctas, int32_t* err_flags,
                                      pa_stream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_static: cudaGetDevice", e);
  const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len);
  if (need > kStaticScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg), "pa_decode_static: needs %zu bytes of scratch, the static area holds %zu", need,
             kStaticScratchBytes);
    return pa::fail(PA_ERR_WORKSPACE, msg, cudaSuccess);
  }
  void* scratch = static_scratch_address(dev, &e);
  if (scratch == nullptr) return pa::fail(PA_ERR_CUDA, "pa_decode_static: cudaGetSymbolAddress", e);
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                   max_context_len, scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype, scratch,
                   kStaticScratchBytes, max_ctas, err_flags, stream);
}
