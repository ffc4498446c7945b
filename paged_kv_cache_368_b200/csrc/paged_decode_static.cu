// pa_decode_static: paged decode attention for callers that cannot allocate
// device memory.
//
// pa_decode needs a caller-provided workspace for the partial results of
// units split across warps.  Some callers have no way to provide one: a
// plugin whose host application owns every device allocation and hands it
// only input and output buffers, code running under an allocation policy
// that forbids cudaMalloc on its path (a real-time thread that must never
// block on the allocator, a pre-planned memory budget), or a binding that
// has no device allocator at all.  For them this entry point uses a scratch
// area that is part of the library image itself: a fixed-size array in
// device global memory, reserved when the library's module is loaded on a
// GPU.  The call enqueues kernels (and, the first time on a device, a memset
// of the array's counters), so it must run on an ordinary host thread, never
// inside a host function enqueued on a stream, where CUDA calls are not
// allowed.
//
// Properties a user must know:
//  * The scratch holds kStaticScratchBytes (10 MiB).  Every GPU on which the
//    library's module is loaded keeps that memory reserved until the process
//    exits.  The need is computed for the grid that will actually be
//    launched (pa_decode's plan): every supported shape fits on a GPU of up
//    to 148 SMs (checked at compile time below); on a larger GPU a shape that
//    does not fit is rejected with PA_ERR_WORKSPACE and a pa_last_error()
//    message, and passing max_ctas > 0 shrinks the grid, and the scratch it
//    needs, until it fits.
//  * All calls share the one array per GPU.  Calls whose kernels may run at
//    the same time on one GPU (different streams, different host threads)
//    race on it and produce wrong results: serialise them.
//  * The array keeps what the last call left.  The only words that must start
//    at zero are the split-unit ticket counters, which every decode launch
//    returns to zero; they are cleared once, when the array is first set up
//    on a device (a cudaMemsetAsync on the caller's stream).
//  * The first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (which may load the module) and clears the
//    counters.  Make that first call before any stream capture begins on
//    that device.  The address is cached per CUDA context; after
//    cudaDeviceReset the first call in the new context sets up again.
//  * No device memory is allocated or freed: no cudaMalloc/cudaFree and no
//    allocating library routine is called.
#include <cstdio>
#include <mutex>

#include "pa_device.cuh"
#include "pa_host.h"
#include "paged_decode_kernel.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(10) << 20;
constexpr int kLargestGridSMs = 148;  // B200

constexpr size_t largest_need(int sms) {
  size_t need = 0;
  for (int D : {64, 128})
    for (int G : {1, 2, 4, 8}) {
      const size_t n = pa::ws_layout(sms * pa::warps_for(D, G), sms * pa::kMaxWarpsPerCta, G, D).total;
      need = n > need ? n : need;
    }
  return need;
}
static_assert(largest_need(kLargestGridSMs) <= kStaticScratchBytes,
              "the static scratch must hold the workspace of every supported shape on a 148-SM GPU");

// The ticket counters at the front of the scratch (the same region for every
// call on a device with `sms` SMs).
size_t ticket_bytes(int sms) { return pa::ws_layout(0, sms * pa::kMaxWarpsPerCta, 1, 64).ml; }

}  // namespace

static __device__ __align__(256) unsigned char pa_static_scratch[kStaticScratchBytes];

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

// Device address of pa_static_scratch in the current context, set up once per
// context: the address is looked up (the host-side name of the array is only
// a stand-in, never a device address) and the ticket counters are zeroed on
// `stream`.
void* static_scratch_address(int dev, cudaStream_t stream, cudaError_t* err, const char** what) {
  static std::mutex mu;
  static CUcontext ctx_of[pa::kMaxDevices * 2] = {};
  static void* addr_of[pa::kMaxDevices * 2] = {};
  *err = cudaSuccess;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) {
    *err = cudaErrorNotSupported;
    *what = "pa_decode_static: cuCtxGetCurrent entry point not found";
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  CUcontext ctx = nullptr;
  if (get(&ctx) == CUDA_SUCCESS && ctx != nullptr)
    for (int i = 0; i < pa::kMaxDevices * 2; ++i)
      if (ctx_of[i] == ctx) return addr_of[i];
  // Not set up in this context yet.  The lookup also creates the device's
  // primary context if no context is current.
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, pa_static_scratch);
  if (e != cudaSuccess) {
    *err = e;
    *what = "pa_decode_static: cudaGetSymbolAddress";
    return nullptr;
  }
  if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
    *err = cudaErrorInvalidDevice;
    *what = "pa_decode_static: cuCtxGetCurrent";
    return nullptr;
  }
  const int sms = pa::device_sms(dev);
  e = cudaMemsetAsync(p, 0, ticket_bytes(sms), stream);
  if (e != cudaSuccess) {
    *err = e;
    *what = "pa_decode_static: clearing the ticket counters";
    return nullptr;
  }
  for (int i = 0; i < pa::kMaxDevices * 2; ++i)
    if (ctx_of[i] == nullptr) {
      ctx_of[i] = ctx;
      addr_of[i] = p;
      break;
    }
  return p;
}

}  // namespace

extern "C" pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int max_context_len, float scale,
                                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                                      int64_t num_blocks, pa_dtype dtype, int max_ctas, int32_t* err_flags,
                                      pa_stream_t stream) {
  pa::DecodePlan plan;
  const pa_status st = pa::plan_decode(num_seqs, max_blocks_per_seq, max_context_len, scale, num_heads,
                                       num_kv_heads, head_dim, block_size, num_blocks, dtype, max_ctas, &plan);
  if (st != PA_OK) return st;
  if (num_seqs == 0) return PA_OK;
  if (!pa::decode_pointers_ok(out, q, k_cache, v_cache, block_tables, context_lens)) return PA_ERR_INVALID;
  const pa_status gst = pa::plan_decode_grid(max_ctas, &plan);
  if (gst != PA_OK) return gst;
  if (plan.layout.total > kStaticScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "pa_decode_static: a %d-CTA grid needs %zu bytes of scratch, the static area holds %zu "
             "(pass max_ctas to shrink the grid)",
             plan.ctas, plan.layout.total, kStaticScratchBytes);
    return pa::fail(PA_ERR_WORKSPACE, msg, cudaSuccess);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_static: cudaGetDevice", e);
  const char* what = "";
  void* scratch = static_scratch_address(dev, reinterpret_cast<cudaStream_t>(stream), &e, &what);
  if (scratch == nullptr) return pa::fail(PA_ERR_CUDA, what, e);
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                   max_context_len, scale, num_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype, scratch,
                   kStaticScratchBytes, max_ctas, err_flags, stream);
}
