// Device self-tests (no counterpart on the pages):
//  * the bounded barrier wait every kernel of the library relies on: one CTA
//    waits on shared-memory barriers that nothing ever completes and must give
//    up after the given limit, flag the timeout and return, leaving the
//    context usable;
//  * the polynomial 2^x of the multi-token kernel (exp2_poly.cuh), evaluated
//    beside CUDA's exp2f on the same inputs.
#include <algorithm>

#include "exp2_poly.cuh"
#include "pa_host.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint64_t limit_ns, int32_t* err_flags) {
  __shared__ __align__(8) uint64_t bars[2];
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncwarp();
  // Phase 0 of either barrier never completes: no thread arrives on it.  Both
  // wait flavours used by the kernels are exercised: the plain probe loop
  // (decode) and the suspending probe (tensor-core prefill).
  const bool plain = mbar_wait_bounded(&bars[0], 0, limit_ns);
  const bool suspending = tc5::wait(&bars[1], 0, limit_ns);
  if (threadIdx.x == 0) {
    if (!plain) set_err(err_flags, PA_ERRF_TIMEOUT);
    if (!suspending) set_err(err_flags + 1, PA_ERRF_TIMEOUT);
  }
}

// y_poly: the scalar polynomial for even i, the packed two-input form (on
// the pair x[i-1], x[i]) for odd i, so both forms the kernels use are checked.
__global__ void exp2_selftest_kernel(const float* x, float* y_poly, float* y_ref, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    if (i & 1) {
      float a, b;
      exp2_poly2(a, b, x[i - 1], v);
      y_poly[i] = b;
    } else {
      y_poly[i] = exp2_poly(v);
    }
    y_ref[i] = exp2f(v);
  }
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_selftest_exp2(const float* x, float* y_poly, float* y_ref, int64_t n, pa_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_ref))) return PA_ERR_INVALID;
  if (n == 0) return PA_OK;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096));
  pa::exp2_selftest_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y_poly, y_ref, n);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching exp2_selftest_kernel", e);
}

extern "C" pa_status pa_selftest_wait_timeout(uint64_t limit_ns, int32_t* err_flags, pa_stream_t stream) {
  if (!err_flags || limit_ns == 0 || limit_ns > 100000000ull) return PA_ERR_INVALID;
  pa::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, err_flags);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching wait_timeout_kernel", e);
}
