// fpx_diag.cu -- diagnostics with no counterpart in the paper:
//   fpx_diag_bounded_wait  exercises the bounded device-side wait that every pipeline barrier
//                          of the library uses, on a barrier phase that nothing completes;
//   fpx_diag_exp2          evaluates the FMA-pipe exp2 that the attention softmax applies to a
//                          share of its elements, so that its error can be tested directly.
#include <cuda_runtime.h>

#include <climits>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {

__global__ void bounded_wait_kernel(StatusBlock* st, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  // nobody arrives: the wait must give up after limit_ns and report it
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!done) {
    if (sm100::mbar_try_wait(b, 0)) break;
    if (globaltimer_ns() - t0 > limit_ns) done = true;
  }
  if (done && threadIdx.x == 0) record_error(st, FPX_ERR_TIMEOUT, 40);
}

// y[i] = exp2_poly2(x[i]) (pairs of elements, as the softmax evaluates them).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float y0, y1;
  sm100::exp2_poly2(y0, y1, x0, x1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace fpx

extern "C" fpx_status fpx_diag_exp2(const float* x, float* y, int64_t n, fpx_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return FPX_ERR_INVALID_ARG;
  if (n == 0) return FPX_OK;
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > INT32_MAX) return FPX_ERR_UNSUPPORTED;
  fpx::exp2_poly_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                          reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? FPX_OK : FPX_ERR_CUDA;
}

extern "C" fpx_status fpx_diag_bounded_wait(void* ws, uint64_t limit_ns, fpx_stream_t stream) {
  if (!ws) return FPX_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return FPX_ERR_ALIGNMENT;
  if (limit_ns == 0 || limit_ns > fpx::kWaitLimitNs) return FPX_ERR_INVALID_ARG;
  fpx::bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<fpx::StatusBlock*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? FPX_OK : FPX_ERR_CUDA;
}
