// fpx_diag.cu -- fpx_diag_bounded_wait: exercises the bounded device-side wait that every
// pipeline barrier of the library uses, on a barrier phase that nothing completes.
#include <cuda_runtime.h>

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

}  // namespace fpx

extern "C" fpx_status fpx_diag_bounded_wait(void* ws, uint64_t limit_ns, fpx_stream_t stream) {
  if (!ws) return FPX_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return FPX_ERR_ALIGNMENT;
  if (limit_ns == 0 || limit_ns > fpx::kWaitLimitNs) return FPX_ERR_INVALID_ARG;
  fpx::bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<fpx::StatusBlock*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? FPX_OK : FPX_ERR_CUDA;
}
