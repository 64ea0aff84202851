// fpx_noalloc.cu -- fpx_select_noalloc: the thresholding / CSR stage for callers that cannot
// hand the library a workspace.
//
// Who needs it: code that is not allowed to allocate device memory at the point where it runs
// -- for example a plugin inside a serving engine whose framework owns every byte of device
// memory and offers no scratch buffer, or latency-critical code that must not call cudaMalloc
// because an allocation can synchronise the device.  Such callers still own the inputs and
// outputs (scores, row_ptr, col_idx, nnz); only the stage's scratch moves into a fixed array
// that lives in the library's own device image.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes (2 MiB).  Every GPU
// that loads the library keeps it until the process exits.  All calls on a device share it:
// calls whose work overlaps on the GPU (different streams without ordering) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "fpx_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

// Host code must not use g_select_scratch's name as an address: on the host it is only a
// stand-in for the device symbol.  The device address is looked up with the device current and
// kept once a lookup has succeeded; a failed lookup (e.g. attempted inside a stream capture) is
// not kept, so the next call tries again.
std::mutex g_mu;
void* g_addr[kMaxDevices];

cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_select_scratch);
    if (e != cudaSuccess || a == nullptr) {
      cudaGetLastError();  // do not leave the failed lookup as the thread's sticky-looking error
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_addr[dev] = a;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t fpx_select_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

fpx_status fpx_select_noalloc(const fpx_problem* p, const float* scores, float alpha,
                              int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d,
                              fpx_stream_t stream) {
  const size_t need = fpx_workspace_bytes(p, 1);  // 0 for an invalid or unsupported problem
  if (need == 0) return FPX_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return FPX_ERR_CAPACITY;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return FPX_ERR_CUDA;
  // The array keeps whatever the previous call left in it; the status block must start at zero
  // (every other part of the scratch is fully rewritten by the stage's kernels).
  if (cudaMemsetAsync(scratch, 0, fpx::kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return FPX_ERR_CUDA;
  return fpx_select(p, scores, alpha, sink_blocks, window_blocks, row_ptr, col_idx, col_capacity,
                    nnz_d, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
