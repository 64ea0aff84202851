// fpx_attn_simt.cu -- CUDA-core block-sparse attention (FlashPrefill App. B, "Block Sparse
// Attention") for fp32 inputs and the shapes the tensor-core mainloop does not take
// (block < 128, head dim 64, ...).
//
// One CTA per CSR row (h, s, I); D/64 threads per query row, each owning 64 of the D dims.
// Keys are streamed through shared memory 32 at a time (fp32, dequantised); every chunk does
// one online-softmax update (exp2 domain) per query row.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fpx_internal.h"

namespace fpx {

constexpr int kSimtChunk = 32;

template <typename T>
__device__ __forceinline__ float load_val(const T* p);
template <>
__device__ __forceinline__ float load_val<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_val<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float load_val<__nv_fp8_e4m3>(const __nv_fp8_e4m3* p) {
  return static_cast<float>(*p);
}

template <typename OT>
__device__ __forceinline__ void store_val(OT* p, float x);
template <>
__device__ __forceinline__ void store_val<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_val<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

template <typename T, typename OT, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(
    ProblemDesc p, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, OT* __restrict__ o,
    float* __restrict__ lse, SeqTables t, const int32_t* __restrict__ order, StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  constexpr int TPR = D / 64;  // threads per query row
  __shared__ float sk[kSimtChunk][D + 1];
  __shared__ float sv[kSimtChunk][D + 1];
  if (!*t.valid) return;
  const int32_t* __restrict__ blk_base = t.blk_base;

  const int r = order ? order[blockIdx.x] : blockIdx.x;
  const int h = r / p.nb_total;
  const int b = r - h * p.nb_total;
  const int s = seq_of_block(blk_base, p.num_seqs, b);
  const int I = b - blk_base[s];
  const int n_s = seq_len(p, s);
  const int64_t tok0 = seq_start(p, s);
  const int kvh = h / p.group;
  const int row = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int qpos = I * p.block + row;  // local query position
  const bool valid = row < p.block && qpos < n_s;

  const float qs = p.q_scale ? p.q_scale[h] : 1.f;
  const float ks = p.k_scale ? p.k_scale[kvh] : 1.f;
  const float vs = p.v_scale ? p.v_scale[kvh] : 1.f;
  const float sl2 = p.scale * qs * ks * 1.4426950408889634f;  // logits in log2 units

  float qv[64], acc[64];
  const T* qrow = q + ((tok0 + (valid ? qpos : 0)) * p.hq + h) * D + part * 64;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    qv[i] = valid ? load_val(qrow + i) * sl2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -CUDART_INF_F, l = 0.f;

  const int beg = row_ptr[r], end = row_ptr[r + 1];
  for (int e = beg; e < end; ++e) {
    const int J = col_idx[e];
    if (J < 0 || J > I) {
      if (threadIdx.x == 0) record_error(st, FPX_ERR_DEVICE_INPUT, 20, r, J);
      continue;
    }
    for (int c0 = J * p.block; c0 < min((J + 1) * p.block, n_s); c0 += kSimtChunk) {
      const int nk = min(kSimtChunk, min((J + 1) * p.block, n_s) - c0);
      __syncthreads();
      for (int i = threadIdx.x; i < kSimtChunk * D; i += blockDim.x) {
        const int kr = i / D, dd = i % D;
        float kx = 0.f, vx = 0.f;
        if (kr < nk) {
          const int64_t off = ((tok0 + c0 + kr) * p.hkv + kvh) * D + dd;
          kx = load_val(k + off);
          vx = load_val(v + off) * vs;
        }
        sk[kr][dd] = kx;
        sv[kr][dd] = vx;
      }
      __syncthreads();
      float sc[kSimtChunk];
      float cmax = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < kSimtChunk; ++c) {
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) dot = fmaf(qv[i], sk[c][part * 64 + i], dot);
        if (TPR == 2) dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        const bool ok = c < nk && (c0 + c) <= qpos;
        sc[c] = ok ? dot : -CUDART_INF_F;
        cmax = fmaxf(cmax, sc[c]);
      }
      const float m_new = fmaxf(m, cmax);
      if (m_new == -CUDART_INF_F) continue;  // every key of the chunk is masked for this row
      const float corr = ex2_approx(m - m_new);
      l *= corr;
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] *= corr;
#pragma unroll
      for (int c = 0; c < kSimtChunk; ++c) {
        const float pc = ex2_approx(sc[c] - m_new);
        l += pc;
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = fmaf(pc, sv[c][part * 64 + i], acc[i]);
      }
      m = m_new;
    }
  }
  if (!valid) return;
  const int64_t tq = tok0 + qpos;
  OT* orow = o + (tq * p.hq + h) * D + part * 64;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) store_val(orow + i, acc[i] * inv);
  if (lse && part == 0)
    lse[static_cast<int64_t>(h) * p.total_tokens + tq] =
        l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -CUDART_INF_F;
}

template <typename T, typename OT>
static cudaError_t launch_simt_t(const ProblemDesc& p, const void* q, const void* k,
                                 const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                 void* o, float* lse, SeqTables t, const int32_t* order,
                                 StatusBlock* st, cudaStream_t s) {
  const int R = p.hq * p.nb_total;
  const int threads = p.block * (p.d / 64);
  if (p.d == 128)
    FPX_CHAIN((attn_simt_kernel<T, OT, 128>), R, threads, 0, s, p, static_cast<const T*>(q),
              static_cast<const T*>(k), static_cast<const T*>(v), row_ptr, col_idx,
              static_cast<OT*>(o), lse, t, order, st);
  else
    FPX_CHAIN((attn_simt_kernel<T, OT, 64>), R, threads, 0, s, p, static_cast<const T*>(q),
              static_cast<const T*>(k), static_cast<const T*>(v), row_ptr, col_idx,
              static_cast<OT*>(o), lse, t, order, st);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                             const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                             void* o, float* lse, SeqTables t, const int32_t* order,
                             StatusBlock* st, cudaStream_t s) {
  if (p.hq * p.nb_total == 0) return cudaSuccess;
  switch (dt) {
    case FPX_F32:
      return launch_simt_t<float, float>(p, q, k, v, row_ptr, col_idx, o, lse, t, order, st, s);
    case FPX_BF16:
      return launch_simt_t<__nv_bfloat16, __nv_bfloat16>(p, q, k, v, row_ptr, col_idx, o, lse,
                                                         t, order, st, s);
    default:
      return launch_simt_t<__nv_fp8_e4m3, __nv_bfloat16>(p, q, k, v, row_ptr, col_idx, o, lse,
                                                         t, order, st, s);
  }
}

}  // namespace fpx
