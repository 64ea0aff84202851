// fpx_search.cu -- pattern discovery (pool + score) and max-based thresholding (select) kernels.
//
// FlashPrefill ("Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context
// Prefilling"), §3 Method and App. B:
//   * pool_kernel   mean of every B-token block of Q (per Q head) and K (per KV head).  One
//                   streaming pass over Q and K with 16-byte vector loads: this is the HBM-bound
//                   part of the search.
//   * score_kernel  s_IJ = scale * <qbar_I, kbar_J> for the causal pairs J <= I, written as fp32
//                   triangular rows.  64 x 64 register-tiled fp32 dot products out of shared
//                   memory (the pooled vectors are L2-resident).  Used for D = 64; D = 128
//                   takes the tensor-core kernel of fpx_score_sm100.cu.
//   * select_*      per query-block row: row max, the alpha test exp(s - m) >= alpha OR sink OR
//                   window, warp ballot/popc compaction into CSR (no sort, no cumulative sum
//                   over scores).
// K may be read from a paged cache (FlashPrefill V2 abstract: paged KV cache): the pool kernel
// then takes key block J of sequence s from its page (kv_block_row).
// Radius rescue branch (RBS-Attention abstract: a rescue branch from the maximum key-block
// radius, thresholded independently and OR-ed with the centroid branch):
//   * radius_kernel max distance of a key from its block centroid, and the pooled query norms;
//                   the select count pass then also tests u = s + scale * |qbar_I| * r_J.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fpx_internal.h"

namespace fpx {

// ------------------------------------------------------------------------------------------
// plan: per-sequence block and causal-pair offsets, and device-side cu_seqlens checks.
// ------------------------------------------------------------------------------------------
constexpr int kPlanThreads = 256;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(ProblemDesc p, SeqTables t,
                                                            StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  __shared__ int64_t w_nb[kPlanThreads / 32], w_tri[kPlanThreads / 32];
  __shared__ int s_bad;
  const int S = p.num_seqs;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  // contiguous chunk of sequences per thread
  const int per = (S + kPlanThreads - 1) / kPlanThreads;
  const int lo = min(S, tid * per), hi = min(S, lo + per);
  int64_t nb_sum = 0, tri_sum = 0;
  bool bad = false;
  for (int s = lo; s < hi; ++s) {
    const int n = seq_len(p, s);
    if (n < 0) bad = true;
    const int64_t nb = n > 0 ? (n + p.block - 1) / p.block : 0;
    nb_sum += nb;
    tri_sum += nb * (nb + 1) / 2;
  }
  if (bad) atomicOr(&s_bad, 1);
  // block-wide exclusive scan of (nb_sum, tri_sum): warp shuffles, then across warps
  int64_t a = nb_sum, b = tri_sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += x;
      b += y;
    }
  }
  if (lane == 31) {
    w_nb[wid] = a;
    w_tri[wid] = b;
  }
  __syncthreads();
  int64_t base_nb = 0, base_tri = 0, tot_nb = 0, tot_tri = 0;
#pragma unroll
  for (int i = 0; i < kPlanThreads / 32; ++i) {
    if (i < wid) {
      base_nb += w_nb[i];
      base_tri += w_tri[i];
    }
    tot_nb += w_nb[i];
    tot_tri += w_tri[i];
  }
  int64_t nb_run = base_nb + a - nb_sum, tri_run = base_tri + b - tri_sum;
  for (int s = lo; s < hi; ++s) {
    const int n = seq_len(p, s);
    const int64_t nb = n > 0 ? (n + p.block - 1) / p.block : 0;
    t.blk_base[s] = static_cast<int32_t>(nb_run);
    t.tri_base[s] = tri_run;
    nb_run += nb;
    tri_run += nb * (nb + 1) / 2;
  }
  if (tid == 0) {
    bool good = s_bad == 0;
    if (!good) record_error(st, FPX_ERR_DEVICE_INPUT, 3);
    if (tot_nb != p.nb_total || tot_tri != p.tri_total) {
      record_error(st, FPX_ERR_DEVICE_INPUT, 1);
      good = false;
    }
    if (p.cu && (p.cu[0] != 0 || p.cu[S] != p.total_tokens)) {
      record_error(st, FPX_ERR_DEVICE_INPUT, 2);
      good = false;
    }
    // Every later kernel of the stage returns at once unless the tables are consistent with
    // the sizes the host used for the grids and the caller used for the buffers.
    *t.valid = good ? 1 : 0;
    t.blk_base[S] = static_cast<int32_t>(tot_nb);
    t.tri_base[S] = tot_tri;
  }
}

cudaError_t launch_plan(const ProblemDesc& p, SeqTables t, StatusBlock* st, cudaStream_t s) {
  FPX_CHAIN(plan_kernel, 1, kPlanThreads, 0, s, p, t, st);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// pool: qbar[b, h, :] = mean of the valid rows of global block b.  grid.x = NB blocks,
// grid.y = column chunks of Q's Hq*D row followed by those of K's Hkv*D row.  With qlo / klo
// given (tensor-core scores), the mean x is stored split for tf32 products: qbar = hi = x rounded
// to tf32 (ties away from zero; the tensor core ignores the 13 low mantissa bits) and
// qlo = lo = x - hi (exact), so that x = hi + lo.
// ------------------------------------------------------------------------------------------
constexpr int kPoolThreads = 128;

template <typename T>
struct Vec16;  // one 16-byte load converted to fp32
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void add(const int4& raw, float* acc) {
    const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += f[i];
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(const int4& raw, float* acc) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(b[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
};
template <>
struct Vec16<__nv_fp8_e4m3> {
  static constexpr int N = 16;
  __device__ static void add(const int4& raw, float* acc) {
    const __nv_fp8x2_storage_t* b = reinterpret_cast<const __nv_fp8x2_storage_t*>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(b[i], __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(ProblemDesc p, const T* __restrict__ q,
                                                            const T* __restrict__ k,
                                                            float* __restrict__ qbar,
                                                            float* __restrict__ kbar,
                                                            float* __restrict__ qlo,
                                                            float* __restrict__ klo,
                                                            const int32_t* __restrict__ blk_base,
                                                            const int32_t* __restrict__ valid,
                                                            int q_chunks, StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  constexpr int V = Vec16<T>::N;
  if (!*valid) return;
  const int b = blockIdx.x;
  const int s = seq_of_block(blk_base, p.num_seqs, b);
  const int I = b - blk_base[s];
  const int n_s = seq_len(p, s);
  const int rows = min(p.block, n_s - I * p.block);
  const int64_t tok0 = static_cast<int64_t>(seq_start(p, s)) + static_cast<int64_t>(I) * p.block;

  const bool is_q = blockIdx.y < q_chunks;
  const int chunk = is_q ? blockIdx.y : blockIdx.y - q_chunks;
  const int row_elems = (is_q ? p.hq : p.hkv) * p.d;
  const int c0 = (chunk * kPoolThreads + threadIdx.x) * V;
  if (c0 >= row_elems) return;
  // K rows come from the block's page when K is paged
  const int64_t row0 = is_q ? tok0 : kv_block_row(p, s, I, seq_start(p, s));
  if (row0 < 0) {  // page index outside the cache: recorded, the block's mean is zero
    if (threadIdx.x == 0) record_error(st, FPX_ERR_DEVICE_INPUT, 4, s, I);
    float* dst = kbar + static_cast<int64_t>(b) * row_elems + c0;
#pragma unroll
    for (int i = 0; i < V; i += 4)
      *reinterpret_cast<float4*>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (klo) {
      float* lo = klo + static_cast<int64_t>(b) * row_elems + c0;
#pragma unroll
      for (int i = 0; i < V; i += 4)
        *reinterpret_cast<float4*>(lo + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const T* src = (is_q ? q : k) + row0 * row_elems + c0;
  float* dst = (is_q ? qbar : kbar) + static_cast<int64_t>(b) * row_elems + c0;

  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  int r = 0;
  for (; r + 8 <= rows; r += 8) {  // eight 16-byte loads in flight per thread
    int4 raw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      raw[u] = __ldcs(reinterpret_cast<const int4*>(src + static_cast<int64_t>(r + u) * row_elems));
#pragma unroll
    for (int u = 0; u < 8; ++u) Vec16<T>::add(raw[u], acc);
  }
  for (; r < rows; ++r)
    Vec16<T>::add(__ldcs(reinterpret_cast<const int4*>(src + static_cast<int64_t>(r) * row_elems)),
                  acc);
  const float inv = 1.f / static_cast<float>(rows);
  float* lo = is_q ? qlo : klo;
  if (lo) {
    lo += static_cast<int64_t>(b) * row_elems + c0;
    float lv[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float x = acc[i] * inv;
      const float hi = __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
      acc[i] = hi;
      lv[i] = x - hi;
    }
#pragma unroll
    for (int i = 0; i < V; i += 4)
      *reinterpret_cast<float4*>(lo + i) = make_float4(lv[i], lv[i + 1], lv[i + 2], lv[i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] *= inv;
  }
#pragma unroll
  for (int i = 0; i < V; i += 4)
    *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
}

cudaError_t launch_pool(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                        float* qbar, float* kbar, float* qlo, float* klo, SeqTables t,
                        StatusBlock* st, cudaStream_t s) {
  const int32_t* blk_base = t.blk_base;
  if (p.nb_total == 0) return cudaSuccess;
  const int V = dt == FPX_F32 ? 4 : dt == FPX_BF16 ? 8 : 16;
  const int per_cta = kPoolThreads * V;
  const int q_chunks = (p.hq * p.d + per_cta - 1) / per_cta;
  const int k_chunks = (p.hkv * p.d + per_cta - 1) / per_cta;
  dim3 grid(p.nb_total, q_chunks + k_chunks);
  switch (dt) {
    case FPX_F32:
      FPX_CHAIN(pool_kernel<float>, grid, kPoolThreads, 0, s, p, static_cast<const float*>(q),
                static_cast<const float*>(k), qbar, kbar, qlo, klo, blk_base, t.valid, q_chunks,
                st);
      break;
    case FPX_BF16:
      FPX_CHAIN(pool_kernel<__nv_bfloat16>, grid, kPoolThreads, 0, s, p,
                static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qbar,
                kbar, qlo, klo, blk_base, t.valid, q_chunks, st);
      break;
    default:
      FPX_CHAIN(pool_kernel<__nv_fp8_e4m3>, grid, kPoolThreads, 0, s, p,
                static_cast<const __nv_fp8_e4m3*>(q), static_cast<const __nv_fp8_e4m3*>(k), qbar,
                kbar, qlo, klo, blk_base, t.valid, q_chunks, st);
      break;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// rescue-branch inputs: radius[kvh * NB + b] = max over the block's valid rows j of
// || k_j - kbar_b ||_2 (the largest distance of a key from its block centroid) and
// qnorm[h * NB + b] = || qbar_b ||_2.  One warp per (block, head); D / 32 elements per lane.
// ------------------------------------------------------------------------------------------
constexpr int kRadWarps = 8;

template <typename T>
__device__ __forceinline__ float to_f32(T x) { return static_cast<float>(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_fp8_e4m3>(__nv_fp8_e4m3 x) { return static_cast<float>(x); }

template <typename T, int D>
__global__ void __launch_bounds__(kRadWarps * 32) radius_kernel(
    ProblemDesc p, const T* __restrict__ k, const float* __restrict__ qbar,
    const float* __restrict__ kbar, const float* __restrict__ qlo, const float* __restrict__ klo,
    float* __restrict__ qnorm, float* __restrict__ radius, const int32_t* __restrict__ blk_base,
    const int32_t* __restrict__ valid) {
  pdl_enter();  // after the previous kernel on the stream
  constexpr int E = D / 32;  // elements per lane
  if (!*valid) return;
  const int lane = threadIdx.x & 31;
  const int64_t pair = static_cast<int64_t>(blockIdx.x) * kRadWarps + (threadIdx.x >> 5);
  const int64_t n_k = static_cast<int64_t>(p.nb_total) * p.hkv;
  const int64_t n_q = static_cast<int64_t>(p.nb_total) * p.hq;
  if (pair >= n_k + n_q) return;
  if (pair >= n_k) {  // query norm of pooled block b, head h
    const int64_t qi = pair - n_k;
    const int b = static_cast<int>(qi / p.hq), h = static_cast<int>(qi - static_cast<int64_t>(b) * p.hq);
    const float* hi = qbar + (static_cast<int64_t>(b) * p.hq + h) * D;
    const float* lo = qlo ? qlo + (static_cast<int64_t>(b) * p.hq + h) * D : nullptr;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float x = hi[lane * E + e] + (lo ? lo[lane * E + e] : 0.f);
      acc = fmaf(x, x, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) qnorm[static_cast<int64_t>(h) * p.nb_total + b] = sqrtf(acc);
    return;
  }
  const int b = static_cast<int>(pair / p.hkv), kvh = static_cast<int>(pair - static_cast<int64_t>(b) * p.hkv);
  const int s = seq_of_block(blk_base, p.num_seqs, b);
  const int I = b - blk_base[s];
  const int rows = min(p.block, seq_len(p, s) - I * p.block);
  const int64_t row0 = kv_block_row(p, s, I, seq_start(p, s));
  float c[E];
  {
    const float* hi = kbar + (static_cast<int64_t>(b) * p.hkv + kvh) * D;
    const float* lo = klo ? klo + (static_cast<int64_t>(b) * p.hkv + kvh) * D : nullptr;
#pragma unroll
    for (int e = 0; e < E; ++e) c[e] = hi[lane * E + e] + (lo ? lo[lane * E + e] : 0.f);
  }
  float best = 0.f;
  if (row0 >= 0) {  // an invalid page was recorded by the pool kernel; its radius stays 0
    const T* base = k + (row0 * p.hkv + kvh) * D + lane * E;
    const int64_t stride = static_cast<int64_t>(p.hkv) * D;
    for (int j0 = 0; j0 < rows; j0 += 4) {  // four rows in flight
      float d2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float acc = 0.f;
        if (j0 + u < rows) {
          const T* src = base + (j0 + u) * stride;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float x = to_f32<T>(src[e]) - c[e];
            acc = fmaf(x, x, acc);
          }
        }
        d2[u] = acc;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float a = d2[u];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        best = fmaxf(best, a);
      }
    }
  }
  if (lane == 0) radius[static_cast<int64_t>(kvh) * p.nb_total + b] = sqrtf(best);
}

cudaError_t launch_radius(const ProblemDesc& p, fpx_dtype dt, const void* k, const float* qbar,
                          const float* kbar, const float* qlo, const float* klo, float* qnorm,
                          float* radius, SeqTables t, cudaStream_t s) {
  if (p.nb_total == 0) return cudaSuccess;
  const int64_t pairs = static_cast<int64_t>(p.nb_total) * (p.hkv + p.hq);
  const unsigned grid = static_cast<unsigned>((pairs + kRadWarps - 1) / kRadWarps);
#define FPX_RAD(T, DD)                                                                        \
  FPX_CHAIN((radius_kernel<T, DD>), grid, kRadWarps * 32, 0, s, p, static_cast<const T*>(k),   \
            qbar, kbar, qlo, klo, qnorm, radius, t.blk_base, t.valid)
  if (p.d == 128) {
    if (dt == FPX_F32) FPX_RAD(float, 128);
    else if (dt == FPX_BF16) FPX_RAD(__nv_bfloat16, 128);
    else FPX_RAD(__nv_fp8_e4m3, 128);
  } else {
    if (dt == FPX_F32) FPX_RAD(float, 64);
    else if (dt == FPX_BF16) FPX_RAD(__nv_bfloat16, 64);
    else FPX_RAD(__nv_fp8_e4m3, 64);
  }
#undef FPX_RAD
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// score: one CTA per (64 x 64 tile of global block pairs (b, c) with c <= b, Q head); the tiles
// of the lower triangle are enumerated by blockIdx.x.  A pair is written iff both blocks lie in
// the same sequence and c <= b; tiles that hold no such pair return at once.
// ------------------------------------------------------------------------------------------
constexpr int kScoreTile = 64;
constexpr int kScoreThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each

template <int D>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ProblemDesc p,
                                                              const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              float* __restrict__ scores,
                                                              const int32_t* __restrict__ blk_base,
                                                              const int64_t* __restrict__ tri_base,
                                                              const int32_t* __restrict__ valid) {
  pdl_enter();  // after the previous kernel on the stream
  if (!*valid) return;
  extern __shared__ float4 score_smem[];
  float* sq = reinterpret_cast<float*>(score_smem);  // [D][64] (transposed)
  float* sk = sq + D * kScoreTile;                   // [D][64]
  // lower-triangle tile index -> (x, y), y <= x
  const int k = blockIdx.x;
  int x = static_cast<int>((sqrtf(8.f * k + 1.f) - 1.f) * 0.5f);
  while (x * (x + 1) / 2 > k) --x;
  while ((x + 1) * (x + 2) / 2 <= k) ++x;
  const int y = k - x * (x + 1) / 2;
  const int h = blockIdx.y;
  const int kvh = h / p.group;
  const int b0 = x * kScoreTile, c0 = y * kScoreTile;
  const int b_last = min(p.nb_total, b0 + kScoreTile) - 1;
  // key tiles left of the first sequence this query tile touches hold no valid pair
  const int first_col = blk_base[seq_of_block(blk_base, p.num_seqs, b0)];
  if (c0 + kScoreTile <= first_col) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float scale = p.scale;
  if (p.q_scale) scale *= p.q_scale[h] * p.k_scale[kvh];

  // consecutive threads take consecutive rows, so the transposed shared-memory stores below
  // hit consecutive banks
  for (int i = tid; i < kScoreTile * (D / 4); i += kScoreThreads) {
    const int row = i % kScoreTile, c4 = (i / kScoreTile) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f), u = v;
    if (b0 + row <= b_last)
      v = *reinterpret_cast<const float4*>(qbar + (static_cast<int64_t>(b0 + row) * p.hq + h) * D + c4);
    if (c0 + row < p.nb_total)
      u = *reinterpret_cast<const float4*>(kbar + (static_cast<int64_t>(c0 + row) * p.hkv + kvh) * D + c4);
    sq[(c4 + 0) * kScoreTile + row] = v.x;
    sq[(c4 + 1) * kScoreTile + row] = v.y;
    sq[(c4 + 2) * kScoreTile + row] = v.z;
    sq[(c4 + 3) * kScoreTile + row] = v.w;
    sk[(c4 + 0) * kScoreTile + row] = u.x;
    sk[(c4 + 1) * kScoreTile + row] = u.y;
    sk[(c4 + 2) * kScoreTile + row] = u.z;
    sk[(c4 + 3) * kScoreTile + row] = u.w;
  }
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int dd = 0; dd < D; ++dd) {
    const float4 a = *reinterpret_cast<const float4*>(sq + dd * kScoreTile + ty * 4);
    const float4 c = *reinterpret_cast<const float4*>(sk + dd * kScoreTile + tx * 4);
    const float av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], cv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + ty * 4 + i;
    if (b > b_last) continue;
    const int s = seq_of_block(blk_base, p.num_seqs, b);
    const int first = blk_base[s];
    const int I = b - first;
    const int64_t row_base = static_cast<int64_t>(h) * p.tri_total + tri_base[s] +
                             static_cast<int64_t>(I) * (I + 1) / 2 - first;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c >= first && c <= b) scores[row_base + c] = acc[i][j] * scale;
    }
  }
}

cudaError_t launch_score(const ProblemDesc& p, fpx_dtype, const float* qbar, const float* kbar,
                         const float* qlo, const float* klo, float* scores, SeqTables t,
                         StatusBlock* st, cudaStream_t s) {
  if (p.nb_total == 0) return cudaSuccess;
  if (qlo && klo) return launch_score_tc(p, qbar, kbar, qlo, klo, scores, t, st, s);
  const int nt = (p.nb_total + kScoreTile - 1) / kScoreTile;
  dim3 grid(nt * (nt + 1) / 2, p.hq);
  const size_t smem = 2 * sizeof(float) * p.d * kScoreTile;
  if (p.d == 128) {
    cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    FPX_CHAIN(score_kernel<128>, grid, kScoreThreads, smem, s, p, qbar, kbar, scores, t.blk_base,
              t.tri_base, t.valid);
  } else {
    FPX_CHAIN(score_kernel<64>, grid, kScoreThreads, smem, s, p, qbar, kbar, scores, t.blk_base,
              t.tri_base, t.valid);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// select: a CTA owns 8 consecutive rows r = (h, s, I) (warp per row).
//   count: row max, kept-block count per row, CTA total, and the row's keep bitmask (bit J of
//          word J / 32 at mask[r * mask_words + J / 32]: the ballot of the keep test)
//   scan:  exclusive scan of the CTA totals (one CTA), nnz, capacity check (on overflow: an
//          empty CSR, row_ptr all zero)
//   emit:  per-CTA exclusive scan of its counts -> row_ptr; the bitmask (1/32 of the scores'
//          bytes) compacted into col_idx with popc prefixes
// ------------------------------------------------------------------------------------------
constexpr int kSelWarps = 8;
constexpr int kSelRowsPerWarp = 1;
constexpr int kSelRows = kSelWarps * kSelRowsPerWarp;

struct RowInfo {
  int64_t base;  // first score of the row
  int len;       // I + 1
  int I;
};

__device__ __forceinline__ RowInfo row_info(const ProblemDesc& p, const SeqTables& t, int r) {
  const int h = r / p.nb_total;
  const int b = r - h * p.nb_total;
  const int s = seq_of_block(t.blk_base, p.num_seqs, b);
  const int I = b - t.blk_base[s];
  RowInfo ri;
  ri.base = static_cast<int64_t>(h) * p.tri_total + t.tri_base[s] + static_cast<int64_t>(I) * (I + 1) / 2;
  ri.len = I + 1;
  ri.I = I;
  return ri;
}

// The keep decision of FlashPrefill's max-based dynamic threshold for one block of a row.
__device__ __forceinline__ bool keep_block(float score, float rowmax, float alpha, int J, int I,
                                           int sink, int window) {
  if (alpha == 0.f) return true;
  if (J < sink || J > I - window) return true;
  return expf(score - rowmax) >= alpha;
}

__device__ __forceinline__ float row_max_warp(const float* __restrict__ row, int len, int lane) {
  float m0 = -CUDART_INF_F, m1 = m0, m2 = m0, m3 = m0;
  for (int j = lane; j < len; j += 128) {  // four independent loads in flight per lane
    m0 = fmaxf(m0, __ldg(row + j));
    if (j + 32 < len) m1 = fmaxf(m1, __ldg(row + j + 32));
    if (j + 64 < len) m2 = fmaxf(m2, __ldg(row + j + 64));
    if (j + 96 < len) m3 = fmaxf(m3, __ldg(row + j + 96));
  }
  float m = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

__global__ void __launch_bounds__(kSelWarps * 32) select_count_kernel(
    ProblemDesc p, const float* __restrict__ scores, float alpha, int sink, int window,
    float* __restrict__ rowmax, int32_t* __restrict__ counts, int64_t* __restrict__ cta_tot,
    uint32_t* __restrict__ mask, int mask_words, const float* __restrict__ qn,
    const float* __restrict__ rad, float alpha_r, SeqTables t) {
  pdl_enter();  // after the previous kernel on the stream
  if (!*t.valid) return;
  __shared__ int w_tot[kSelWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = p.hq * p.nb_total;
  int tot = 0;
  for (int k = 0; k < kSelRowsPerWarp; ++k) {
    const int r = blockIdx.x * kSelRows + warp * kSelRowsPerWarp + k;
    if (r >= R) break;
    const RowInfo ri = row_info(p, t, r);
    const float* row = scores + ri.base;
    // rescue branch (qn != nullptr): u_J = s_J + scale_h * ||qbar_I|| * r_J, kept iff
    // alpha_r == 0 or exp(u_J - max u) >= alpha_r, OR-ed with the base test
    float m, mu = 0.f, cr = 0.f;
    const float* radk = nullptr;
    if (qn) {
      const int h = r / p.nb_total, b = r - h * p.nb_total;
      const int kvh = h / p.group;
      const int first = t.blk_base[seq_of_block(t.blk_base, p.num_seqs, b)];
      float sc = p.scale;
      if (p.q_scale) sc *= p.q_scale[h] * p.k_scale[kvh];
      cr = sc * qn[r];
      radk = rad + static_cast<int64_t>(kvh) * p.nb_total + first;
      float m0 = -CUDART_INF_F, u0 = -CUDART_INF_F;
      for (int j = lane; j < ri.len; j += 32) {
        const float v = row[j];
        m0 = fmaxf(m0, v);
        u0 = fmaxf(u0, fmaf(cr, radk[j], v));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        u0 = fmaxf(u0, __shfl_xor_sync(0xffffffffu, u0, o));
      }
      m = m0;
      mu = u0;
    } else {
      m = row_max_warp(row, ri.len, lane);
    }
    int cnt = 0;
    for (int j0 = 0; j0 < ri.len; j0 += 128) {  // four loads in flight per lane
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 32 * u + lane;
        v[u] = j < ri.len ? row[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 32 * u + lane;
        bool kp = j < ri.len && keep_block(v[u], m, alpha, j, ri.I, sink, window);
        if (radk && j < ri.len && !kp)
          kp = alpha_r == 0.f || expf(fmaf(cr, radk[j], v[u]) - mu) >= alpha_r;
        const unsigned bal = __ballot_sync(0xffffffffu, kp);
        const int w = (j0 >> 5) + u;
        if (lane == 0 && w < mask_words) mask[static_cast<int64_t>(r) * mask_words + w] = bal;
        cnt += __popc(bal);
      }
    }
    if (lane == 0) {
      rowmax[r] = m;
      counts[r] = cnt;
    }
    tot += cnt;
  }
  if (lane == 0) w_tot[warp] = tot;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t a = 0;
#pragma unroll
    for (int i = 0; i < kSelWarps; ++i) a += w_tot[i];
    cta_tot[blockIdx.x] = a;
  }
}

constexpr int kScanThreads = 1024;

// Exclusive scan of the per-CTA totals (single CTA); nnz, row_ptr[R], capacity check.
__global__ void __launch_bounds__(kScanThreads) select_scan_kernel(
    int R, int nblk, int64_t* __restrict__ cta_tot, int32_t* __restrict__ row_ptr,
    int64_t capacity, int64_t* __restrict__ nnz_d, int* __restrict__ overflow,
    const int32_t* __restrict__ valid, StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  __shared__ int64_t warp_tot[32];
  if (!*valid) {  // inconsistent cu_seqlens (already recorded): publish an empty CSR
    for (int i = threadIdx.x; i <= R; i += blockDim.x) row_ptr[i] = 0;
    if (threadIdx.x == 0) {
      if (nnz_d) *nnz_d = 0;
      *overflow = 1;
    }
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = (nblk + kScanThreads - 1) / kScanThreads;
  const int lo = min(nblk, tid * per), hi = min(nblk, lo + per);
  int64_t sum = 0;
  for (int i = lo; i < hi; ++i) sum += cta_tot[i];
  int64_t x = sum;  // inclusive warp scan
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int64_t v = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    warp_tot[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int64_t run = x - sum + (w > 0 ? warp_tot[w - 1] : 0);
  for (int i = lo; i < hi; ++i) {
    const int64_t c = cta_tot[i];
    cta_tot[i] = run;  // in place: exclusive offsets
    run += c;
  }
  const int64_t total = warp_tot[31];
  if (total > capacity) {
    // col_idx cannot hold the selection: publish an empty CSR (every row_ptr entry 0), so that
    // no reader of (row_ptr, col_idx) can index past the capacity; nnz_d reports the count the
    // caller would need, and the emit kernel writes nothing.
    for (int i = tid; i <= R; i += kScanThreads) row_ptr[i] = 0;
    if (tid == 0) {
      if (nnz_d) *nnz_d = total;
      *overflow = 1;
      record_error(st, FPX_ERR_CAPACITY, 10, static_cast<int>(total >> 32),
                   static_cast<int>(total & 0xffffffff));
    }
    return;
  }
  if (tid == kScanThreads - 1) {
    row_ptr[R] = static_cast<int32_t>(total);
    if (nnz_d) *nnz_d = total;
    *overflow = 0;
  }
}

__global__ void __launch_bounds__(kSelWarps * 32) select_emit_kernel(
    ProblemDesc p, const int32_t* __restrict__ counts, const int64_t* __restrict__ cta_off,
    int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
    const int* __restrict__ overflow, const uint32_t* __restrict__ mask, int mask_words,
    SeqTables t) {
  pdl_enter();  // after the previous kernel on the stream
  if (!*t.valid || *overflow) return;  // the scan published an empty CSR
  __shared__ int32_t s_off[kSelRows];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = p.hq * p.nb_total;
  const int r0 = blockIdx.x * kSelRows;
  static_assert(kSelRows <= 32, "one lane per row in the CTA-local scan");
  if (warp == 0) {  // exclusive scan of this CTA's counts (one per lane)
    const int c = (lane < kSelRows && r0 + lane < R) ? counts[r0 + lane] : 0;
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < kSelRows) s_off[lane] = x - c;
  }
  __syncthreads();
  const int64_t base = cta_off[blockIdx.x];
  if (threadIdx.x < kSelRows && r0 + threadIdx.x < R)
    row_ptr[r0 + threadIdx.x] = static_cast<int32_t>(base + s_off[threadIdx.x]);
  for (int k = 0; k < kSelRowsPerWarp; ++k) {
    const int rl = warp * kSelRowsPerWarp + k;
    const int r = r0 + rl;
    if (r >= R) break;
    const RowInfo ri = row_info(p, t, r);
    const uint32_t* words = mask + static_cast<int64_t>(r) * mask_words;
    const int nw = (ri.len + 31) >> 5;
    const unsigned below = (1u << lane) - 1u;
    int64_t out = base + s_off[rl];
    for (int w0 = 0; w0 < nw; w0 += 32) {  // 32 words per load, one per lane
      const uint32_t mine = w0 + lane < nw ? __ldcs(words + w0 + lane) : 0u;
      const int n = min(32, nw - w0);
      for (int q = 0; q < n; ++q) {
        const uint32_t word = __shfl_sync(0xffffffffu, mine, q);
        if ((word >> lane) & 1u) col_idx[out + __popc(word & below)] = 32 * (w0 + q) + lane;
        out += __popc(word);
      }
    }
  }
}

int select_ctas(const ProblemDesc& p) { return (p.hq * p.nb_total + kSelRows - 1) / kSelRows; }

cudaError_t launch_select_finish(const ProblemDesc& p, int32_t* row_ptr, int32_t* col_idx,
                                 int64_t capacity, int64_t* nnz_d, const int32_t* counts,
                                 int64_t* cta_tot, int* overflow, const uint32_t* mask,
                                 int mask_words, SeqTables t, StatusBlock* st, cudaStream_t s) {
  const int R = p.hq * p.nb_total;
  const int nblk = select_ctas(p);
  FPX_CHAIN(select_scan_kernel, 1, kScanThreads, 0, s, R, nblk, cta_tot, row_ptr, capacity, nnz_d,
            overflow, t.valid, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || R == 0) return e;
  FPX_CHAIN(select_emit_kernel, nblk, kSelWarps * 32, 0, s, p, counts, cta_tot, row_ptr, col_idx,
            overflow, mask, mask_words, t);
  return cudaGetLastError();
}

cudaError_t launch_select(const ProblemDesc& p, const float* scores, float alpha, int sink,
                          int window, int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                          int64_t* nnz_d, float* rowmax, int32_t* counts, int64_t* cta_tot,
                          int* overflow, uint32_t* mask, int mask_words, const float* qn,
                          const float* rad, float alpha_r, SeqTables t, StatusBlock* st,
                          cudaStream_t s) {
  const int R = p.hq * p.nb_total;
  const int nblk = select_ctas(p);
  if (R > 0) {
    FPX_CHAIN(select_count_kernel, nblk, kSelWarps * 32, 0, s, p, scores, alpha, sink, window,
              rowmax, counts, cta_tot, mask, mask_words, qn, rad, alpha_r, t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  FPX_CHAIN(select_scan_kernel, 1, kScanThreads, 0, s, R, nblk, cta_tot, row_ptr, capacity, nnz_d,
            overflow, t.valid, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || R == 0) return e;
  FPX_CHAIN(select_emit_kernel, nblk, kSelWarps * 32, 0, s, p, counts, cta_tot, row_ptr, col_idx,
            overflow, mask, mask_words, t);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// order: the attention schedule, from the CSR the attention will read.  Items are grouped by KV
// head (so the CTAs resident at any moment share K/V blocks through L2) and, inside a group,
// sorted by their real cost, heaviest first (longest-processing-time order, so that the last
// items to start are the short ones): cost = the kept tiles of the item's CSR rows.
// Rows (CUDA-core kernel): item r = h*NB + b.  Units (tensor-core kernel, two Q heads of one KV
// group at one query block): item u = (kvh*NB + b)*slots + pair, slots = ceil((Hq/Hkv) / 2).
// One CTA runs a counting sort over (KV head, cost bucket) bins in shared memory; the order of
// items inside one bin is arbitrary (it changes where, not what, each item computes).  It also
// resets the work-queue head that the persistent attention kernel takes items from.
// ------------------------------------------------------------------------------------------
constexpr int kOrderThreads = 1024;
constexpr int kOrderMaxBins = 16384;  // 64 KB of shared-memory histogram
constexpr size_t kOrderSmemBudget = 200 * 1024;  // histogram + cached bins

struct OrderShape {
  int slots, per_kv, n_items, nbk, cost_cap, kvb;  // kvb: KV-head groups (<= kOrderMaxBins)
};

inline OrderShape order_shape(const ProblemDesc& p, int nb_max, bool units) {
  OrderShape o;
  o.slots = units ? (p.group + 1) / 2 : p.group;
  o.per_kv = p.nb_total * o.slots;
  o.n_items = p.hkv * o.per_kv;
  o.cost_cap = (units ? 2 : 1) * nb_max;
  o.kvb = p.hkv < kOrderMaxBins ? p.hkv : kOrderMaxBins;
  const int cap_bins = kOrderMaxBins / o.kvb;
  o.nbk = o.cost_cap + 1 < cap_bins ? o.cost_cap + 1 : cap_bins;
  return o;
}

// (KV head, cost) of item i; the bin sorts heavier items first inside a KV head.
__device__ __forceinline__ int order_bin(const ProblemDesc& p, const OrderShape& o,
                                         const int32_t* __restrict__ row_ptr, int i, int units) {
  int kvh, cost;
  if (units) {
    kvh = i / o.per_kv;
    const int rem = i - kvh * o.per_kv;
    const int b = rem / o.slots;
    const int pair = rem - b * o.slots;
    const int h0 = kvh * p.group + 2 * pair;
    const int r0 = h0 * p.nb_total + b;
    cost = __ldg(row_ptr + r0 + 1) - __ldg(row_ptr + r0);
    if (2 * pair + 1 < p.group) {
      const int r1 = r0 + p.nb_total;
      cost += __ldg(row_ptr + r1 + 1) - __ldg(row_ptr + r1);
    }
  } else {
    const int h = i / p.nb_total;
    kvh = h / p.group;
    cost = __ldg(row_ptr + i + 1) - __ldg(row_ptr + i);
  }
  cost = min(max(cost, 0), o.cost_cap);
  const int bucket = static_cast<int>(static_cast<int64_t>(cost) * o.nbk / (o.cost_cap + 1));
  const int kvg = static_cast<int>(static_cast<int64_t>(kvh) * o.kvb / p.hkv);
  return kvg * o.nbk + (o.nbk - 1 - bucket);
}

__global__ void __launch_bounds__(kOrderThreads) order_kernel(
    ProblemDesc p, const int32_t* __restrict__ valid, const int32_t* __restrict__ row_ptr,
    int32_t* __restrict__ order, int* __restrict__ queue_head, OrderShape o, int units,
    int cache_bins) {
  pdl_enter();  // after the previous kernel on the stream
  extern __shared__ int hist[];  // [kvb * nbk] counts, then (cache_bins) uint16 bin per item
  __shared__ int warp_sum[kOrderThreads / 32];
  if (!*valid) return;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nbins = o.kvb * o.nbk;
  uint16_t* bin_of = reinterpret_cast<uint16_t*>(hist + nbins);
  for (int i = tid; i < nbins; i += kOrderThreads) hist[i] = 0;
  if (tid == 0) *queue_head = 0;
  __syncthreads();
  // pass 1: four items per thread in flight (their row_ptr loads are independent)
  for (int i0 = tid; i0 < o.n_items; i0 += 4 * kOrderThreads) {
    int bins[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kOrderThreads;
      bins[u] = i < o.n_items ? order_bin(p, o, row_ptr, i, units) : -1;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (bins[u] < 0) continue;
      atomicAdd(&hist[bins[u]], 1);
      if (cache_bins) bin_of[i0 + u * kOrderThreads] = static_cast<uint16_t>(bins[u]);
    }
  }
  __syncthreads();
  // exclusive scan of the histogram: a contiguous chunk per thread, then across the CTA
  const int per = (nbins + kOrderThreads - 1) / kOrderThreads;
  const int lo = min(nbins, tid * per), hi = min(nbins, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += hist[i];
  int x = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_sum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int v = warp_sum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, d);
      if (lane >= d) v += y;
    }
    warp_sum[lane] = v;
  }
  __syncthreads();
  int run = x - sum + (wid > 0 ? warp_sum[wid - 1] : 0);
  for (int i = lo; i < hi; ++i) {
    const int c = hist[i];
    hist[i] = run;
    run += c;
  }
  __syncthreads();
  // pass 2: scatter (bins from shared memory, or recomputed when they did not fit)
  for (int i = tid; i < o.n_items; i += kOrderThreads) {
    const int bin = cache_bins ? static_cast<int>(bin_of[i]) : order_bin(p, o, row_ptr, i, units);
    order[atomicAdd(&hist[bin], 1)] = i;
  }
}

cudaError_t launch_order(const ProblemDesc& p, int nb_max, SeqTables t, const int32_t* row_ptr,
                         int32_t* order, int* queue_head, bool units, cudaStream_t s) {
  const OrderShape o = order_shape(p, nb_max, units);
  if (o.n_items == 0) return cudaSuccess;
  // the histogram, and the items' bins (uint16) when they fit in the shared memory budget
  const size_t hist_bytes = sizeof(int) * static_cast<size_t>(o.kvb) * o.nbk;
  const size_t bins_bytes = sizeof(uint16_t) * static_cast<size_t>(o.n_items);
  const int cache_bins = hist_bytes + bins_bytes <= kOrderSmemBudget ? 1 : 0;
  const size_t smem = hist_bytes + (cache_bins ? bins_bytes : 0);
  cudaError_t e = cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  FPX_CHAIN(order_kernel, 1, kOrderThreads, smem, s, p, t.valid, row_ptr, order, queue_head, o,
            units ? 1 : 0, cache_bins);
  return cudaGetLastError();
}

}  // namespace fpx
