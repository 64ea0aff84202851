// fpx_search.cu -- pattern discovery (pool + score) and max-based thresholding (select) kernels.
//
// FlashPrefill ("Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context
// Prefilling"), §3 Method and App. B:
//   * pool_kernel   mean of every B-token block of Q (per Q head) and K (per KV head).  One
//                   streaming pass over Q and K with 16-byte vector loads: this is the HBM-bound
//                   part of the search.
//   * score_kernel  s_IJ = scale * <qbar_I, kbar_J> for the causal pairs J <= I, written as fp32
//                   triangular rows.  64 x 64 register-tiled fp32 dot products out of shared
//                   memory (the pooled vectors are L2-resident).
//   * select_*      per query-block row: row max, the alpha test exp(s - m) >= alpha OR sink OR
//                   window, warp ballot/popc compaction into CSR (no sort, no cumulative sum
//                   over scores).
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
  __shared__ int64_t s_nb[kPlanThreads];
  __shared__ int64_t s_tri[kPlanThreads];
  __shared__ int s_bad[kPlanThreads];
  const int S = p.num_seqs;
  const int tid = threadIdx.x;
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
  s_nb[tid] = nb_sum;
  s_tri[tid] = tri_sum;
  s_bad[tid] = bad ? 1 : 0;
  __syncthreads();
  if (tid == 0) {  // exclusive scan of the per-thread sums (256 entries)
    int64_t a = 0, b = 0;
    for (int i = 0; i < kPlanThreads; ++i) {
      const int64_t x = s_nb[i], y = s_tri[i];
      s_nb[i] = a;
      s_tri[i] = b;
      a += x;
      b += y;
    }
    bool good = true;
    for (int i = 0; i < kPlanThreads; ++i) good = good && s_bad[i] == 0;
    if (!good) record_error(st, FPX_ERR_DEVICE_INPUT, 3);
    if (a != p.nb_total || b != p.tri_total) {
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
    t.blk_base[S] = static_cast<int32_t>(a);
    t.tri_base[S] = b;
  }
  __syncthreads();
  int64_t nb_run = s_nb[tid], tri_run = s_tri[tid];
  for (int s = lo; s < hi; ++s) {
    const int n = seq_len(p, s);
    const int64_t nb = n > 0 ? (n + p.block - 1) / p.block : 0;
    t.blk_base[s] = static_cast<int32_t>(nb_run);
    t.tri_base[s] = tri_run;
    nb_run += nb;
    tri_run += nb * (nb + 1) / 2;
  }
}

cudaError_t launch_plan(const ProblemDesc& p, SeqTables t, StatusBlock* st, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, 0, s>>>(p, t, st);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// pool: qbar[b, h, :] = mean of the valid rows of global block b.  grid.x = NB blocks,
// grid.y = column chunks of Q's Hq*D row followed by those of K's Hkv*D row.
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
                                                            const int32_t* __restrict__ blk_base,
                                                            const int32_t* __restrict__ valid,
                                                            int q_chunks) {
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
  const T* src = (is_q ? q : k) + tok0 * row_elems + c0;
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
#pragma unroll
  for (int i = 0; i < V; i += 4)
    *reinterpret_cast<float4*>(dst + i) =
        make_float4(acc[i] * inv, acc[i + 1] * inv, acc[i + 2] * inv, acc[i + 3] * inv);
}

cudaError_t launch_pool(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                        float* qbar, float* kbar, SeqTables t, cudaStream_t s) {
  const int32_t* blk_base = t.blk_base;
  if (p.nb_total == 0) return cudaSuccess;
  const int V = dt == FPX_F32 ? 4 : dt == FPX_BF16 ? 8 : 16;
  const int per_cta = kPoolThreads * V;
  const int q_chunks = (p.hq * p.d + per_cta - 1) / per_cta;
  const int k_chunks = (p.hkv * p.d + per_cta - 1) / per_cta;
  dim3 grid(p.nb_total, q_chunks + k_chunks);
  switch (dt) {
    case FPX_F32:
      pool_kernel<float><<<grid, kPoolThreads, 0, s>>>(p, static_cast<const float*>(q),
                                                        static_cast<const float*>(k), qbar, kbar,
                                                        blk_base, t.valid, q_chunks);
      break;
    case FPX_BF16:
      pool_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, s>>>(
          p, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qbar,
          kbar, blk_base, t.valid, q_chunks);
      break;
    default:
      pool_kernel<__nv_fp8_e4m3><<<grid, kPoolThreads, 0, s>>>(
          p, static_cast<const __nv_fp8_e4m3*>(q), static_cast<const __nv_fp8_e4m3*>(k), qbar,
          kbar, blk_base, t.valid, q_chunks);
      break;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// score: one CTA per (64 consecutive global query blocks, Q head).  It walks the 64-wide key
// tiles from the first block of the earliest sequence it touches up to its diagonal tile; a
// pair (b, c) of global blocks is written iff both lie in the same sequence and c <= b.
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
  if (!*valid) return;
  extern __shared__ float4 score_smem[];
  float* sq = reinterpret_cast<float*>(score_smem);  // [D][64] (transposed)
  float* sk = sq + D * kScoreTile;                   // [D][64]
  const int h = blockIdx.y;
  const int kvh = h / p.group;
  const int b0 = blockIdx.x * kScoreTile;
  const int b_last = min(p.nb_total, b0 + kScoreTile) - 1;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float scale = p.scale;
  if (p.q_scale) scale *= p.q_scale[h] * p.k_scale[kvh];

  // query tile (transposed into [d][row])
  for (int i = tid; i < kScoreTile * (D / 4); i += kScoreThreads) {
    const int row = i / (D / 4), c4 = (i % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (b0 + row <= b_last)
      v = *reinterpret_cast<const float4*>(qbar + (static_cast<int64_t>(b0 + row) * p.hq + h) * D + c4);
    sq[(c4 + 0) * kScoreTile + row] = v.x;
    sq[(c4 + 1) * kScoreTile + row] = v.y;
    sq[(c4 + 2) * kScoreTile + row] = v.z;
    sq[(c4 + 3) * kScoreTile + row] = v.w;
  }
  // per-row metadata for the 4 rows this thread writes
  int row_seq[4], row_first[4];
  int64_t row_base[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + ty * 4 + i;
    if (b <= b_last) {
      const int s = seq_of_block(blk_base, p.num_seqs, b);
      const int I = b - blk_base[s];
      row_seq[i] = s;
      row_first[i] = blk_base[s];
      row_base[i] = static_cast<int64_t>(h) * p.tri_total + tri_base[s] +
                    static_cast<int64_t>(I) * (I + 1) / 2 - blk_base[s];
    } else {
      row_seq[i] = -1;
      row_first[i] = 0;
      row_base[i] = 0;
    }
  }
  const int first_col = blk_base[seq_of_block(blk_base, p.num_seqs, b0)];
  for (int c0 = (first_col / kScoreTile) * kScoreTile; c0 <= b_last; c0 += kScoreTile) {
    __syncthreads();
    for (int i = tid; i < kScoreTile * (D / 4); i += kScoreThreads) {
      const int col = i / (D / 4), c4 = (i % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + col < p.nb_total)
        v = *reinterpret_cast<const float4*>(kbar + (static_cast<int64_t>(c0 + col) * p.hkv + kvh) * D + c4);
      sk[(c4 + 0) * kScoreTile + col] = v.x;
      sk[(c4 + 1) * kScoreTile + col] = v.y;
      sk[(c4 + 2) * kScoreTile + col] = v.z;
      sk[(c4 + 3) * kScoreTile + col] = v.w;
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
      if (row_seq[i] < 0) continue;
      const int b = b0 + ty * 4 + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + tx * 4 + j;
        if (c >= row_first[i] && c <= b) scores[row_base[i] + c] = acc[i][j] * scale;
      }
    }
  }
}

cudaError_t launch_score(const ProblemDesc& p, fpx_dtype, const float* qbar, const float* kbar,
                         float* scores, SeqTables t, cudaStream_t s) {
  if (p.nb_total == 0) return cudaSuccess;
  dim3 grid((p.nb_total + kScoreTile - 1) / kScoreTile, p.hq);
  const size_t smem = 2 * sizeof(float) * p.d * kScoreTile;
  if (p.d == 128) {
    cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    score_kernel<128><<<grid, kScoreThreads, smem, s>>>(p, qbar, kbar, scores, t.blk_base,
                                                         t.tri_base, t.valid);
  } else {
    score_kernel<64><<<grid, kScoreThreads, smem, s>>>(p, qbar, kbar, scores, t.blk_base,
                                                        t.tri_base, t.valid);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// select: warp per row r = (h, s, I).
// ------------------------------------------------------------------------------------------
constexpr int kSelWarps = 8;

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

__global__ void __launch_bounds__(kSelWarps * 32) select_count_kernel(
    ProblemDesc p, const float* __restrict__ scores, float alpha, int sink, int window,
    float* __restrict__ rowmax, int32_t* __restrict__ counts, SeqTables t) {
  if (!*t.valid) return;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int R = p.hq * p.nb_total;
  if (r >= R) return;
  const RowInfo ri = row_info(p, t, r);
  const float* row = scores + ri.base;
  float m = -CUDART_INF_F;
  for (int j = lane; j < ri.len; j += 32) m = fmaxf(m, __ldcs(row + j));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int cnt = 0;
  for (int j0 = 0; j0 < ri.len; j0 += 32) {
    const int j = j0 + lane;
    const bool kp = j < ri.len && keep_block(row[j], m, alpha, j, ri.I, sink, window);
    cnt += __popc(__ballot_sync(0xffffffffu, kp));
  }
  if (lane == 0) {
    rowmax[r] = m;
    counts[r] = cnt;
  }
}

constexpr int kScanThreads = 1024;

// Exclusive scan of counts into row_ptr (single CTA); nnz, capacity check.
__global__ void __launch_bounds__(kScanThreads) select_scan_kernel(
    int R, const int32_t* __restrict__ counts, int32_t* __restrict__ row_ptr, int64_t capacity,
    int64_t* __restrict__ nnz_d, int* __restrict__ overflow, const int32_t* __restrict__ valid,
    StatusBlock* st) {
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
  const int per = (R + kScanThreads - 1) / kScanThreads;
  const int lo = min(R, tid * per), hi = min(R, lo + per);
  int64_t sum = 0;
  for (int i = lo; i < hi; ++i) sum += counts[i];
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
    row_ptr[i] = static_cast<int32_t>(run);
    run += counts[i];
  }
  if (tid == kScanThreads - 1) {
    const int64_t total = warp_tot[31];
    row_ptr[R] = static_cast<int32_t>(total);
    if (nnz_d) *nnz_d = total;
    const bool over = total > capacity;
    *overflow = over ? 1 : 0;
    if (over) record_error(st, FPX_ERR_CAPACITY, 10, static_cast<int>(total >> 32),
                           static_cast<int>(total & 0xffffffff));
  }
}

__global__ void __launch_bounds__(kSelWarps * 32) select_emit_kernel(
    ProblemDesc p, const float* __restrict__ scores, float alpha, int sink, int window,
    const float* __restrict__ rowmax, const int32_t* __restrict__ row_ptr,
    int32_t* __restrict__ col_idx, const int* __restrict__ overflow, SeqTables t) {
  if (*overflow || !*t.valid) return;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int R = p.hq * p.nb_total;
  if (r >= R) return;
  const RowInfo ri = row_info(p, t, r);
  const float* row = scores + ri.base;
  const float m = rowmax[r];
  int32_t out = row_ptr[r];
  for (int j0 = 0; j0 < ri.len; j0 += 32) {
    const int j = j0 + lane;
    const bool kp = j < ri.len && keep_block(__ldcs(row + j), m, alpha, j, ri.I, sink, window);
    const unsigned bal = __ballot_sync(0xffffffffu, kp);
    if (kp) col_idx[out + __popc(bal & ((1u << lane) - 1u))] = j;
    out += __popc(bal);
  }
}

cudaError_t launch_select(const ProblemDesc& p, const float* scores, float alpha, int sink,
                          int window, int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                          int64_t* nnz_d, float* rowmax, int32_t* counts, int* overflow,
                          SeqTables t, StatusBlock* st, cudaStream_t s) {
  const int R = p.hq * p.nb_total;
  if (R > 0) {
    const int grid = (R + kSelWarps - 1) / kSelWarps;
    select_count_kernel<<<grid, kSelWarps * 32, 0, s>>>(p, scores, alpha, sink, window, rowmax,
                                                       counts, t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  select_scan_kernel<<<1, kScanThreads, 0, s>>>(R, counts, row_ptr, capacity, nnz_d, overflow,
                                                t.valid, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || R == 0) return e;
  select_emit_kernel<<<(R + kSelWarps - 1) / kSelWarps, kSelWarps * 32, 0, s>>>(
      p, scores, alpha, sink, window, rowmax, row_ptr, col_idx, overflow, t);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// order: the attention schedule.  Items are grouped by KV head (so the CTAs resident at any
// moment share K/V blocks through L2) and, inside a group, heaviest first (largest local block
// index I first, since a row can keep at most I + 1 blocks), then sequence, then slot:
//   pos = kvh*slots*NB + slots*sum_s' max(0, nb_s' - 1 - I) + slots*#{s' < s : nb_s' > I} + sub
// Rows (CUDA-core kernel): item r = h*NB + b, slots = Hq/Hkv, sub = h % slots.
// Units (tensor-core kernel, two Q heads of one KV group): item u = (kvh*NB + b)*slots + sub
// with slots = ceil((Hq/Hkv) / 2), sub = the head pair.
// ------------------------------------------------------------------------------------------
__global__ void order_kernel(ProblemDesc p, const int32_t* __restrict__ blk_base,
                             const int32_t* __restrict__ valid, int32_t* __restrict__ order,
                             int units) {
  if (!*valid) return;
  const int slots = units ? (p.group + 1) / 2 : p.group;
  const int n_items = p.hkv * p.nb_total * slots;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_items) return;
  int kvh, b, sub;
  if (units) {
    kvh = i / (p.nb_total * slots);
    const int rem = i - kvh * p.nb_total * slots;
    b = rem / slots;
    sub = rem - b * slots;
  } else {
    const int h = i / p.nb_total;
    b = i - h * p.nb_total;
    kvh = h / p.group;
    sub = h - kvh * p.group;
  }
  const int s = seq_of_block(blk_base, p.num_seqs, b);
  const int I = b - blk_base[s];
  int64_t heavier = 0, same_earlier = 0;
  for (int s2 = 0; s2 < p.num_seqs; ++s2) {
    const int nb2 = blk_base[s2 + 1] - blk_base[s2];
    heavier += max(0, nb2 - 1 - I);
    if (s2 < s && nb2 > I) ++same_earlier;
  }
  const int64_t pos = static_cast<int64_t>(kvh) * slots * p.nb_total + slots * heavier +
                      slots * same_earlier + sub;
  order[pos] = i;
}

cudaError_t launch_order(const ProblemDesc& p, SeqTables t, int32_t* order, bool units,
                         cudaStream_t s) {
  const int slots = units ? (p.group + 1) / 2 : p.group;
  const int n_items = p.hkv * p.nb_total * slots;
  if (n_items == 0) return cudaSuccess;
  order_kernel<<<(n_items + 255) / 256, 256, 0, s>>>(p, t.blk_base, t.valid, order, units ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace fpx
