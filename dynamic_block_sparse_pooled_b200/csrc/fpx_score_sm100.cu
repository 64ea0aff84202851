// fpx_score_sm100.cu -- pooled block scores on the 5th-generation tensor cores
// (FlashPrefill §3 Method, "Instantaneous Pattern Discovery": s_IJ = scale * <qbar_I, kbar_J>
// for every causal pair of pooled blocks J <= I).
//
// Per head the scores are one lower-triangular [NB x NB] product of the pooled Q rows and the
// pooled K rows of its KV head (inner dimension D = 128), a dense contraction: each CTA computes
// one 128 x 128 tile of it with tcgen05.mma into TMEM and writes the causal pairs of the tile.
//
// Precision: the pooled vectors are fp32 and the selection compares exp(s - m) against alpha,
// so the scores must keep fp32 accuracy.  The tensor cores multiply tf32 (10 explicit mantissa
// bits); the pool kernel therefore stores each mean split as x = hi + lo (hi = x rounded to tf32,
// lo = x - hi exactly), and the product is accumulated as hi*hi + hi*lo + lo*hi in fp32 (the
// lo*lo term is below 2^-21 of |x||y|): a relative error of ~2^-21 per product instead of 2^-11.
//
// Data flow per CTA (128 threads): D is consumed in four chunks of 32 fp32 (one 128-byte
// swizzle row).  One thread issues the TMA loads of the four operand tiles of a chunk
// (Q hi / lo, K hi / lo: 128 rows x 128 B each, 128B-swizzled, zero-filled past the last block)
// into a 3-stage ring -- the first three before TMEM is even allocated -- and the 4 k-steps x 3
// products of each chunk as soon as its tiles land.
// The 128 x 128 fp32 accumulator is read back from TMEM (one row per thread), staged through
// shared memory and written row by row with coalesced stores.  Every wait is bounded; a timeout
// records FPX_ERR_TIMEOUT and the CTA drains its loads and MMAs before it releases TMEM.
#include <cuda_runtime.h>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {
namespace sm100 {

constexpr int kSTile = 128;          // query blocks x key blocks per CTA
constexpr int kSThreads = 128;
constexpr int kSChunks = 4;          // D = 128 in chunks of 32 fp32 (one 128-byte swizzle row)
constexpr int kSStages = 3;
constexpr uint32_t kSOpBytes = kSTile * 128;      // one operand chunk: 128 rows x 128 B
constexpr uint32_t kSStageBytes = 4 * kSOpBytes;  // Q hi, Q lo, K hi, K lo
constexpr uint32_t kSOffBar = kSStages * kSStageBytes;
constexpr int kSStageStride = kSTile + 1;         // epilogue staging row stride (fp32)
constexpr size_t kSSmemBytes = kSOffBar + 64 + 1024;
static_assert(kSTile * kSStageStride * 4 + kSTile * 16 <= kSOffBar, "staging fits in the ring");
constexpr uint32_t kSIdesc = make_idesc(2, 2, false, kSTile, kSTile);  // tf32 x tf32 -> fp32

__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kSThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                ProblemDesc p, float* __restrict__ scores, const int32_t* __restrict__ blk_base,
                const int64_t* __restrict__ tri_base, const int32_t* __restrict__ valid,
                StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  // lower-triangle tile index -> (x, y), y <= x
  const int kt = blockIdx.x;
  int x = static_cast<int>((sqrtf(8.f * kt + 1.f) - 1.f) * 0.5f);
  while (x * (x + 1) / 2 > kt) --x;
  while ((x + 1) * (x + 2) / 2 <= kt) ++x;
  const int y = kt - x * (x + 1) / 2;
  const int h = blockIdx.y;
  const int kvh = h / p.group;
  const int b0 = x * kSTile, c0 = y * kSTile;
  const int b_last = min(p.nb_total, b0 + kSTile) - 1;
  // Whether the tables are valid and whether the tile holds any causal pair (key tiles left of
  // the first sequence of the query tile hold none) is decided after the set-up below, so that
  // these global loads overlap it.
  const int tables_ok = *valid;
  const int first_col = blk_base[seq_of_block(blk_base, p.num_seqs, b0)];

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_u32);
  const uint32_t bar0 = sbase + kSOffBar;
  auto bar_full = [&](int i) { return bar0 + 8u * i; };              // stage i loaded
  auto bar_done = [&](int i) { return bar0 + 8u * (kSStages + i); };  // stage i consumed
  const uint32_t bar_all = bar0 + 8u * (2 * kSStages);                // every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kSOffBar + 8 * (2 * kSStages + 1));
  volatile int* fail_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  auto load_chunk = [&](int c) {
    const int sidx = c % kSStages;
    const uint32_t sb = sbase + sidx * kSStageBytes;
    mbar_arrive_expect_tx(bar_full(sidx), kSStageBytes);
    tma_load_3d(sb + 0 * kSOpBytes, &tmQh, bar_full(sidx), c * 32, h, b0);
    tma_load_3d(sb + 1 * kSOpBytes, &tmQl, bar_full(sidx), c * 32, h, b0);
    tma_load_3d(sb + 2 * kSOpBytes, &tmKh, bar_full(sidx), c * 32, kvh, c0);
    tma_load_3d(sb + 3 * kSOpBytes, &tmKl, bar_full(sidx), c * 32, kvh, c0);
  };
  volatile int never = 0;
  if (tid == 0) {
    for (int i = 0; i < 2 * kSStages + 1; ++i) mbar_init(bar0 + 8u * i, 1);
    fence_mbar_init();
    // the first stages are requested at once (the pooled vectors are always readable), so that
    // their latency overlaps the set-up below
    tma_prefetch_desc(&tmQh);
    tma_prefetch_desc(&tmQl);
    tma_prefetch_desc(&tmKh);
    tma_prefetch_desc(&tmKl);
    for (int c = 0; c < kSStages; ++c) load_chunk(c);
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kSTile);
    tmem_relinquish();
  }
  const bool skip = !tables_ok || c0 + kSTile <= first_col;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (skip) {  // uniform across the CTA: drain the requested loads, release TMEM
    if (tid == 0)
      for (int c = 0; c < kSStages; ++c) mbar_wait(bar_full(c), 0, &never);
    __syncwarp();
    if (warp == 0) tmem_dealloc(tmem, kSTile);
    return;
  }

  if (tid == 0) {
    int loaded = kSStages, issued = 0;
    bool ok = true;
    for (int c = 0; c < kSChunks; ++c) {
      const int sidx = c % kSStages;
      if (!mbar_wait(bar_full(sidx), (c / kSStages) & 1, &never)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = sbase + sidx * kSStageBytes;
      const uint64_t qh = smem_desc_sw128(sb + 0 * kSOpBytes, 16, 1024);
      const uint64_t ql = smem_desc_sw128(sb + 1 * kSOpBytes, 16, 1024);
      const uint64_t kh = smem_desc_sw128(sb + 2 * kSOpBytes, 16, 1024);
      const uint64_t kl = smem_desc_sw128(sb + 3 * kSOpBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // K = 8 tf32 = 32 bytes per instruction
        const uint64_t o = static_cast<uint64_t>(kk * 32) >> 4;
        mma_tf32_ss(tmem, qh + o, kh + o, kSIdesc, (c > 0 || kk > 0) ? 1u : 0u);
        mma_tf32_ss(tmem, qh + o, kl + o, kSIdesc, 1u);
        mma_tf32_ss(tmem, ql + o, kh + o, kSIdesc, 1u);
      }
      mma_commit(bar_done(sidx));
      ++issued;
      // refill the stage consumed by the previous chunk (its MMAs have had a chunk's time)
      if (c >= 1 && loaded < kSChunks) {
        const int prev = (c - 1) % kSStages;
        if (!mbar_wait(bar_done(prev), ((c - 1) / kSStages) & 1, &never)) {
          ok = false;
          break;
        }
        load_chunk(loaded++);
      }
    }
    if (!ok) {
      record_error(st, FPX_ERR_TIMEOUT, 40, h, kt);
      // drain: every load issued has landed and every MMA issued has completed
      for (int c = issued; c < loaded; ++c)
        mbar_wait(bar_full(c % kSStages), (c / kSStages) & 1, &never);
    }
    *fail_flag = ok ? 0 : 1;
    mma_commit(bar_all);
  }
  // where this thread's query-block row goes (global loads overlap the MMAs): columns
  // [col_lo, col_hi] of the tile are causal pairs of one sequence, stored from row_base + col
  int col_lo = 1, col_hi = 0;
  int64_t row_base = 0;
  {
    const int b = b0 + tid;
    if (b <= b_last) {
      const int s = seq_of_block(blk_base, p.num_seqs, b);
      const int first = blk_base[s];
      const int I = b - first;
      col_lo = max(first, c0);
      col_hi = min(b, c0 + kSTile - 1);
      row_base = static_cast<int64_t>(h) * p.tri_total + tri_base[s] +
                 static_cast<int64_t>(I) * (I + 1) / 2 - first;
    }
  }
  __syncthreads();
  const bool ok = mbar_wait(bar_all, 0, &never) && *fail_flag == 0;
  if (ok) {
    tc_fence_after();
    // TMEM row (one query block per thread) -> shared staging [row][col], stride 129 floats
    float* stage_f = reinterpret_cast<float*>(gbase);
    float scale = p.scale;
    if (p.q_scale) scale *= p.q_scale[h] * p.k_scale[kvh];
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + q4 * 32, r);
      tmem_wait_ld(r);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        stage_f[tid * kSStageStride + q4 * 32 + j] = __uint_as_float(r[j]) * scale;
    }
    int64_t* m_base = reinterpret_cast<int64_t*>(gbase + kSTile * kSStageStride * 4);
    int* m_lo = reinterpret_cast<int*>(m_base + kSTile);
    int* m_hi = m_lo + kSTile;
    m_base[tid] = row_base;
    m_lo[tid] = col_lo;
    m_hi[tid] = col_hi;
    tc_fence_before();
    __syncthreads();
    // row by row: a warp writes the causal part of one query-block row with coalesced stores;
    // the four 32-column pieces of a row (and two rows) are read before any is stored, so the
    // shared-memory latency is not paid once per store
#pragma unroll 2
    for (int rr = warp; rr < kSTile; rr += kSThreads / 32) {
      const int64_t base = m_base[rr] + c0;
      const int lo = m_lo[rr] - c0, hi = m_hi[rr] - c0;
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = stage_f[rr * kSStageStride + 32 * u + lane];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int col = 32 * u + lane;
        if (col >= lo && col <= hi) scores[base + col] = v[u];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kSTile);
  }
}

}  // namespace sm100

bool score_tc_supported(const ProblemDesc& p) { return p.d == 128; }

cudaError_t launch_score_tc(const ProblemDesc& p, const float* qhi, const float* khi,
                            const float* qlo, const float* klo, float* scores, SeqTables t,
                            StatusBlock* st, cudaStream_t s) {
  using namespace sm100;
  if (p.nb_total == 0) return cudaSuccess;
  CUtensorMap mqh, mql, mkh, mkl;
  if (!make_tmap_rows128(&mqh, qhi, p.nb_total, p.hq, 128, 4) ||
      !make_tmap_rows128(&mql, qlo, p.nb_total, p.hq, 128, 4) ||
      !make_tmap_rows128(&mkh, khi, p.nb_total, p.hkv, 128, 4) ||
      !make_tmap_rows128(&mkl, klo, p.nb_total, p.hkv, 128, 4))
    return cudaErrorInvalidValue;
  const int nt = (p.nb_total + kSTile - 1) / kSTile;
  dim3 grid(nt * (nt + 1) / 2, p.hq);
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSSmemBytes));
  if (e != cudaSuccess) return e;
  FPX_CHAIN(score_tc_kernel, grid, kSThreads, kSSmemBytes, s, mqh, mql, mkh, mkl, p, scores,
            t.blk_base, t.tri_base, t.valid, st);
  return cudaGetLastError();
}

}  // namespace fpx
