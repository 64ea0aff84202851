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
// bits); each operand is therefore split as x = hi + lo with hi = x rounded to tf32 and
// lo = x - hi (exact in fp32), and the product is accumulated as hi*hi + hi*lo + lo*hi in fp32
// (the lo*lo term is below 2^-20 of |x||y|).  The relative error of a product is then ~2^-20
// instead of 2^-11 for a single tf32 product.
//
// Data flow per CTA (128 threads): D is consumed in four chunks of 32 fp32 (one 128-byte
// swizzle row).  All threads load a chunk of the 128 pooled-Q and 128 pooled-K rows from global
// memory (L2-resident, written just before by the pool kernel), split it into hi / lo and store
// the four operand tiles into shared memory in the 128B-swizzled K-major layout; one thread
// then issues the 4 k-steps x 3 products of the chunk.  Two stages alternate, so the loads of
// chunk c + 1 overlap the MMAs of chunk c.  The 128 x 128 fp32 accumulator is read back from
// TMEM (one row per thread), staged through shared memory and written row by row with coalesced
// stores.  Every wait is bounded; a timeout records FPX_ERR_TIMEOUT and the CTA drains its MMAs
// before it releases TMEM.
#include <cuda_runtime.h>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {
namespace sm100 {

constexpr int kSTile = 128;          // query blocks x key blocks per CTA
constexpr int kSThreads = 128;
constexpr int kSChunk = 32;          // fp32 per swizzle row (128 bytes)
constexpr uint32_t kSOpBytes = kSTile * 128;     // one operand chunk: 128 rows x 128 B
constexpr uint32_t kSStageBytes = 4 * kSOpBytes;  // A_hi, A_lo, B_hi, B_lo
constexpr uint32_t kSOffBar = 2 * kSStageBytes;
constexpr int kSStageStride = kSTile + 1;         // epilogue staging row stride (fp32)
constexpr size_t kSSmemBytes = 2 * kSStageBytes + 64 + 1024;
static_assert(kSTile * kSStageStride * 4 <= 2 * kSStageBytes, "staging fits in the stages");
constexpr uint32_t kSIdesc = make_idesc(2, 2, false, kSTile, kSTile);  // tf32 x tf32 -> fp32

__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// x = hi + lo, hi = x rounded to the nearest tf32 (ties away from zero; the tensor core ignores
// the 13 low mantissa bits), lo = x - hi exactly.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  hi = __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
  lo = x - hi;
}

__global__ void __launch_bounds__(kSThreads, 1)
score_tc_kernel(ProblemDesc p, const float* __restrict__ qbar, const float* __restrict__ kbar,
                float* __restrict__ scores, const int32_t* __restrict__ blk_base,
                const int64_t* __restrict__ tri_base, const int32_t* __restrict__ valid,
                StatusBlock* st) {
  if (!*valid) return;
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
  // key tiles left of the first sequence this query tile touches hold no valid pair
  if (c0 + kSTile <= blk_base[seq_of_block(blk_base, p.num_seqs, b0)]) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_u32);
  const uint32_t bar0 = sbase + kSOffBar;  // stage s: bar0 + 8 s; drain: bar0 + 16
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kSOffBar + 24);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    mbar_init(bar0 + 16, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kSTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  float scale = p.scale;
  if (p.q_scale) scale *= p.q_scale[h] * p.k_scale[kvh];
  volatile int never = 0;
  bool ok = true;
  constexpr int kChunks = 128 / kSChunk;
  for (int c = 0; c < kChunks && ok; ++c) {
    const int stage = c & 1;
    const uint32_t sb = sbase + stage * kSStageBytes;
    if (c >= 2 && !mbar_wait(bar0 + 8 * stage, ((c - 2) >> 1) & 1, &never)) {
      ok = false;
      break;
    }
    // 128 rows x 8 float4 per operand: consecutive threads take consecutive 16-byte pieces of
    // a row (coalesced loads); piece j of row r lands at r * 128 + ((j ^ (r & 7)) * 16)
    // (128B swizzle), eight threads covering one 128-byte row without bank conflicts.
    uint8_t* st_base = gbase + stage * kSStageBytes;
#pragma unroll 4
    for (int i = tid; i < kSTile * 8; i += kSThreads) {
      const int r = i >> 3, j = i & 7;
      const int d0 = c * kSChunk + j * 4;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (b0 + r < p.nb_total)
        a = *reinterpret_cast<const float4*>(qbar + (static_cast<int64_t>(b0 + r) * p.hq + h) * 128 + d0);
      if (c0 + r < p.nb_total)
        b = *reinterpret_cast<const float4*>(kbar + (static_cast<int64_t>(c0 + r) * p.hkv + kvh) * 128 + d0);
      float4 ah, al, bh, bl;
      split_tf32(a.x, ah.x, al.x);
      split_tf32(a.y, ah.y, al.y);
      split_tf32(a.z, ah.z, al.z);
      split_tf32(a.w, ah.w, al.w);
      split_tf32(b.x, bh.x, bl.x);
      split_tf32(b.y, bh.y, bl.y);
      split_tf32(b.z, bh.z, bl.z);
      split_tf32(b.w, bh.w, bl.w);
      const uint32_t off = r * 128 + ((j ^ (r & 7)) << 4);
      *reinterpret_cast<float4*>(st_base + 0 * kSOpBytes + off) = ah;
      *reinterpret_cast<float4*>(st_base + 1 * kSOpBytes + off) = al;
      *reinterpret_cast<float4*>(st_base + 2 * kSOpBytes + off) = bh;
      *reinterpret_cast<float4*>(st_base + 3 * kSOpBytes + off) = bl;
    }
    // generic-proxy stores -> visible to the tensor core (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint64_t ahi = smem_desc_sw128(sb + 0 * kSOpBytes, 16, 1024);
      const uint64_t alo = smem_desc_sw128(sb + 1 * kSOpBytes, 16, 1024);
      const uint64_t bhi = smem_desc_sw128(sb + 2 * kSOpBytes, 16, 1024);
      const uint64_t blo = smem_desc_sw128(sb + 3 * kSOpBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // K = 8 tf32 = 32 bytes per instruction
        const uint64_t o = static_cast<uint64_t>(kk * 32) >> 4;
        mma_tf32_ss(tmem, ahi + o, bhi + o, kSIdesc, (c > 0 || kk > 0) ? 1u : 0u);
        mma_tf32_ss(tmem, ahi + o, blo + o, kSIdesc, 1u);
        mma_tf32_ss(tmem, alo + o, bhi + o, kSIdesc, 1u);
      }
      mma_commit(bar0 + 8 * stage);
    }
    __syncwarp();
  }
  // the last commit (chunk 3, stage 1, second use) covers every MMA of the tile
  if (ok && !mbar_wait(bar0 + 8, 1, &never)) ok = false;
  if (!ok) {
    if (tid == 0) {
      record_error(st, FPX_ERR_TIMEOUT, 40, h, kt);
      mma_commit(bar0 + 16);  // drain whatever was issued before TMEM is released
    }
    mbar_wait(bar0 + 16, 0, &never);
  } else {
    tc_fence_after();
    // TMEM row (one query block per thread) -> shared staging [row][col], stride 129 floats
    float* stage_f = reinterpret_cast<float*>(gbase);
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
    tc_fence_before();
    __syncthreads();
    // row by row: a warp writes the causal part of one query-block row with coalesced stores
    for (int rr = warp; rr < kSTile; rr += kSThreads / 32) {
      const int b = b0 + rr;
      if (b > b_last) break;
      const int s = seq_of_block(blk_base, p.num_seqs, b);
      const int first = blk_base[s];
      const int I = b - first;
      const int lo = max(first, c0), hi = min(b, c0 + kSTile - 1);
      const int64_t row_base = static_cast<int64_t>(h) * p.tri_total + tri_base[s] +
                               static_cast<int64_t>(I) * (I + 1) / 2 - first;
      for (int col = lo + lane; col <= hi; col += 32)
        scores[row_base + col] = stage_f[rr * kSStageStride + (col - c0)];
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

cudaError_t launch_score_tc(const ProblemDesc& p, const float* qbar, const float* kbar,
                            float* scores, SeqTables t, StatusBlock* st, cudaStream_t s) {
  using namespace sm100;
  if (p.nb_total == 0) return cudaSuccess;
  const int nt = (p.nb_total + kSTile - 1) / kSTile;
  dim3 grid(nt * (nt + 1) / 2, p.hq);
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSSmemBytes));
  if (e != cudaSuccess) return e;
  score_tc_kernel<<<grid, kSThreads, kSSmemBytes, s>>>(p, qbar, kbar, scores, t.blk_base,
                                                        t.tri_base, t.valid, st);
  return cudaGetLastError();
}

}  // namespace fpx
