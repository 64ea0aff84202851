// fpx_attn_sm100.cu -- block-sparse prefill attention on the 5th-generation tensor cores
// (FlashPrefill App. B, "Block Sparse Attention": iterate only over the selected blocks,
// causal masking where required, online softmax with a final normalisation).
//
// Tile = one CSR row (Q head h, sequence s, query block I): 128 query rows x D = 128.
//   * TMA loads the Q tile once and, for every kept key block J of the row, the K_J and V_J
//     tiles (coordinates gathered from col_idx) into a two-stage shared-memory ring.
//   * S = Q K_J^T runs as tcgen05.mma (M = 128, N = 128) with the fp32 accumulator in TMEM.
//   * Each of the 128 threads owns one query row (= one TMEM lane): it reads its S row with
//     tcgen05.ld, applies the token causal mask (diagonal block only), updates the running max
//     and sum in the exp2 domain, rescales its O row in TMEM when the max moved, and writes P
//     (bf16, or e4m3 for fp8 inputs) back into TMEM over S.
//   * O += P V_J runs as tcgen05.mma with A = P read from TMEM and B = V from shared memory.
//   * The epilogue divides O by the row sum and writes O (bf16) and the natural-log LSE.
// Every wait is bounded (FPX_ERR_TIMEOUT is recorded and the CTA exits cleanly).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {
namespace sm100 {

constexpr int kTileM = 128;                 // query rows per tile (= block)
constexpr int kTileN = 128;                 // keys per tile (= block)
constexpr int kHeadDim = 128;
constexpr int kThreads = 128;
constexpr uint32_t kTileBytesMax = 32768;   // one 128 x 128 bf16 tile
constexpr uint32_t kTmemCols = 256;         // S/P: columns [0, 128), O: [128, 256)
constexpr size_t kSmemBytes = 5 * kTileBytesMax + 1024 /*align*/ + 256 /*barriers*/;

template <bool kFp8>
struct Cfg {
  static constexpr uint32_t kElem = kFp8 ? 1 : 2;
  static constexpr uint32_t kTileBytes = kTileM * kHeadDim * kElem;  // 16 KB or 32 KB
  static constexpr uint32_t kBoxBytes = 128 * 128;                   // 128 rows x 128 B
  static constexpr int kBoxes = kTileBytes / kBoxBytes;              // 1 or 2 (along D)
  static constexpr int kKStep = kFp8 ? 32 : 16;                      // MMA K per instruction
  static constexpr int kQKSteps = kHeadDim / kKStep;                 // 4 or 8
  static constexpr int kPVSteps = kTileN / kKStep;                   // 4 or 8
  static constexpr int kPCols = kTileN * kElem / 4;                  // P columns in TMEM
  static constexpr uint32_t kIdescQK = make_idesc(kFp8 ? 0 : 1, kFp8 ? 0 : 1, false, 128, 128);
  static constexpr uint32_t kIdescPV = make_idesc(kFp8 ? 0 : 1, kFp8 ? 0 : 1, true, 128, 128);
};

// Byte offset of K slice `kk` inside a K-major, 128B-swizzled [128 rows x D] tile made of
// kBoxes boxes of [128 rows x 128 B].
template <bool kFp8>
__device__ __forceinline__ uint32_t kmajor_koff(int kk) {
  constexpr int per_box = 128 / (Cfg<kFp8>::kKStep * Cfg<kFp8>::kElem);  // k-steps per 128 B
  return (kk / per_box) * Cfg<kFp8>::kBoxBytes + (kk % per_box) * 32;
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, ProblemDesc p,
               const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
               __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
               SeqTables tab, const int32_t* __restrict__ order, StatusBlock* st) {
  using C = Cfg<kFp8>;
  if (!*tab.valid) return;  // inconsistent cu_seqlens (recorded by the plan kernel)
  const int32_t* __restrict__ blk_base = tab.blk_base;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_u32);
  const uint32_t sQ = sbase;
  // stage x: K at sK0 + x * kTileBytesMax, V at sV0 + x * kTileBytesMax
  const uint32_t sK0 = sbase + kTileBytesMax, sV0 = sbase + 3 * kTileBytesMax;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + 5 * kTileBytesMax);
  const uint32_t bar_q = smem_u32(&bars[0]);
  const uint32_t bar_kv0 = smem_u32(&bars[1]);  // stage x: bar_kv0 + 8 * x
  const uint32_t bar_mma = smem_u32(&bars[3]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[4]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[5]);

  const int tid = threadIdx.x, warp = tid >> 5;

  // ---- tile coordinates -------------------------------------------------------------------
  const int r = order ? order[blockIdx.x] : blockIdx.x;
  const int h = r / p.nb_total;
  const int b = r - h * p.nb_total;
  const int s = seq_of_block(blk_base, p.num_seqs, b);
  const int I = b - blk_base[s];
  const int n_s = seq_len(p, s);
  const int tok0 = seq_start(p, s);
  const int kvh = h / p.group;
  const int q_tok = tok0 + I * kTileM;
  const int beg = row_ptr[r], end = row_ptr[r + 1];

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv0, 1);
    mbar_init(bar_kv0 + 8, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem, tO = tmem + 128;

  // TMA loads in flight (thread 0's bookkeeping, used to drain them on an aborted tile)
  int kv_issued0 = 0, kv_issued1 = 0, kv_waited0 = 0, kv_waited1 = 0;
  bool q_issued = false, q_waited = false;

  // Loads the K/V tiles of key block J into stage `stg` (thread 0 only).
  auto issue_kv = [&](int J, int stg) {
    const int kv_tok = tok0 + J * kTileN;
    if (stg) ++kv_issued1; else ++kv_issued0;
    const uint32_t bar = bar_kv0 + 8 * stg;
    mbar_arrive_expect_tx(bar, 2 * C::kTileBytes);
#pragma unroll
    for (int bx = 0; bx < C::kBoxes; ++bx) {
      tma_load_3d(sK0 + stg * kTileBytesMax + bx * C::kBoxBytes, &tmK, bar, bx * 128 / C::kElem, kvh, kv_tok);
      tma_load_3d(sV0 + stg * kTileBytesMax + bx * C::kBoxBytes, &tmV, bar, bx * 128 / C::kElem, kvh, kv_tok);
    }
  };
  auto valid_J = [&](int J) { return J >= 0 && J <= I; };

  // next valid entry at or after e (all threads compute the same sequence)
  auto next_valid = [&](int e) {
    while (e < end && !valid_J(col_idx[e])) ++e;
    return e;
  };

  int e = next_valid(beg);
  if (tid == 0) {
    for (int x = beg; x < end; ++x)
      if (!valid_J(col_idx[x])) { record_error(st, FPX_ERR_DEVICE_INPUT, 30, r, col_idx[x]); break; }
    if (e < end) {
      q_issued = true;
      mbar_arrive_expect_tx(bar_q, C::kTileBytes);
#pragma unroll
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_3d(sQ + bx * C::kBoxBytes, &tmQ, bar_q, bx * 128 / C::kElem, h, q_tok);
      issue_kv(col_idx[e], 0);
    }
  }

  float sl2 = p.scale * 1.4426950408889634f;
  float vsc = 1.f;
  if (kFp8) {
    sl2 *= p.q_scale[h] * p.k_scale[kvh];
    vsc = p.v_scale[kvh];
  }
  const int my_row = tid;  // TMEM lane == query row of this thread
  float m_run = -CUDART_INF_F, l_run = 0.f;
  uint32_t mma_phase = 0;
  int it = 0;
  bool ok = true;

  while (e < end && ok) {
    const int J = col_idx[e];
    const int stg = it & 1;
    const int e_next = next_valid(e + 1);
    if (tid == 0) {
      if (e_next < end) issue_kv(col_idx[e_next], stg ^ 1);
      bool good = true;
      if (it == 0) good = q_waited = mbar_wait(bar_q, 0, abort_flag);
      if (good) {
        good = mbar_wait(bar_kv0 + 8 * stg, (it >> 1) & 1, abort_flag);
        if (good) { if (stg) ++kv_waited1; else ++kv_waited0; }
      }
      if (good) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::kQKSteps; ++kk) {
          const uint64_t ad = smem_desc_sw128(sQ + kmajor_koff<kFp8>(kk), 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK0 + stg * kTileBytesMax + kmajor_koff<kFp8>(kk), 16, 1024);
          if (kFp8) mma_f8_ss(tS, ad, bd, C::kIdescQK, kk > 0);
          else mma_f16_ss(tS, ad, bd, C::kIdescQK, kk > 0);
        }
        mma_commit(bar_mma);
      } else {
        *abort_flag = 1;
      }
    }
    if (!mbar_wait(bar_mma, mma_phase, abort_flag)) { ok = false; break; }
    mma_phase ^= 1;
    tc_fence_after();

    // ---- softmax on this thread's row ------------------------------------------------------
    uint32_t sr[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_base + c * 32, sr + c * 32);
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_wait_ld(sr + c * 32);
    float x[128];
    float mx = -CUDART_INF_F;
    const bool diag = (J == I);
#pragma unroll
    for (int j = 0; j < 128; ++j) {
      float v = __uint_as_float(sr[j]) * sl2;
      if (diag && j > my_row) v = -CUDART_INF_F;
      x[j] = v;
      mx = fmaxf(mx, v);
    }
    const float m_new = fmaxf(m_run, mx);  // finite: key 0 of the block is always visible
    const float corr = ex2_approx(m_run - m_new);
    // Rescale O rows whose max moved (the previous P*V has completed).  tcgen05.ld/st are
    // warp-collective, so the whole warp takes the branch; rows that did not move scale by 1.
    if (it > 0 && __any_sync(0xffffffffu, m_new > m_run)) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t orow[32];
        tmem_ld32(tO + lane_base + c * 32, orow);
        tmem_wait_ld(orow);
#pragma unroll
        for (int j = 0; j < 32; ++j) orow[j] = __float_as_uint(__uint_as_float(orow[j]) * corr);
        tmem_st32(tO + lane_base + c * 32, orow);
      }
    }
    float psum = 0.f;
    uint32_t pk[64];
    if (kFp8) {
#pragma unroll
      for (int j = 0; j < 128; j += 4) {
        const float p0 = ex2_approx(x[j] - m_new), p1 = ex2_approx(x[j + 1] - m_new);
        const float p2 = ex2_approx(x[j + 2] - m_new), p3 = ex2_approx(x[j + 3] - m_new);
        psum += (p0 + p1) + (p2 + p3);
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
        pk[j / 4] = lo | (hi << 16);
      }
      tmem_st32(tS + lane_base, pk);
    } else {
#pragma unroll
      for (int j = 0; j < 128; j += 2) {
        const float p0 = ex2_approx(x[j] - m_new), p1 = ex2_approx(x[j + 1] - m_new);
        psum += p0 + p1;
        pk[j / 2] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tS + lane_base, pk);
      tmem_st32(tS + lane_base + 32, pk + 32);
    }
    l_run = l_run * corr + psum;
    m_run = m_new;
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();

    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::kPVSteps; ++kk) {
        const uint32_t voff = kk * C::kKStep * 128;  // kKStep key rows of 128 B
        const uint64_t bd = smem_desc_sw128(sV0 + stg * kTileBytesMax + voff, 16384, 1024);
        if (kFp8) mma_f8_ts(tO, tS + kk * 8, bd, C::kIdescPV, (it > 0 || kk > 0));
        else mma_f16_ts(tO, tS + kk * 8, bd, C::kIdescPV, (it > 0 || kk > 0));
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase, abort_flag)) { ok = false; break; }
    mma_phase ^= 1;
    tc_fence_after();
    e = e_next;
    ++it;
  }

  if (!ok) {
    if (tid == 0) record_error(st, FPX_ERR_TIMEOUT, 31, r, it);
    *abort_flag = 1;
  }

  // ---- epilogue -------------------------------------------------------------------------------
  // `ok` and `it` are uniform across the CTA, so every warp executes the (warp-collective) TMEM
  // loads together; only the global stores depend on the row.
  const int qpos = I * kTileM + my_row;
  const bool write = qpos < n_s;
  const int64_t tq = static_cast<int64_t>(tok0) + qpos;
  uint4* orow = reinterpret_cast<uint4*>(o + (tq * p.hq + h) * kHeadDim);
  if (ok && it == 0) {
    if (write) {
#pragma unroll
      for (int i = 0; i < 16; ++i) orow[i] = make_uint4(0, 0, 0, 0);
      if (lse) lse[static_cast<int64_t>(h) * p.total_tokens + tq] = -CUDART_INF_F;
    }
  } else if (ok) {
    const float inv = vsc / l_run;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t ov[32];
      tmem_ld32(tO + lane_base + c * 32, ov);
      tmem_wait_ld(ov);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]) * inv, __uint_as_float(ov[8 * i + 1]) * inv);
        w.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]) * inv, __uint_as_float(ov[8 * i + 3]) * inv);
        w.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]) * inv, __uint_as_float(ov[8 * i + 5]) * inv);
        w.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]) * inv, __uint_as_float(ov[8 * i + 7]) * inv);
        if (write) orow[c * 4 + i] = w;
      }
    }
    if (lse && write)
      lse[static_cast<int64_t>(h) * p.total_tokens + tq] =
          (m_run + __log2f(l_run)) * 0.6931471805599453f;
  }

  // ---- teardown: never release TMEM while an MMA may still be writing it ----------------------
  if (!ok && tid == 0) {
    // drain: bounded waits for this tile's own TMA loads still in flight and for a committed
    // MMA, so that neither writes shared memory or TMEM after the CTA has released them
    volatile int never = 0;
    if (q_issued && !q_waited) mbar_wait(bar_q, 0, &never);
    if (kv_issued0 > kv_waited0) mbar_wait(bar_kv0, (kv_issued0 - 1) & 1, &never);
    if (kv_issued1 > kv_waited1) mbar_wait(bar_kv0 + 8, (kv_issued1 - 1) & 1, &never);
    mbar_wait(bar_mma, mma_phase, &never);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [T, H, D] tensor -> 3-D map {D, H, T}, box {128 bytes, 1 head, 128 tokens}, 128B swizzle.
static bool make_map(CUtensorMap* map, const void* base, int T, int H, int D, bool fp8) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {D * es, static_cast<cuuint64_t>(H) * D * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult rc = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

}  // namespace sm100

bool attn_tc_supported(const ProblemDesc& p, fpx_dtype dt) {
  return (dt == FPX_BF16 || dt == FPX_E4M3) && p.d == 128 && p.block == 128;
}

cudaError_t launch_attn_tc(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                           const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                           void* o, float* lse, SeqTables t, const int32_t* order,
                           StatusBlock* st, cudaStream_t s, bool* encode_failed) {
  using namespace sm100;
  *encode_failed = false;
  const int R = p.hq * p.nb_total;
  if (R == 0) return cudaSuccess;
  const bool fp8 = dt == FPX_E4M3;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, p.total_tokens, p.hq, p.d, fp8) ||
      !make_map(&mk, k, p.total_tokens, p.hkv, p.d, fp8) ||
      !make_map(&mv, v, p.total_tokens, p.hkv, p.d, fp8)) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  auto kern = fp8 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  kern<<<R, kThreads, kSmemBytes, s>>>(mq, mk, mv, p, row_ptr, col_idx,
                                       static_cast<__nv_bfloat16*>(o), lse, t, order, st);
  return cudaGetLastError();
}

}  // namespace fpx
