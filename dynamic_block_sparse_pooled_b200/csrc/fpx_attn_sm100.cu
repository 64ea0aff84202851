// fpx_attn_sm100.cu -- block-sparse prefill attention on the 5th-generation tensor cores
// (FlashPrefill App. B, "Block Sparse Attention": iterate only over the selected blocks, causal
// masking where required, online softmax with a final normalisation).
//
// Work unit = two query tiles that share one KV head ("GQA head packing"): Q heads h0 = 2p and
// h1 = 2p + 1 of KV group g, both at query block I of sequence s (128 rows x D = 128 each).
// The CTA walks the union of the two heads' CSR rows; a key block is loaded once (TMA, gathered
// by block index) and multiplied only by the tile(s) that kept it.
//
// Persistent schedule: one CTA per SM; the load warp takes units from a queue that the order
// kernel sorted by kept-tile count (heaviest first inside each KV head) and hands each to the
// other roles through a two-slot ring in shared memory.  TMEM is allocated once per CTA; the
// K / V rings, the S / P barriers and their phases run on across units, so the next unit's K / V
// loads and S MMAs start while the previous unit's last softmax and epilogue finish.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for tile 0: one query row (= one TMEM lane) per thread
//   warps 4-7  softmax for tile 1
//   warp  8    tcgen05.mma issue for both tiles (one elected lane), TMEM allocation
//   warp  10   TMA loads (one elected lane): Q0/Q1 once, then K_J and V_J into 2-slot rings
//   warps 9, 11 idle (complete the third warpgroup)
// setmaxnreg moves registers from the third warpgroup to the two softmax warpgroups, which
// hold a whole 128-column S row in registers.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_t (bf16 / e4m3)
// is written over the first columns of S_t and read from TMEM by the P*V MMA.
//
// The tensor pipe buffers only a few MMA instructions, so the issuing thread must never stop for
// long between groups.  One warp issues every MMA in a fixed order per union entry n:
//     O_1 += P_1(n') V_n', S_1(n) = Q_1 K_n^T | O_0 += P_0(n) V_n, S_0(n + 1) = Q_0 K_{n+1}^T
// where n' is tile 1's previous entry.  Softmax 0 of entry n then runs while the pipe executes
// tile 1's P*V and S, and softmax 1 while it executes tile 0's P*V and next S, so the two
// softmaxes alternate on the MUFU instead of contending for it.  S_t of an entry is always
// issued after the previous O_t += P_t V (same thread, in-order pipe), so when softmax t sees S_t
// complete, O_t is stable and may be rescaled in place.  Each ring slot is released by one commit
// after the last MMA that reads it.
//
// Softmax: exp2 domain, lazy rescale (the reference max only moves when the block max exceeds it
// by more than 2^8), the S row read from TMEM in two halves (the second in flight while the first
// is reduced) and P written back in two halves (the first while the second is computed); e4m3
// forms P in the same pass as the block max once a reference exists, and redoes the block in two
// passes only when the max moves the reference.  Every
// wait is bounded: a broken pipeline records FPX_ERR_TIMEOUT, drains its own TMA loads and MMAs,
// releases TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <climits>
#include <mutex>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {
namespace sm100 {

constexpr int kTileM = 128;   // query rows per tile (= block)
constexpr int kTileN = 128;   // keys per block
constexpr int kHeadDim = 128;
constexpr int kThreads = 384;
// softmax / other warpgroups' registers after setmaxnreg: 256 x S + 128 x O <= 384 x 168 (the
// registers at launch), both multiples of 8
#ifndef FPX_SOFTMAX_REGS
#define FPX_SOFTMAX_REGS 208
#endif
constexpr int kSoftmaxRegs = FPX_SOFTMAX_REGS;
constexpr int kOtherRegs = (384 * 168 - 256 * kSoftmaxRegs) / 128 / 8 * 8;
static_assert(kOtherRegs >= 24 && kSoftmaxRegs % 8 == 0 && kSoftmaxRegs <= 256, "register split");
constexpr int kMmaWarp = 8;    // issues every MMA; allocates TMEM
constexpr int kLoadWarp = 10;
constexpr uint32_t kSlotBytes = 32768;  // one 128 x 128 bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;    // lazy rescale threshold (log2 units)
// shared memory: Q0, Q1, K slot 0/1, V slot 0/1 (32 KB each), then barriers, the TMEM base
// address, the abort flag and the two-slot unit ring
constexpr uint32_t kOffQ = 0, kOffK = 2 * kSlotBytes, kOffV = 4 * kSlotBytes,
                   kOffBar = 6 * kSlotBytes;
constexpr size_t kSmemBytes = 6 * kSlotBytes + 256 + 1024;

enum Bar {
  kBarQ = 0,        // Q tiles of the current unit landed (one phase per unit)
  kBarKFull = 1,    // +slot
  kBarKEmpty = 3,   // +slot
  kBarVFull = 5,    // +slot
  kBarVEmpty = 7,   // +slot
  kBarSFull = 9,    // +tile
  kBarPReady = 11,  // +tile
  kBarODone = 13,   // +tile: one phase per unit in which the tile had entries
  kBarDrain = 15,
  kBarQEmpty = 16,  // every S of the current unit completed (one phase per unit)
  kBarUFull = 17,   // +slot: a unit index published in the ring
  kBarUEmpty = 19,  // +slot: every reader took it
  kNumBars = 21
};
constexpr int kUnitReaders = 9;  // the MMA warp and the eight softmax warps

template <bool kFp8>
struct Cfg {
  static constexpr uint32_t kElem = kFp8 ? 1 : 2;
  static constexpr uint32_t kTileBytes = kTileM * kHeadDim * kElem;  // 16 KB or 32 KB
  static constexpr uint32_t kBoxBytes = 128 * 128;                   // 128 rows x 128 B
  static constexpr int kBoxes = kTileBytes / kBoxBytes;              // 1 or 2 (along D)
  static constexpr int kKStep = kFp8 ? 32 : 16;                      // MMA K per instruction
  static constexpr int kQKSteps = kHeadDim / kKStep;
  static constexpr int kPVSteps = kTileN / kKStep;
  static constexpr uint32_t kIdescQK = make_idesc(kFp8 ? 0 : 1, kFp8 ? 0 : 1, false, 128, 128);
  static constexpr uint32_t kIdescPV = make_idesc(kFp8 ? 0 : 1, kFp8 ? 0 : 1, true, 128, 128);
};

// Byte offset of K slice `kk` inside a K-major, 128B-swizzled [128 rows x D] tile made of
// kBoxes boxes of [128 rows x 128 B].
template <bool kFp8>
__device__ __forceinline__ uint32_t kmajor_koff(int kk) {
  constexpr int per_box = 128 / (Cfg<kFp8>::kKStep * Cfg<kFp8>::kElem);
  return (kk / per_box) * Cfg<kFp8>::kBoxBytes + (kk % per_box) * 32;
}

// Union of two CSR rows, consumed in list order.  Every entry of each row is visited exactly
// once; entries outside [0, I] are skipped.  With ascending rows (as fpx_select writes them) the
// union is ascending and shared blocks are visited once for both tiles.  The head of each row is
// held in a register and its successor is loaded as soon as it is consumed, so the global-load
// latency falls between two calls (one pipeline step) instead of inside one.
struct RowMerge {
  const int32_t* ci;
  int a, a_end, b, b_end, I;
  int va, vb;  // ci[a], ci[b] (INT_MAX past the end)
  __device__ __forceinline__ RowMerge(const int32_t* ci_, int a_, int a_end_, int b_, int b_end_,
                                      int I_)
      : ci(ci_), a(a_), a_end(a_end_), b(b_), b_end(b_end_), I(I_) {
    va = a < a_end ? ci[a] : INT_MAX;
    vb = b < b_end ? ci[b] : INT_MAX;
  }
  __device__ __forceinline__ bool ok(int J) const { return J >= 0 && J <= I; }
  __device__ __forceinline__ bool next(int& J, int& uses) {
    while (a < a_end && !ok(va)) va = ++a < a_end ? ci[a] : INT_MAX;
    while (b < b_end && !ok(vb)) vb = ++b < b_end ? ci[b] : INT_MAX;
    if (a >= a_end && b >= b_end) return false;
    const int ja = a < a_end ? va : INT_MAX;
    const int jb = b < b_end ? vb : INT_MAX;
    J = min(ja, jb);
    uses = (ja == J ? 1 : 0) | (jb == J ? 2 : 0);
    if (ja == J) va = ++a < a_end ? ci[a] : INT_MAX;
    if (jb == J) vb = ++b < b_end ? ci[b] : INT_MAX;
    return true;
  }
};

// Maximum of 64 fp32 values (3-input max, four independent chains).
__device__ __forceinline__ float row_max64(const uint32_t* r) {
  float m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = __uint_as_float(r[k]);
#pragma unroll
  for (int j = 4; j < 60; j += 8)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      m[k] = max3f(m[k], __uint_as_float(r[j + k]), __uint_as_float(r[j + 4 + k]));
  return max3f(max3f(m[0], m[1], __uint_as_float(r[60])), max3f(m[2], m[3], __uint_as_float(r[61])),
               fmaxf(__uint_as_float(r[62]), __uint_as_float(r[63])));
}

// One in kPolyEvery element pairs takes exp2 on the FMA pipe instead of the MUFU (0: none).  The
// MUFU issues four ex2 per cycle per SM sub-partition, so a 128-column row costs ~1000 cycles
// there; moving a quarter of the pairs to the FMA pipe was measured fastest (one in two or three
// saturates the FMA pipe instead).
#ifndef FPX_POLY_EVERY
#define FPX_POLY_EVERY 4
#endif
constexpr int kPolyEvery = FPX_POLY_EVERY;

// Columns [J0, J0 + N) of the S row in r become P, packed in place (bf16 pairs at r[J0 / 2 ..],
// or e4m3 quads at r[J0 / 4 ..]); returns their sum.
template <bool kFp8, int J0, int N>
__device__ __forceinline__ float softmax_part_to_p(uint32_t* r, float sl2, float neg_m) {
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = J0; j < J0 + N; j += 2) {
    float x0, x1, p0, p1;
    ffma2(x0, x1, __uint_as_float(r[j]), __uint_as_float(r[j + 1]), sl2, sl2, neg_m, neg_m);
    constexpr int kEvery = kPolyEvery > 0 ? kPolyEvery : 1;
    if (kPolyEvery > 0 && (j / 2) % kEvery == kEvery - 1) {
      exp2_poly2(p0, p1, x0, x1);
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    fadd2(s[(j / 2) % 4 * 2], s[(j / 2) % 4 * 2 + 1], p0, p1);
    if (kFp8) {
      const uint32_t v = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
      if ((j & 2) == 0) r[j / 4] = v;
      else r[j / 4] |= v << 16;
    } else {
      r[j / 2] = pack_bf16x2(p0, p1);
    }
  }
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

struct Unit {
  int kvh, b, s, I, tok0, n_s, ntiles;
  int h[2], r[2], beg[2], end[2];
};

__device__ __forceinline__ Unit decode_unit(const ProblemDesc& p, const int32_t* blk_base,
                                            const int32_t* row_ptr, int u) {
  Unit w;
  const int pairs = (p.group + 1) / 2;
  const int per_kv = p.nb_total * pairs;
  w.kvh = u / per_kv;
  const int rem = u - w.kvh * per_kv;
  w.b = rem / pairs;
  const int pair = rem - w.b * pairs;
  w.s = seq_of_block(blk_base, p.num_seqs, w.b);
  w.I = w.b - blk_base[w.s];
  w.tok0 = seq_start(p, w.s);
  w.n_s = seq_len(p, w.s);
  w.ntiles = (2 * pair + 1 < p.group) ? 2 : 1;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    w.h[t] = w.kvh * p.group + 2 * pair + t;
    if (t < w.ntiles) {
      w.r[t] = w.h[t] * p.nb_total + w.b;
      w.beg[t] = row_ptr[w.r[t]];
      w.end[t] = row_ptr[w.r[t] + 1];
    } else {
      w.r[t] = -1;
      w.beg[t] = w.end[t] = 0;
    }
  }
  return w;
}

// 128 bits [bit0, bit0 + 128) of a bitmask row of `words` words, as four words (bit c of the
// result in word c / 32); bits outside the row read as 0.
__device__ __forceinline__ void bits128(const uint32_t* __restrict__ row, int words, int64_t bit0,
                                        uint32_t out[4]) {
  const int64_t w0 = bit0 >> 5;  // floor, also for negative bit0
  const int sh = static_cast<int>(bit0 & 31);
  uint32_t wv[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int64_t wi = w0 + i;
    wv[i] = (wi >= 0 && wi < words) ? __ldg(row + wi) : 0u;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) out[i] = __funnelshift_r(wv[i], wv[i + 1], sh);
}

// kMask: the vertical / slash token mask (query i of sequence s attends key j <= i iff bit
// s_start + j of vbits[h] or bit s_start + (i - j) of sbits[h] is set) is applied inside every
// listed key block, and a row that no key reaches gets O = 0, LSE = -inf.
template <bool kFp8, bool kMask>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, ProblemDesc p,
               const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
               __nv_bfloat16* __restrict__ o, float* __restrict__ lse, SeqTables tab,
               const int32_t* __restrict__ order, int* __restrict__ queue_head, int n_units,
               const uint32_t* __restrict__ vbits, const uint32_t* __restrict__ sbits, int words,
               StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  using C = Cfg<kFp8>;
  constexpr unsigned kFull = 0xffffffffu;
  if (!*tab.valid) return;  // inconsistent cu_seqlens (recorded by the plan kernel)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_u32);
  const uint32_t bar0 = sbase + kOffBar;  // barrier i at bar0 + 8 * i
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * kNumBars + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * kNumBars + 8);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(bar(kBarQ), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarKFull + i), 1);
      mbar_init(bar(kBarKEmpty + i), 1);
      mbar_init(bar(kBarVFull + i), 1);
      mbar_init(bar(kBarVEmpty + i), 1);
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarPReady + i), kTileM / 32);  // one arrival per softmax warp
      mbar_init(bar(kBarODone + i), 1);
      mbar_init(bar(kBarUFull + i), 1);
      mbar_init(bar(kBarUEmpty + i), kUnitReaders);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Unit k of this CTA sits in ring slot k & 1; its readers (the MMA warp and the eight softmax
  // warps, each fully converged here) release the slot once they have read it.  -1 ends the
  // loop.  The wait is warp-uniform, so a timeout takes the whole warp out together.
  auto take_unit = [&](int k, int& u) -> bool {
    const uint32_t b = bar(kBarUFull + (k & 1));
    if (!__all_sync(kFull, mbar_wait(b, (k >> 1) & 1, abort_flag))) return false;
    u = unit_ring[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kBarUEmpty + (k & 1)));
    return true;
  };

  if (warp >= 8) {
  setmaxnreg_dec<kOtherRegs>();
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer ----
    // Takes units from the queue (heaviest first), publishes each to the other roles, then
    // loads its Q tiles and the K / V blocks of the union of its two CSR rows into the rings.
    // Warp-uniform loop; lane 0 / one elected lane issue.
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int n = 0;        // K / V ring entries issued (over all units)
    int k = 0;        // units published
    int q_loads = 0;  // units whose Q tiles were requested
    bool ok = true;
    while (true) {
      int u = -1;
      if (lane == 0) {
        const int qi = atomicAdd(queue_head, 1);
        u = qi < n_units ? order[qi] : -1;
      }
      u = __shfl_sync(kFull, u, 0);
      if (!__all_sync(kFull, mbar_wait(bar(kBarUEmpty + (k & 1)), ((k >> 1) & 1) ^ 1,
                                       abort_flag))) {
        ok = false;
        break;
      }
      if (lane == 0) {
        unit_ring[k & 1] = u;
        mbar_arrive(bar(kBarUFull + (k & 1)));  // release: the slot write is visible first
      }
      __syncwarp();
      ++k;
      if (u < 0) break;
      const Unit w = decode_unit(p, tab.blk_base, row_ptr, u);
      // Q tiles of this unit (every unit has them, with or without entries): the buffers are
      // free once every S of the previous unit has completed
      if (k > 1 && !__all_sync(kFull, mbar_wait(bar(kBarQEmpty), (k - 2) & 1, abort_flag))) {
        ok = false;
        break;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(kBarQ), C::kTileBytes * w.ntiles);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (t >= w.ntiles) break;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sbase + kOffQ + t * kSlotBytes + bx * C::kBoxBytes, &tmQ, bar(kBarQ),
                        bx * 128 / C::kElem, w.h[t], w.tok0 + w.I * kTileM);
        }
      }
      ++q_loads;
      RowMerge m(col_idx, w.beg[0], w.end[0], w.beg[1], w.end[1], w.I);
      int J, uses;
      while (m.next(J, uses)) {
        const int slot = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        // first K / V row of block J (its page when K / V are paged); a page index outside the
        // cache is recorded and read past the end of the map (TMA fills zeros there)
        int64_t kv_row = kv_block_row(p, w.s, J, w.tok0);
        if (kv_row < 0) {
          if (elect_one()) record_error(st, FPX_ERR_DEVICE_INPUT, 34, w.s, J);
          kv_row = static_cast<int64_t>(p.num_pages) * kTileN;
        }
        const int kv_tok = static_cast<int>(kv_row);
        if (!__all_sync(kFull, mbar_wait(bar(kBarKEmpty + slot), ph ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(kBarKFull + slot), C::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sbase + kOffK + slot * kSlotBytes + bx * C::kBoxBytes, &tmK,
                        bar(kBarKFull + slot), bx * 128 / C::kElem, w.kvh, kv_tok);
        }
        if (!__all_sync(kFull, mbar_wait(bar(kBarVEmpty + slot), ph ^ 1, abort_flag))) {
          // K of this entry is in flight; only its K barrier is drained below
          volatile int never = 0;
          mbar_wait(bar(kBarKFull + slot), ph, &never);
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(kBarVFull + slot), C::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sbase + kOffV + slot * kSlotBytes + bx * C::kBoxBytes, &tmV,
                        bar(kBarVFull + slot), bx * 128 / C::kElem, w.kvh, kv_tok);
        }
        ++n;
      }
      if (!ok) break;
    }
    if (!ok) *abort_flag = 1;
    // Drain: wait (bounded) until every load this warp issued has landed: the last Q (one Q
    // load at most is in flight) and the last two ring entries.
    volatile int never = 0;
    if (q_loads > 0) mbar_wait(bar(kBarQ), (q_loads - 1) & 1, &never);
    for (int e = n - 2; e < n; ++e) {
      if (e < 0) continue;
      const int slot = e & 1;
      const uint32_t ph = (e >> 1) & 1;
      mbar_wait(bar(kBarKFull + slot), ph, &never);
      mbar_wait(bar(kBarVFull + slot), ph, &never);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer -------
    // Warp-uniform sequential loop; one elected lane issues and commits.  Order per union entry
    // n:  O_1 += P_1(n') V_n' (tile 1's previous entry), S_1(n) | O_0 += P_0(n) V_n, S_0(n + 1).
    // Softmax 0 of entry n runs while the tensor pipe executes tile 1's P*V and S, and softmax 1
    // while it executes tile 0's P*V and next S, so the two softmaxes alternate.
    // Matrix descriptors of every buffer, built once.  A k-step inside a buffer only moves the
    // start-address field (bits 0-13, address >> 4): a constant add to the descriptor.
    const uint64_t qdesc0 = smem_desc_sw128(sbase + kOffQ, 16, 1024);
    const uint64_t qdesc1 = qdesc0 + (kSlotBytes >> 4);
    const uint64_t dk0 = smem_desc_sw128(sbase + kOffK, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(sbase + kOffV, 16384, 1024);
    constexpr uint64_t kSlotDesc = kSlotBytes >> 4;
    const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
    auto issue_s = [&](uint32_t tS, uint64_t qdesc, int slot) {
      const uint64_t kdesc = dk0 + slot * kSlotDesc;
#pragma unroll
      for (int kk = 0; kk < C::kQKSteps; ++kk) {
        const uint64_t off = kmajor_koff<kFp8>(kk) >> 4;
        if (kFp8) mma_f8_ss(tS, qdesc + off, kdesc + off, C::kIdescQK, kk > 0);
        else mma_f16_ss(tS, qdesc + off, kdesc + off, C::kIdescQK, kk > 0);
      }
    };
    auto issue_pv = [&](uint32_t tO, uint32_t tS, int slot, bool started) {
      const uint64_t vdesc = dv0 + slot * kSlotDesc;
#pragma unroll
      for (int kk = 0; kk < C::kPVSteps; ++kk) {
        const uint32_t acc = (started || kk > 0) ? 1u : 0u;
        const uint64_t bd = vdesc + ((kk * C::kKStep * 128) >> 4);
        if (kFp8) mma_f8_ts(tO, tS + kk * 8, bd, C::kIdescPV, acc);
        else mma_f16_ts(tO, tS + kk * 8, bd, C::kIdescPV, acc);
      }
    };
    int n = 0;  // ring entries consumed (over all units)
    int k = 0;  // units taken
    uint32_t p_phase0 = 0, p_phase1 = 0;
    bool ok = true;
    while (ok) {
      int u;
      if (!take_unit(k, u)) { ok = false; break; }
      ++k;
      if (u < 0) break;
      const Unit w = decode_unit(p, tab.blk_base, row_ptr, u);
      RowMerge m(col_idx, w.beg[0], w.end[0], w.beg[1], w.end[1], w.I);
      int J, uses;
      bool have = m.next(J, uses);
      if (!__all_sync(kFull, mbar_wait(bar(kBarQ), (k - 1) & 1, abort_flag))) { ok = false; break; }
      bool o0_started = false, o1_started = false;
      int pend = -1;  // ring index of tile 1's entry whose P*V is not issued yet
      // A P*V and the S that follows it in the same tile are issued back to back from one
      // elected block: any wait or bookkeeping between them would leave the tensor pipe idle.
      if (have) {  // S_0 of the first entry
        if (!__all_sync(kFull, mbar_wait(bar(kBarKFull + (n & 1)), (n >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (elect_one() && (uses & 1)) {
          tc_fence_after();
          issue_s(tS0, qdesc0, n & 1);
          mma_commit(bar(kBarSFull + 0));
        }
        __syncwarp();
      }
      while (have) {
        const int slot = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        // tile 1: O_1 += P_1 V of its previous entry, then S_1 of this entry
        const bool pv1 = pend >= 0;
        const int ps = pend & 1;
        if (pv1) {
          if (!__all_sync(kFull, mbar_wait(bar(kBarPReady + 1), p_phase1, abort_flag))) { ok = false; break; }
          p_phase1 ^= 1;
          if (!__all_sync(kFull, mbar_wait(bar(kBarVFull + ps), (pend >> 1) & 1, abort_flag))) { ok = false; break; }
        }
        if (elect_one()) {
          tc_fence_after();
          if (pv1) {
            issue_pv(tO1, tS1, ps, o1_started);
            mma_commit(bar(kBarVEmpty + ps));
          }
          if (uses & 2) {
            issue_s(tS1, qdesc1, slot);
            mma_commit(bar(kBarSFull + 1));
          }
          mma_commit(bar(kBarKEmpty + slot));  // every S reading K_n has been issued
        }
        __syncwarp();
        if (pv1) {
          o1_started = true;
          pend = -1;
        }
        // The next union entry (global loads of the CSR arrays) and its K tile, while this
        // entry's MMAs run and softmax 0 works.
        int uses_next = 0;
        const bool have_next = m.next(J, uses_next);
        const int nslot = (n + 1) & 1;
        if (have_next &&
            !__all_sync(kFull, mbar_wait(bar(kBarKFull + nslot), ((n + 1) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        const bool s0_next = have_next && (uses_next & 1);
        // tile 0: O_0 += P_0 V of this entry, then S_0 of the next entry
        if (uses & 1) {
          if (!__all_sync(kFull, mbar_wait(bar(kBarPReady + 0), p_phase0, abort_flag))) { ok = false; break; }
          p_phase0 ^= 1;
          if (!__all_sync(kFull, mbar_wait(bar(kBarVFull + slot), ph, abort_flag))) { ok = false; break; }
        }
        if (elect_one()) {
          tc_fence_after();
          if (uses & 1) {
            issue_pv(tO0, tS0, slot, o0_started);
            if (!(uses & 2)) mma_commit(bar(kBarVEmpty + slot));
          }
          if (s0_next) {
            issue_s(tS0, qdesc0, nslot);
            mma_commit(bar(kBarSFull + 0));
          }
        }
        __syncwarp();
        if (uses & 1) o0_started = true;
        if (uses & 2) pend = n;
        ++n;
        have = have_next;
        uses = uses_next;
      }
      if (!ok) break;
      // every S of this unit is issued: Q may be reloaded once they complete
      if (elect_one()) mma_commit(bar(kBarQEmpty));
      __syncwarp();
      if (pend >= 0) {  // tile 1's last P*V
        const int ps = pend & 1;
        if (!__all_sync(kFull, mbar_wait(bar(kBarPReady + 1), p_phase1, abort_flag)) ||
            !__all_sync(kFull, mbar_wait(bar(kBarVFull + ps), (pend >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        p_phase1 ^= 1;
        if (elect_one()) {
          tc_fence_after();
          issue_pv(tO1, tS1, ps, o1_started);
          mma_commit(bar(kBarVEmpty + ps));
        }
        __syncwarp();
        o1_started = true;
      }
      // O_t is final once its P*V complete; a tile without entries gets no commit (its softmax
      // warps do not wait for one)
      if (elect_one()) {
        if (o0_started) mma_commit(bar(kBarODone + 0));
        if (o1_started) mma_commit(bar(kBarODone + 1));
      }
      __syncwarp();
    }
    if (!ok) *abort_flag = 1;
    // drain: every MMA issued by this warp completes before TMEM can be released
    if (elect_one()) mma_commit(bar(kBarDrain));
    volatile int never = 0;
    mbar_wait(bar(kBarDrain), 0, &never);
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax ----------
    const int t = warp >> 2;                 // tile
    const int row = tid & 127;               // query row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_base;
    const uint32_t tO = tmem + 256 + t * 128 + lane_base;
    uint32_t s_phase = 0;   // S_t phases (over all units)
    uint32_t od_phase = 0;  // O_t-done phases: one per unit in which this tile had entries
    int k = 0;
    int my_r = -1, it = 0;
    bool ok = true;
    while (ok) {
      int u;
      if (!take_unit(k, u)) { ok = false; break; }
      ++k;
      if (u < 0) break;
      const Unit w = decode_unit(p, tab.blk_base, row_ptr, u);
      if (t >= w.ntiles) continue;
      const int my_h = w.h[t];
      my_r = w.r[t];
      const int qpos = w.I * kTileM + row;
      const bool write = qpos < w.n_s;
      const int64_t tq = static_cast<int64_t>(w.tok0) + qpos;
      float sl2 = p.scale * 1.4426950408889634f;
      float vsc = 1.f;
      if (kFp8) {
        sl2 *= p.q_scale[my_h] * p.k_scale[w.kvh];
        vsc = p.v_scale[w.kvh];
      }
      float m_ref = -CUDART_INF_F, l_run = 0.f;
      const uint32_t* vrow = kMask ? vbits + static_cast<int64_t>(my_h) * words : nullptr;
      const uint32_t* srow = kMask ? sbits + static_cast<int64_t>(my_h) * words : nullptr;
      it = 0;
      for (int e = w.beg[t]; e < w.end[t]; ++e) {
        const int J = col_idx[e];
        if (J < 0 || J > w.I) {
          if (row == 0) record_error(st, FPX_ERR_DEVICE_INPUT, 30, my_r, J);
          continue;
        }
        // token mask of this row in block J: verticals (bit c = key J*B + c) or slashes (bit
        // c = offset qpos - J*B - c, the 128 offsets read reversed)
        uint32_t am[4];
        if (kMask) {
          uint32_t vm[4], xs[4];
          bits128(vrow, words, static_cast<int64_t>(w.tok0) + J * kTileN, vm);
          bits128(srow, words, static_cast<int64_t>(w.tok0) + qpos - J * kTileN - (kTileN - 1), xs);
#pragma unroll
          for (int i = 0; i < 4; ++i) am[i] = vm[i] | __brev(xs[3 - i]);
        }
        if (!mbar_wait(bar(kBarSFull + t), s_phase, abort_flag)) { ok = false; break; }
        s_phase ^= 1;
        tc_fence_after();
        const bool diag = (J == w.I);
        // token causal mask (key column > query row) and token mask of one 64-column half
        auto mask_half = [&](uint32_t* x, int j0) {
          if (diag) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j0 + j > row) x[j] = __float_as_uint(-CUDART_INF_F);
          }
          if (kMask) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (!((am[(j0 + j) >> 5] >> ((j0 + j) & 31)) & 1u)) x[j] = __float_as_uint(-CUDART_INF_F);
          }
        };
        // the whole S row of this thread: 128 fp32 in registers (one TMEM read)
        uint32_t r[128];
        float rs = 0.f;
        // e4m3: once the reference max is set (every lane of the warp), P is formed against it
        // in the same pass that takes the block max; the lazy-rescale rule keeps that P whenever
        // the block max stays within 2^8 of the reference, which is the rule's own no-rescale
        // case, so the result is the one the two-pass order gives.  Otherwise nothing has been
        // stored yet, S is still in TMEM, and the warp redoes the block in two passes.  (bf16
        // keeps the two-pass order: its P is twice as many TMEM columns, and storing the first
        // half while the second is formed was measured to be worth more than the single pass.)
        const bool spec = kFp8 && it > 0 && __all_sync(kFull, m_ref != -CUDART_INF_F);
        bool redo = !spec;
        if (spec) {
          tmem_ld32(tS, r);
          tmem_ld32(tS + 32, r + 32);
          tmem_wait_ld(r);
          tmem_wait_ld(r + 32);
          tmem_ld32(tS + 64, r + 64);
          tmem_ld32(tS + 96, r + 96);
          mask_half(r, 0);
          const float mx_lo = row_max64(r);
          rs = softmax_part_to_p<kFp8, 0, 64>(r, sl2, -m_ref);
          tmem_wait_ld(r + 64);
          tmem_wait_ld(r + 96);
          mask_half(r + 64, 64);
          const float mx = fmaxf(mx_lo, row_max64(r + 64)) * sl2;
          rs += softmax_part_to_p<kFp8, 64, 64>(r, sl2, -m_ref);
          redo = __any_sync(kFull, mx > m_ref + kRescaleLog2);
          if (!redo) {
            if (kFp8) {
              tmem_st16(tS, r);
              tmem_st16(tS + 16, r + 16);
            } else {
              tmem_st32(tS, r);
              tmem_st32(tS + 32, r + 32);
            }
          }
        }
        if (redo) {
          tmem_ld32(tS, r);
          tmem_ld32(tS + 32, r + 32);
          tmem_wait_ld(r);
          tmem_wait_ld(r + 32);
          // second half in flight while the first half is masked and reduced
          tmem_ld32(tS + 64, r + 64);
          tmem_ld32(tS + 96, r + 96);
          mask_half(r, 0);
          const float mx_lo = row_max64(r);
          tmem_wait_ld(r + 64);
          tmem_wait_ld(r + 96);
          mask_half(r + 64, 64);
          // finite unless kMask: key 0 of a block row is always visible without the token
          // mask; with it a row may see no key yet (m_ref = -inf), and -inf then stands for
          // "none"
          const float mx = fmaxf(mx_lo, row_max64(r + 64)) * sl2;
          // lazy rescale: move the reference max only when the block max exceeds it by > 2^8
          float corr = 1.f;
          if (mx > m_ref + kRescaleLog2) {
            corr = ex2_approx(m_ref - mx);  // 0 for the first block
            l_run *= corr;
            m_ref = mx;
          }
          if (it > 0 && __any_sync(kFull, corr != 1.f)) {
            // O_t is stable: the previous P*V into it completed before S_t was written
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t ov[32];
              tmem_ld32(tO + c * 32, ov);
              tmem_wait_ld(ov);
#pragma unroll
              for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * corr);
              tmem_st32(tO + c * 32, ov);
            }
          }
          // P = exp2(s * sl2 - m_ref), packed in place and written over S
          // first half of P stored while the second half is computed
          // (a row that no key has reached yet: exponents of -inf, P = 0, and the weights the
          // FMA-pipe exp2 gives them are cleared by the rescale that its first key triggers)
          const float neg_m = (kMask && m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
          rs = softmax_part_to_p<kFp8, 0, 64>(r, sl2, neg_m);
          if (kFp8) tmem_st16(tS, r);
          else tmem_st32(tS, r);
          rs += softmax_part_to_p<kFp8, 64, 64>(r, sl2, neg_m);
          if (kFp8) tmem_st16(tS + 16, r + 16);
          else tmem_st32(tS + 32, r + 32);
        }
        l_run += rs;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(bar(kBarPReady + t));
        ++it;
      }
      if (!ok) break;
      // epilogue: wait for the last P*V, normalise, store O (bf16) and the natural-log LSE
      uint4* orow = reinterpret_cast<uint4*>(o + (tq * p.hq + my_h) * kHeadDim);
      if (it == 0) {
        if (write) {
#pragma unroll
          for (int i = 0; i < 16; ++i) orow[i] = make_uint4(0, 0, 0, 0);
          if (lse) lse[static_cast<int64_t>(my_h) * p.total_tokens + tq] = -CUDART_INF_F;
        }
        continue;
      }
      if (!mbar_wait(bar(kBarODone + t), od_phase, abort_flag)) { ok = false; break; }
      od_phase ^= 1;
      tc_fence_after();
      // kMask: a row that no key reached (blocks were listed, the token mask removed every key
      // of them for this row) gets O = 0 and LSE = -inf; every lane still takes part in the
      // warp-wide TMEM loads below
      const bool none = kMask && m_ref == -CUDART_INF_F;
      const float inv = none ? 0.f : vsc / l_run;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld(r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 v4;
          v4.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv);
          v4.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv);
          v4.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv);
          v4.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv);
          if (write) orow[c * 4 + i] = v4;
        }
      }
      if (lse && write)
        lse[static_cast<int64_t>(my_h) * p.total_tokens + tq] =
            none ? -CUDART_INF_F : (m_ref + __log2f(l_run)) * 0.6931471805599453f;
      // O_t's TMEM columns are read: the next unit's first P*V into them waits for this warp's
      // first P of that unit, which comes after these loads in program order
      tc_fence_before();
    }
    if (!ok) {
      *abort_flag = 1;
      if (row == 0) record_error(st, FPX_ERR_TIMEOUT, 31, my_r, it);
    }
  }

  // ---- teardown: every role has drained its own async work ------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------------------------
}  // namespace sm100

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

bool make_tmap_rows128(CUtensorMap* map, const void* base, int T, int H, int D, int elem_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = static_cast<cuuint64_t>(elem_bytes);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {D * es, static_cast<cuuint64_t>(H) * D * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult rc = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

namespace sm100 {
static bool make_map(CUtensorMap* map, const void* base, int T, int H, int D, bool fp8) {
  return make_tmap_rows128(map, base, T, H, D, fp8 ? 1 : 2);
}

}  // namespace sm100

bool attn_tc_supported(const ProblemDesc& p, fpx_dtype dt) {
  return (dt == FPX_BF16 || dt == FPX_E4M3) && p.d == 128 && p.block == 128;
}

int64_t attn_tc_units(const ProblemDesc& p) {
  return static_cast<int64_t>(p.hkv) * p.nb_total * ((p.group + 1) / 2);
}

// Streaming multiprocessors of the current device (one resident CTA each: the kernel's shared
// memory admits no second one), looked up once per device.
static int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      return 148;
    counts[dev] = n;
  }
  return counts[dev];
}

cudaError_t launch_attn_tc(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                           const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                           void* o, float* lse, SeqTables t, const int32_t* order,
                           int* queue_head, const uint32_t* vbits, const uint32_t* sbits,
                           int words, StatusBlock* st, cudaStream_t s, bool* encode_failed) {
  using namespace sm100;
  *encode_failed = false;
  const int64_t units = attn_tc_units(p);
  if (units == 0) return cudaSuccess;
  const bool fp8 = dt == FPX_E4M3;
  CUtensorMap mq, mk, mv;
  const int kv_rows = p.page_table ? p.num_pages * p.block : p.total_tokens;
  if (!make_map(&mq, q, p.total_tokens, p.hq, p.d, fp8) ||
      !make_map(&mk, k, kv_rows, p.hkv, p.d, fp8) ||
      !make_map(&mv, v, kv_rows, p.hkv, p.d, fp8)) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  const bool mask = vbits != nullptr;
  auto kern = fp8 ? (mask ? attn_tc_kernel<true, true> : attn_tc_kernel<true, false>)
                  : (mask ? attn_tc_kernel<false, true> : attn_tc_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM takes units from the queue (heaviest first) until it is empty
  const int64_t grid = units < sm_count() ? units : sm_count();
  FPX_CHAIN(kern, static_cast<unsigned>(grid), kThreads, kSmemBytes, s, mq, mk, mv, p, row_ptr,
            col_idx, static_cast<__nv_bfloat16*>(o), lse, t, order, queue_head,
            static_cast<int>(units), vbits, sbits, words, st);
  return cudaGetLastError();
}

}  // namespace fpx
