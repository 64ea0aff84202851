// fpx_probe.cu -- query-probe vertical / slash pattern discovery and the key-block candidate list
// of the attention that consumes it.
//
// FlashPrefill §3 Method ("Instantaneous Pattern Discovery") places uniformly distributed query
// probes to find vertical patterns (the same key columns matter to every query) and slash
// patterns (the same query-key offsets matter everywhere).  The page gives no formula; the
// library implements this reading (token granularity, the page's max-based thresholding as the
// selection rule):
//   probes      m = min(n_probe, n) query tokens of a sequence of n, at ceil((p + 1) n / m) - 1;
//   A[p, j]     the exact causal softmax row of probe p over keys j <= pos_p (per Q head);
//   verticals   key j with max_p A[p, j] >= alpha_v * max_{p,j} A (alpha_v == 0: every key);
//   slashes     offset d with max_p A[p, pos_p - d] >= alpha_s * max_{p,j} A (alpha_s == 0: all).
// (max over keys of the vertical scores and max over offsets of the slash scores are both the
// largest probe probability, max_{p,j} A.)
//
// Both searches are dense contractions of the probe rows with every key, so they run on tcgen05:
// a CTA takes one KV group of one sequence and a chunk of kChunkBlocks key blocks; its probe rows
// (the group's Q heads x probes, up to 4 tiles of 128 rows) sit in shared memory in the 128B-
// swizzled K-major layout, K blocks arrive by TMA into a two-slot ring, and S = Qprobe K^T lands
// in TMEM (one 128-column tile per 128 probe rows).  One thread per probe row then reads its S
// row from TMEM:
//   pass 1 (stats)  running max and sum of 2^x over the chunk (x = scale * log2(e) * logit, keys
//                   j <= pos_p), written as one partial per (chunk, row);
//   reduce          per probe: lse2 = log2 sum 2^x over all chunks; per (sequence, head): the
//                   largest probability max_p 2^(xmax_p - lse2_p); per probe the thresholds of
//                   both selections as logit-domain bounds
//                       A >= alpha * Amax  <=>  x >= lse2_p + log2(alpha) + log2(Amax);
//   pass 2 (mark)   the same S tiles, compared with the two bounds: no exponentials; a key above
//                   the vertical bound sets its bit, an element above the slash bound sets the
//                   bit of its offset pos_p - j (atomicOr, rare by construction).
// Output: two token-granular bitmasks per Q head, uint32 [hq][words], words = ceil(T / 32):
// bit (cu[s] + x) marks key token x of sequence s as a vertical (vert_bits) or offset x as a
// slash (slash_bits).
//
// The attention over the pattern (fpx_vs_prefill) iterates over key blocks that can hold an
// allowed key for some row of the query block and applies the exact token mask inside them:
// block J of row (h, s, I) is a candidate iff it holds a vertical, or a slash offset lies in
// [(I - J) B - B + 1, (I - J) B + B - 1] (the offsets a B x B block pair spans; a superset at a
// ragged tail, where the mask then removes the extra keys).  vs_flags_kernel summarises both per
// (head, block); vs_count_kernel writes the select stage's keep bitmask and counts from them, and
// the select stage's own scan / emit kernels build the CSR.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cmath>
#include <limits>

#include "fpx_internal.h"
#include "fpx_sm100.cuh"

namespace fpx {
namespace probe {

using namespace sm100;

constexpr int kKeys = 128;        // keys per block (one MMA N)
constexpr int kRowsPerTile = 128;  // probe rows per tile (one MMA M)
constexpr int kHeadDim = 128;
constexpr uint32_t kQTileBytesBf16 = kRowsPerTile * kHeadDim * 2;  // 32 KB
constexpr uint32_t kKSlotBytes = kKeys * kHeadDim * 2;             // 32 KB (bf16; e4m3 uses half)
constexpr uint32_t kBoxBytes = 128 * 128;                          // 128 rows x 128 B

// Per tile count: K ring slots and S buffers in TMEM (two S buffers, so that the next block's
// MMA overlaps this block's row work, where two fit in the 512 TMEM columns).
template <int kTiles>
struct PLayout {
  static constexpr int kBufs = kTiles <= 2 ? 2 : 1;
  static constexpr int kSlots = kTiles <= 2 ? 3 : 2;
  static constexpr uint32_t kTmemCols = kBufs * kTiles * 128 <= 128   ? 128
                                        : kBufs * kTiles * 128 <= 256 ? 256
                                                                      : 512;
};

__host__ __device__ constexpr size_t probe_smem_bytes(int tiles) {
  return static_cast<size_t>(tiles) * kQTileBytesBf16 +
         static_cast<size_t>(tiles <= 2 ? 3 : 2) * kKSlotBytes + 256 + 1024;
}

enum PBar { kPKFull = 0, kPKEmpty = 3, kPSFull = 6, kPSFree = 8, kPDrain = 10, kPNumBars = 11 };

template <bool kFp8>
struct PCfg {
  static constexpr uint32_t kElem = kFp8 ? 1 : 2;
  static constexpr uint32_t kRowBytes = kHeadDim * kElem;            // 256 or 128
  static constexpr uint32_t kTileBytes = kRowsPerTile * kRowBytes;   // per 128 rows
  static constexpr int kBoxes = kRowBytes / 128;
  static constexpr int kKStep = kFp8 ? 32 : 16;
  static constexpr int kSteps = kHeadDim / kKStep;
  static constexpr uint32_t kIdesc = make_idesc(kFp8 ? 0 : 1, kFp8 ? 0 : 1, false, 128, 128);
};

template <bool kFp8>
__device__ __forceinline__ uint32_t koff(int kk) {
  constexpr int per_box = 128 / (PCfg<kFp8>::kKStep * PCfg<kFp8>::kElem);
  return (kk / per_box) * kBoxBytes + (kk % per_box) * 32;
}

// Position of probe pp among m probes of a sequence of n tokens: ceil((pp + 1) n / m) - 1.
__device__ __forceinline__ int probe_pos(int pp, int n, int m) {
  return static_cast<int>((static_cast<int64_t>(pp + 1) * n + m - 1) / m) - 1;
}

// Sequence of chunk c: largest s with chunk_base[s] <= c (empty sequences own no chunk).
__device__ __forceinline__ int seq_of_chunk(const int32_t* chunk_base, int num_seqs, int c) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (chunk_base[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// chunk_base[s] = sum over s' < s of ceil(nb_s' / chunk_blocks) (one CTA; tables from the plan).
__global__ void __launch_bounds__(1024) probe_plan_kernel(ProblemDesc p, SeqTables t,
                                                          int chunk_blocks,
                                                          int32_t* __restrict__ chunk_base) {
  pdl_enter();  // after the previous kernel on the stream
  __shared__ int warp_sum[32];
  if (!*t.valid) return;
  const int S = p.num_seqs, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int per = (S + 1023) / 1024;
  const int lo = min(S, tid * per), hi = min(S, lo + per);
  int sum = 0;
  for (int s = lo; s < hi; ++s) {
    const int nb = t.blk_base[s + 1] - t.blk_base[s];
    sum += (nb + chunk_blocks - 1) / chunk_blocks;
  }
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
  for (int s = lo; s < hi; ++s) {
    chunk_base[s] = run;
    const int nb = t.blk_base[s + 1] - t.blk_base[s];
    run += (nb + chunk_blocks - 1) / chunk_blocks;
  }
  if (tid == 1023) chunk_base[S] = warp_sum[31];
}

// Probe rows of one (sequence, KV group) and what the kernels need to know about them.
struct ProbeArgs {
  int n_probe;        // probes requested per sequence (m = min(n_probe, n) are used)
  int tiles;          // ceil(group * n_probe / 128)
  int words;          // bitmask words per head
  int chunk_blocks;   // key blocks per CTA
  int all_v, all_s;   // alpha == 0: every key / offset selected
  float log2_alpha_v, log2_alpha_s;
};

// One pass over a chunk of key blocks for the probe rows of one (sequence, KV group).
// kMark = false: partial (max, sum) of 2^x per row -> partial[(c * hkv + g) * rows_pad + row];
// kMark = true: marks against the bounds bound[(s * hq + h) * n_probe + pp] (float2: vertical,
// slash).
template <bool kFp8, int kTiles, bool kMark>
__global__ void __launch_bounds__(kTiles * 128 + 32, 1)
probe_pass_kernel(const __grid_constant__ CUtensorMap tmK, ProblemDesc p, ProbeArgs a,
                  const uint8_t* __restrict__ q, SeqTables tab,
                  const int32_t* __restrict__ chunk_base, float2* __restrict__ partial,
                  const float2* __restrict__ bound, uint32_t* __restrict__ vbits,
                  uint32_t* __restrict__ sbits, StatusBlock* st) {
  pdl_enter();  // after the previous kernel on the stream
  using C = PCfg<kFp8>;
  using L = PLayout<kTiles>;
  constexpr int kRowThreads = kTiles * 128;
  constexpr int kCtrlWarp = kTiles * 4;
  if (!*tab.valid) return;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_u32);
  const uint32_t off_k = kTiles * C::kTileBytes;
  const uint32_t off_bar = off_k + L::kSlots * kKSlotBytes;
  const uint32_t bar0 = sbase + off_bar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + off_bar + 8 * kPNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + off_bar + 8 * kPNumBars + 4);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, g = blockIdx.y;
  const int s = seq_of_chunk(chunk_base, p.num_seqs, c);
  const int n_s = seq_len(p, s);
  const int tok0 = seq_start(p, s);
  const int nb_s = (n_s + kKeys - 1) / kKeys;
  const int J0 = (c - chunk_base[s]) * a.chunk_blocks;
  const int J1 = min(nb_s, J0 + a.chunk_blocks);
  const int m = min(a.n_probe, n_s);
  const int rows = p.group * a.n_probe;

  if (tid == 0) {
    for (int i = 0; i < L::kSlots; ++i) {
      mbar_init(bar(kPKFull + i), 1);
      mbar_init(bar(kPKEmpty + i), 1);
    }
    for (int i = 0; i < L::kBufs; ++i) {
      mbar_init(bar(kPSFull + i), 1);
      mbar_init(bar(kPSFree + i), kRowThreads / 32);
    }
    mbar_init(bar(kPDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // probe rows -> shared memory (one thread per row), 128B-swizzled K-major like a TMA tile
  const int row = tid;  // valid for tid < kRowThreads
  int pp = 0, hl = 0, pos = -1;
  bool row_valid = false;
  if (tid < kRowThreads) {
    hl = row / a.n_probe;
    pp = row - hl * a.n_probe;
    row_valid = row < rows && pp < m;
    pos = row_valid ? probe_pos(pp, n_s, m) : -1;
    const int tile = row >> 7, r = row & 127;
    const uint32_t dst0 = static_cast<uint32_t>(tile) * C::kTileBytes + r * 128;
    const int4* src = reinterpret_cast<const int4*>(
        q + ((static_cast<int64_t>(tok0) + max(pos, 0)) * p.hq + g * p.group + hl) *
                static_cast<int64_t>(C::kRowBytes));
#pragma unroll
    for (int ch = 0; ch < static_cast<int>(C::kRowBytes / 16); ++ch) {
      const int4 v = row_valid ? __ldg(src + ch) : make_int4(0, 0, 0, 0);
      const int box = ch >> 3, cc = ch & 7;
      *reinterpret_cast<int4*>(gbase + dst0 + box * kBoxBytes + ((cc ^ (r & 7)) << 4)) = v;
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
  if (warp == kCtrlWarp) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kCtrlWarp) {
    // ---- TMA loads of the chunk's K blocks (a kSlots ring) and the QK^T MMAs into kBufs
    //      S buffers (one elected lane) -------------------------------------------------------
    constexpr unsigned kFull = 0xffffffffu;
    const uint64_t qdesc0 = smem_desc_sw128(sbase, 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(sbase + off_k, 16, 1024);
    const int nblk = J1 - J0;
    bool ok = true;
    int loaded = 0;
    auto load_block = [&](int idx) {  // block J0 + idx into ring slot idx % kSlots
      const int slot = idx % L::kSlots;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(kPKFull + slot), C::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(sbase + off_k + slot * kKSlotBytes + bx * kBoxBytes, &tmK,
                      bar(kPKFull + slot), bx * 128 / C::kElem, g, tok0 + (J0 + idx) * kKeys);
      }
      __syncwarp();
    };
    for (; loaded < min(L::kSlots, nblk); ++loaded) load_block(loaded);
    for (int e = 0; e < nblk && ok; ++e) {
      const int slot = e % L::kSlots;
      const int buf = e % L::kBufs;
      if (!__all_sync(kFull, mbar_wait(bar(kPKFull + slot), (e / L::kSlots) & 1, abort_flag))) {
        ok = false;
        break;
      }
      // the row threads must have read block e - kBufs's S out of this buffer
      if (e >= L::kBufs &&
          !__all_sync(kFull, mbar_wait(bar(kPSFree + buf), ((e - L::kBufs) / L::kBufs) & 1,
                                       abort_flag))) {
        ok = false;
        break;
      }
      if (elect_one()) {
        tc_fence_after();
        const uint64_t kdesc = kdesc0 + ((slot * kKSlotBytes) >> 4);
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          const uint64_t qdesc = qdesc0 + ((t * C::kTileBytes) >> 4);
          const uint32_t dcol = tmem + (buf * kTiles + t) * 128;
#pragma unroll
          for (int kk = 0; kk < C::kSteps; ++kk) {
            const uint64_t off = koff<kFp8>(kk) >> 4;
            if (kFp8) mma_f8_ss(dcol, qdesc + off, kdesc + off, C::kIdesc, kk > 0);
            else mma_f16_ss(dcol, qdesc + off, kdesc + off, C::kIdesc, kk > 0);
          }
        }
        mma_commit(bar(kPSFull + buf));
        mma_commit(bar(kPKEmpty + slot));
      }
      __syncwarp();
      // refill: block `loaded` (= e + kSlots - 1 in steady state) takes the slot of block
      // loaded - kSlots <= e - 1, whose MMA went out an iteration ago, after block e's MMA is
      // already queued behind it
      if (loaded < nblk && loaded <= e + L::kSlots - 1) {
        const int prev = loaded - L::kSlots;
        if (!__all_sync(kFull, mbar_wait(bar(kPKEmpty + prev % L::kSlots),
                                         (prev / L::kSlots) & 1, abort_flag))) {
          ok = false;
          break;
        }
        load_block(loaded);
        ++loaded;
      }
    }
    if (!ok) *abort_flag = 1;
    // drain: the loads this warp issued, then every MMA, before TMEM is released
    volatile int never = 0;
    for (int e = max(0, loaded - L::kSlots); e < loaded; ++e)
      mbar_wait(bar(kPKFull + e % L::kSlots), (e / L::kSlots) & 1, &never);
    if (elect_one()) mma_commit(bar(kPDrain));
    mbar_wait(bar(kPDrain), 0, &never);
  } else if (tid < kRowThreads) {
    // ---- one probe row per thread ---------------------------------------------------------
    const int tile = row >> 7;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int h = g * p.group + hl;
    float sl2 = p.scale * 1.4426950408889634f;
    if (kFp8 && row_valid) sl2 *= p.q_scale[h] * p.k_scale[g];
    float mrun = -CUDART_INF_F, lrun = 0.f;
    // marks: bounds in raw score units (s * sl2 >= b  <=>  s >= b / sl2, sl2 > 0)
    float bv = CUDART_INF_F, bs = CUDART_INF_F;
    if (kMark && row_valid) {
      const float2 b = bound[(static_cast<int64_t>(s) * p.hq + h) * a.n_probe + pp];
      bv = a.all_v ? CUDART_INF_F : b.x / sl2;  // alpha == 0 is filled elsewhere
      bs = a.all_s ? CUDART_INF_F : b.y / sl2;
    }
    uint32_t* vrow = vbits + static_cast<int64_t>(h) * a.words;
    uint32_t* srow = sbits + static_cast<int64_t>(h) * a.words;
    const unsigned same_head = kMark ? __match_any_sync(0xffffffffu, hl) : 0u;
    const int leader = __ffs(same_head) - 1;
    bool ok = true;
    for (int e = 0; e < J1 - J0; ++e) {
      const int buf = e % L::kBufs;
      if (!mbar_wait(bar(kPSFull + buf), (e / L::kBufs) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem + (buf * kTiles + tile) * 128 + lane_base;
      const int j0 = (J0 + e) * kKeys;
      const int nvis = row_valid ? min(kKeys, pos - j0 + 1) : 0;  // keys j0 .. pos of this block
      // the S row in two halves of 64 columns (register budget of up to 4 tiles x 128 threads)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[64];
        tmem_ld32(taddr + half * 64, r);
        tmem_ld32(taddr + half * 64 + 32, r + 32);
        tmem_wait_ld(r);
        tmem_wait_ld(r + 32);
        if (half == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kPSFree + buf));  // the buffer may be overwritten
        }
        const int nv = min(64, nvis - half * 64);  // visible columns of this half
        if (!kMark) {
          if (nv <= 0) continue;
          float mx = -CUDART_INF_F;
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j < nv) mx = fmaxf(mx, __uint_as_float(r[j]));
          const float mnew = fmaxf(mrun, mx * sl2);
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j < nv) sum += ex2_approx(fmaf(__uint_as_float(r[j]), sl2, -mnew));
          lrun = lrun * ex2_approx(mrun - mnew) + sum;  // mrun = -inf: 0 * 0
          mrun = mnew;
        } else {
          // Branch-free marks: bit j of (vlo, vhi) / (slo, shi) = column j of this half is
          // above the vertical / slash bound.  Verticals: the key column is the same for every
          // lane, so the head's lanes OR their masks together (a warp holds the probe rows of
          // several heads when n_probe is not a multiple of 32) and the head's first lane sets
          // the bits with one atomicOr per 32-bit word.  Slashes: a lane's columns j map to the
          // consecutive offsets pos - key, so its mask, bit-reversed, is a bit range of the
          // slash row; it is OR-ed in word by word (hits are rare).
          uint32_t vlo = 0, vhi = 0, slo = 0, shi = 0;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float x = __uint_as_float(r[j]);
            const uint32_t vis = j < nv ? 1u : 0u;
            const uint32_t hv = (x >= bv ? 1u : 0u) & vis, hs = (x >= bs ? 1u : 0u) & vis;
            if (j < 32) { vlo |= hv << j; slo |= hs << j; }
            else { vhi |= hv << (j - 32); shi |= hs << (j - 32); }
          }
          vlo = __reduce_or_sync(0xffffffffu & same_head, vlo);
          vhi = __reduce_or_sync(0xffffffffu & same_head, vhi);
          const int kbase = j0 + half * 64;
          if (lane == leader && (vlo | vhi)) {
            // keys kbase .. kbase + 63 at bits vbit0 .. vbit0 + 63 of the head's row
            const int64_t vbit0 = static_cast<int64_t>(tok0) + kbase;
            const int64_t w0 = vbit0 >> 5;
            const int sh = static_cast<int>(vbit0 & 31);
            const uint32_t x0 = vlo << sh;
            const uint32_t x1 = sh ? (vhi << sh) | (vlo >> (32 - sh)) : vhi;
            const uint32_t x2 = sh ? vhi >> (32 - sh) : 0u;
            if (x0) atomicOr(vrow + w0, x0);
            if (x1) atomicOr(vrow + w0 + 1, x1);
            if (x2) atomicOr(vrow + w0 + 2, x2);
          }
          if (slo | shi) {
            // column j <-> offset pos - kbase - j: reversed, bit k <-> offset pos - kbase - 63 + k
            const uint32_t rlo = __brev(shi), rhi = __brev(slo);
            const int64_t sbit0 = static_cast<int64_t>(tok0) + pos - kbase - 63;
            const int64_t w0 = sbit0 >> 5;  // floor (bits below the row's start are zero)
            const int sh = static_cast<int>(sbit0 & 31);
            const uint32_t x0 = rlo << sh;
            const uint32_t x1 = sh ? (rhi << sh) | (rlo >> (32 - sh)) : rhi;
            const uint32_t x2 = sh ? rhi >> (32 - sh) : 0u;
            if (x0) atomicOr(srow + w0, x0);
            if (x1) atomicOr(srow + w0 + 1, x1);
            if (x2) atomicOr(srow + w0 + 2, x2);
          }
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (row == 0) record_error(st, FPX_ERR_TIMEOUT, 50, s, g);
    } else if (!kMark) {
      const int rows_pad = kTiles * 128;
      partial[(static_cast<int64_t>(c) * p.hkv + g) * rows_pad + row] = make_float2(mrun, lrun);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kCtrlWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Per (sequence, Q head): combine each probe's chunk partials into lse2 (log2 sum 2^x), take the
// largest probe probability, and write both selections' logit-domain bounds per probe.  With
// alpha == 0 the selection is every key / offset of the sequence: those bits are set here.
__global__ void __launch_bounds__(512) probe_reduce_kernel(
    ProblemDesc p, ProbeArgs a, SeqTables tab, const int32_t* __restrict__ chunk_base,
    const float2* __restrict__ partial, float2* __restrict__ bound, uint32_t* __restrict__ vbits,
    uint32_t* __restrict__ sbits) {
  pdl_enter();  // after the previous kernel on the stream
  __shared__ float warp_max[16];
  if (!*tab.valid) return;
  const int s = blockIdx.x, h = blockIdx.y;
  const int g = h / p.group, hl = h - g * p.group;
  const int n_s = seq_len(p, s), tok0 = seq_start(p, s);
  const int m = min(a.n_probe, n_s);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int rows_pad = a.tiles * 128;
  float lse2 = -CUDART_INF_F, amax2 = -CUDART_INF_F;
  if (tid < m) {
    const int row = hl * a.n_probe + tid;
    float M = -CUDART_INF_F;
    for (int c = chunk_base[s]; c < chunk_base[s + 1]; ++c)
      M = fmaxf(M, partial[(static_cast<int64_t>(c) * p.hkv + g) * rows_pad + row].x);
    float L = 0.f;
    for (int c = chunk_base[s]; c < chunk_base[s + 1]; ++c) {
      const float2 v = partial[(static_cast<int64_t>(c) * p.hkv + g) * rows_pad + row];
      if (v.y > 0.f) L += v.y * exp2f(v.x - M);
    }
    lse2 = M + log2f(L);   // the probe sees key 0 at least: L >= 1
    amax2 = M - lse2;      // log2 of the probe's largest probability
  }
  float mx = amax2;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
  if (lane == 0) warp_max[wid] = mx;
  __syncthreads();
  if (tid == 0) {
    float v = -CUDART_INF_F;
    for (int i = 0; i < (blockDim.x + 31) / 32; ++i) v = fmaxf(v, warp_max[i]);
    warp_max[0] = v;
  }
  __syncthreads();
  const float amax_all = warp_max[0];  // log2 of max_{p,j} A for this (sequence, head)
  if (tid < a.n_probe) {
    float2 b = make_float2(CUDART_INF_F, CUDART_INF_F);
    if (tid < m) b = make_float2(lse2 + a.log2_alpha_v + amax_all, lse2 + a.log2_alpha_s + amax_all);
    bound[(static_cast<int64_t>(s) * p.hq + h) * a.n_probe + tid] = b;
  }
  // alpha == 0: the whole sequence [tok0, tok0 + n_s) in the bitmask (boundary words shared with
  // the neighbouring sequences are OR-ed)
  for (int sel = 0; sel < 2; ++sel) {
    if (!(sel == 0 ? a.all_v : a.all_s) || n_s == 0) continue;
    uint32_t* rowp = (sel == 0 ? vbits : sbits) + static_cast<int64_t>(h) * a.words;
    const int64_t b0 = tok0, b1 = static_cast<int64_t>(tok0) + n_s;  // [b0, b1)
    for (int64_t wd = (b0 >> 5) + tid; wd <= ((b1 - 1) >> 5); wd += blockDim.x) {
      const int64_t lo = max(b0, wd * 32), hi = min(b1, wd * 32 + 32);
      const uint32_t bits = static_cast<uint32_t>(hi - lo) == 32
                                ? 0xffffffffu
                                : ((1u << (hi - lo)) - 1u) << (lo - wd * 32);
      atomicOr(rowp + wd, bits);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Key-block candidates of the vertical / slash attention.
//   vflag[h * NB + b] = 1 iff key block b holds a vertical of head h;
//   sflag[h * NB + blk_base[s] + d] = 1 iff an offset in [d B - B + 1, d B + B - 1] (clipped to
//   [0, n_s - 1]) is a slash of head h in sequence s.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ bool any_bit(const uint32_t* __restrict__ row, int64_t lo, int64_t hi) {
  // any set bit in [lo, hi] (inclusive), lo <= hi
  for (int64_t wd = lo >> 5; wd <= (hi >> 5); ++wd) {
    const int64_t a = max(lo, wd * 32) - wd * 32, b = min(hi, wd * 32 + 31) - wd * 32;
    const uint32_t mask = (b - a == 31) ? 0xffffffffu : (((1u << (b - a + 1)) - 1u) << a);
    if (__ldg(row + wd) & mask) return true;
  }
  return false;
}

__global__ void vs_flags_kernel(ProblemDesc p, SeqTables tab, int words,
                                const uint32_t* __restrict__ vbits,
                                const uint32_t* __restrict__ sbits, uint8_t* __restrict__ vflag,
                                uint8_t* __restrict__ sflag) {
  pdl_enter();  // after the previous kernel on the stream
  if (!*tab.valid) return;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(p.hq) * p.nb_total) return;
  const int h = static_cast<int>(i / p.nb_total);
  const int b = static_cast<int>(i - static_cast<int64_t>(h) * p.nb_total);
  const int s = seq_of_block(tab.blk_base, p.num_seqs, b);
  const int J = b - tab.blk_base[s];
  const int n_s = seq_len(p, s);
  const int64_t tok0 = seq_start(p, s);
  const int B = p.block;
  const uint32_t* vrow = vbits + static_cast<int64_t>(h) * words;
  const uint32_t* srow = sbits + static_cast<int64_t>(h) * words;
  const int64_t klo = static_cast<int64_t>(J) * B;
  const int64_t khi = (klo + B < n_s ? klo + B : static_cast<int64_t>(n_s)) - 1;
  vflag[i] = any_bit(vrow, tok0 + klo, tok0 + khi) ? 1 : 0;
  const int64_t dlo0 = static_cast<int64_t>(J) * B - B + 1;
  const int64_t dhi0 = static_cast<int64_t>(J) * B + B - 1;
  const int64_t dlo = dlo0 > 0 ? dlo0 : 0;
  const int64_t dhi = dhi0 < n_s - 1 ? dhi0 : static_cast<int64_t>(n_s) - 1;
  sflag[i] = (dlo <= dhi && any_bit(srow, tok0 + dlo, tok0 + dhi)) ? 1 : 0;
}

constexpr int kVsWarps = 8;  // rows per CTA, as the select stage's kernels expect

// Row r = (h, s, I): candidate J <= I iff vflag(J) or sflag(I - J); writes the keep bitmask and
// counts in the select stage's layout (its scan and emit kernels build the CSR).
__global__ void __launch_bounds__(kVsWarps * 32) vs_count_kernel(
    ProblemDesc p, SeqTables tab, const uint8_t* __restrict__ vflag,
    const uint8_t* __restrict__ sflag, int32_t* __restrict__ counts,
    int64_t* __restrict__ cta_tot, uint32_t* __restrict__ mask, int mask_words) {
  pdl_enter();  // after the previous kernel on the stream
  __shared__ int w_tot[kVsWarps];
  if (!*tab.valid) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int R = p.hq * p.nb_total;
  const int r = blockIdx.x * kVsWarps + warp;
  int cnt = 0;
  if (r < R) {
    const int h = r / p.nb_total, b = r - h * p.nb_total;
    const int s = seq_of_block(tab.blk_base, p.num_seqs, b);
    const int first = tab.blk_base[s];
    const int I = b - first;
    const uint8_t* vf = vflag + static_cast<int64_t>(h) * p.nb_total + first;
    const uint8_t* sf = sflag + static_cast<int64_t>(h) * p.nb_total + first;
    for (int j0 = 0; j0 <= I; j0 += 32) {
      const int J = j0 + lane;
      const bool kp = J <= I && (vf[J] | sf[I - J]);
      const unsigned bal = __ballot_sync(0xffffffffu, kp);
      if (lane == 0 && (j0 >> 5) < mask_words)
        mask[static_cast<int64_t>(r) * mask_words + (j0 >> 5)] = bal;
      cnt += __popc(bal);
    }
    if (lane == 0) counts[r] = cnt;
  }
  if (lane == 0) w_tot[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t t = 0;
#pragma unroll
    for (int i = 0; i < kVsWarps; ++i) t += w_tot[i];
    cta_tot[blockIdx.x] = t;
  }
}

}  // namespace probe

// ---- host side --------------------------------------------------------------------------------

int probe_tiles(const ProblemDesc& p, int n_probe) { return (p.group * n_probe + 127) / 128; }

size_t probe_smem(int tiles) { return probe::probe_smem_bytes(tiles); }

template <bool kFp8, int kTiles, bool kMark>
static cudaError_t launch_pass_t(const CUtensorMap& mk, const ProblemDesc& p,
                                 const probe::ProbeArgs& a, const void* q, SeqTables t,
                                 const int32_t* chunk_base, int total_chunks, float2* partial,
                                 const float2* bound, uint32_t* vb, uint32_t* sb, StatusBlock* st,
                                 cudaStream_t s) {
  auto kern = probe::probe_pass_kernel<kFp8, kTiles, kMark>;
  const size_t smem = probe::probe_smem_bytes(kTiles);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  FPX_CHAIN(kern, dim3(total_chunks, p.hkv), kTiles * 128 + 32, smem, s, mk, p, a,
            static_cast<const uint8_t*>(q), t, chunk_base, partial, bound, vb, sb, st);
  return cudaGetLastError();
}

template <bool kMark>
static cudaError_t launch_pass(const CUtensorMap& mk, const ProblemDesc& p, bool fp8,
                               const probe::ProbeArgs& a, const void* q, SeqTables t,
                               const int32_t* chunk_base, int total_chunks, float2* partial,
                               const float2* bound, uint32_t* vb, uint32_t* sb, StatusBlock* st,
                               cudaStream_t s) {
#define FPX_PASS(F, T)                                                                          \
  return launch_pass_t<F, T, kMark>(mk, p, a, q, t, chunk_base, total_chunks, partial, bound,   \
                                    vb, sb, st, s)
  switch (a.tiles) {
    case 1: if (fp8) FPX_PASS(true, 1); else FPX_PASS(false, 1);
    case 2: if (fp8) FPX_PASS(true, 2); else FPX_PASS(false, 2);
    case 3: if (fp8) FPX_PASS(true, 3); else FPX_PASS(false, 3);
    default: if (fp8) FPX_PASS(true, 4); else FPX_PASS(false, 4);
  }
#undef FPX_PASS
}

cudaError_t launch_probe(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                         int n_probe, float alpha_v, float alpha_s, int chunk_blocks,
                         int total_chunks, SeqTables t, int32_t* chunk_base, float2* partial,
                         float2* bound, uint32_t* vbits, uint32_t* sbits, int words,
                         StatusBlock* st, cudaStream_t s, bool* encode_failed) {
  *encode_failed = false;
  const bool fp8 = dt == FPX_E4M3;
  probe::ProbeArgs a;
  a.n_probe = n_probe;
  a.tiles = probe_tiles(p, n_probe);
  a.words = words;
  a.chunk_blocks = chunk_blocks;
  a.all_v = alpha_v == 0.f;
  a.all_s = alpha_s == 0.f;
  a.log2_alpha_v = alpha_v > 0.f ? std::log2(alpha_v) : -std::numeric_limits<float>::infinity();
  a.log2_alpha_s = alpha_s > 0.f ? std::log2(alpha_s) : -std::numeric_limits<float>::infinity();
  const size_t bytes = sizeof(uint32_t) * static_cast<size_t>(p.hq) * words;
  cudaError_t e = cudaMemsetAsync(vbits, 0, bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(sbits, 0, bytes, s);
  if (e != cudaSuccess || p.nb_total == 0) return e;
  FPX_CHAIN(probe::probe_plan_kernel, 1, 1024, 0, s, p, t, chunk_blocks, chunk_base);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap mk;
  if (!make_tmap_rows128(&mk, k, p.total_tokens, p.hkv, p.d, fp8 ? 1 : 2)) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  if ((e = launch_pass<false>(mk, p, fp8, a, q, t, chunk_base, total_chunks, partial, nullptr,
                              vbits, sbits, st, s)) != cudaSuccess)
    return e;
  FPX_CHAIN(probe::probe_reduce_kernel, dim3(p.num_seqs, p.hq), 512, 0, s, p, a, t, chunk_base,
            partial, bound, vbits, sbits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.all_v && a.all_s) return cudaSuccess;
  return launch_pass<true>(mk, p, fp8, a, q, t, chunk_base, total_chunks, partial, bound, vbits,
                           sbits, st, s);
}

cudaError_t launch_vs_count(const ProblemDesc& p, SeqTables t, const uint32_t* vbits,
                            const uint32_t* sbits, int words, uint8_t* vflag, uint8_t* sflag,
                            int32_t* counts, int64_t* cta_tot, uint32_t* mask, int mask_words,
                            cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(p.hq) * p.nb_total;
  if (R == 0) return cudaSuccess;
  FPX_CHAIN(probe::vs_flags_kernel, static_cast<unsigned>((R + 255) / 256), 256, 0, s, p, t, words,
            vbits, sbits, vflag, sflag);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  FPX_CHAIN(probe::vs_count_kernel,
            static_cast<unsigned>((R + probe::kVsWarps - 1) / probe::kVsWarps),
            probe::kVsWarps * 32, 0, s, p, t, vflag, sflag, counts, cta_tot, mask, mask_words);
  return cudaGetLastError();
}

}  // namespace fpx
