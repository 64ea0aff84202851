// fpx_common.cuh -- device-side helpers shared by the fpx kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fpx.h"

namespace fpx {

// ------------------------------------------------------------------------------------------
// Workspace layout.  Every workspace starts with a 256-byte status block followed by the
// per-sequence tables; the stage-specific scratch follows, 256-byte aligned.
// ------------------------------------------------------------------------------------------
constexpr size_t kStatusBytes = 256;

struct StatusBlock {
  int code;          // first recorded fpx_status (0 = none)
  int where;         // kernel-specific location of the first error
  int detail0, detail1;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-sequence tables built on the device from cu_seqlens at the start of every stage.
struct SeqTables {
  int32_t* valid;     // 1 iff the device cu_seqlens agree with the host-side sizes
  int32_t* blk_base;  // [S + 1]: first global block of each sequence
  int64_t* tri_base;  // [S + 1]: first causal block pair of each sequence (per head)
};

__host__ __device__ inline size_t seq_tables_bytes(int num_seqs) {
  return 256 + align_up(sizeof(int32_t) * (num_seqs + 1), 256) +
         align_up(sizeof(int64_t) * (num_seqs + 1), 256);
}

__host__ __device__ inline SeqTables seq_tables_at(void* ws, int num_seqs) {
  char* base = static_cast<char*>(ws) + kStatusBytes;
  SeqTables t;
  t.valid = reinterpret_cast<int32_t*>(base);
  t.blk_base = reinterpret_cast<int32_t*>(base + 256);
  t.tri_base =
      reinterpret_cast<int64_t*>(base + 256 + align_up(sizeof(int32_t) * (num_seqs + 1), 256));
  return t;
}

__host__ __device__ inline size_t scratch_offset(int num_seqs) {
  return kStatusBytes + seq_tables_bytes(num_seqs);
}

// Everything a kernel needs to know about the (packed) problem.
struct ProblemDesc {
  const int32_t* cu;   // device cu_seqlens (nullptr => one sequence of total_tokens)
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t hq, hkv, group, d, block;
  int32_t nb_total;    // NB
  int64_t tri_total;   // TRI
  float scale;         // softmax scale of the dequantised dot product
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  // paged K / V (nullptr => K and V are packed like Q): K / V row of token t of key block J of
  // sequence s = page_table[s * pages_per_seq + J] * block + t, pages of `block` tokens
  const int32_t* page_table;
  int32_t pages_per_seq;
  int32_t num_pages;
};

// First K / V row of key block J of sequence s (tok0 = the sequence's first token), or -1 when a
// paged table names a page outside [0, num_pages).
__device__ __forceinline__ int64_t kv_block_row(const ProblemDesc& p, int s, int J, int tok0) {
  if (!p.page_table) return static_cast<int64_t>(tok0) + static_cast<int64_t>(J) * p.block;
  const int pg = p.page_table[static_cast<int64_t>(s) * p.pages_per_seq + J];
  return (pg < 0 || pg >= p.num_pages) ? -1 : static_cast<int64_t>(pg) * p.block;
}

__device__ __forceinline__ void record_error(StatusBlock* st, int code, int where, int d0 = 0,
                                             int d1 = 0) {
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->where = where;
    st->detail0 = d0;
    st->detail1 = d1;
  }
}

__device__ __forceinline__ int seq_start(const ProblemDesc& p, int s) {
  return p.cu ? p.cu[s] : 0;
}
__device__ __forceinline__ int seq_len(const ProblemDesc& p, int s) {
  return p.cu ? p.cu[s + 1] - p.cu[s] : p.total_tokens;
}

// Global block index -> sequence (largest s with blk_base[s] <= b, skipping empty sequences).
__device__ __forceinline__ int seq_of_block(const int32_t* blk_base, int num_seqs, int b) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (blk_base[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------------------------------
// Small numeric helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch.  Every library kernel is launched with programmatic stream
// serialization (launch_chained) and starts with pdl_enter(): it waits until the kernel before it
// on the stream has completed and its writes are visible (griddepcontrol.wait), then lets the
// kernel after it be scheduled (launch_dependents), so that kernel's launch and CTA set-up overlap
// this one's execution instead of following its end.  Without the launch attribute both
// instructions are no-ops.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Upper bound for any single device-side wait.  A correct schedule waits microseconds; the
// bound only turns a broken pipeline into FPX_ERR_TIMEOUT instead of a hung GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

}  // namespace fpx
