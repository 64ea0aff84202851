// fpx_internal.h -- host-side declarations shared by the fpx translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fpx_common.cuh"

namespace fpx {

// Launches kern<<<grid, block, smem, s>>>(args...) with programmatic stream serialization (the
// kernel calls pdl_enter() before it touches anything the previous kernel writes).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// launch_chained in a function returning cudaError_t: returns the error of a failed launch.
// (A kernel name with template arguments is passed in parentheses.)
#define FPX_CHAIN(kern, grid, block, smem, stream, ...)                                        \
  do {                                                                                          \
    const cudaError_t fpx_chain_err_ =                                                          \
        ::fpx::launch_chained(kern, dim3(grid), dim3(block), smem, stream, __VA_ARGS__);       \
    if (fpx_chain_err_ != cudaSuccess) return fpx_chain_err_;                                   \
  } while (0)

// Stage 0 building block, shared by all entry points: per-sequence tables + cu_seqlens checks.
cudaError_t launch_plan(const ProblemDesc& p, SeqTables t, StatusBlock* st, cudaStream_t s);

// fpx_block_scores: pool Q and K (fp32 means into qbar / kbar), then score pooled pairs.
// qlo / klo non-null: the means are stored split as tf32 hi (qbar / kbar) + lo (qlo / klo).
cudaError_t launch_pool(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                        float* qbar, float* kbar, float* qlo, float* klo, SeqTables t,
                        StatusBlock* st, cudaStream_t s);
// Scores on the tensor cores from the split means (qlo / klo non-null; requires
// score_tc_supported), else fp32 CUDA cores from the plain means.
cudaError_t launch_score(const ProblemDesc& p, fpx_dtype dt, const float* qbar, const float* kbar,
                         const float* qlo, const float* klo, float* scores, SeqTables t,
                         StatusBlock* st, cudaStream_t s);
bool score_tc_supported(const ProblemDesc& p);
cudaError_t launch_score_tc(const ProblemDesc& p, const float* qhi, const float* khi,
                            const float* qlo, const float* klo, float* scores, SeqTables t,
                            StatusBlock* st, cudaStream_t s);

// fpx_select: row max + keep count + keep bitmask (mask_words 32-bit words per row), scan into
// row_ptr, emit col_idx from the bitmask.
cudaError_t launch_select(const ProblemDesc& p, const float* scores, float alpha, int sink,
                          int window, int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                          int64_t* nnz_d, float* rowmax, int32_t* counts, int64_t* cta_tot,
                          int* overflow, uint32_t* mask, int mask_words, const float* qn,
                          const float* rad, float alpha_r, SeqTables t, StatusBlock* st,
                          cudaStream_t s);
// Rescue-branch inputs after the pool pass: qnorm [Hq, NB] = ||qbar||, radius [Hkv, NB] = max
// distance of a key of the block from its centroid (qlo / klo: the tf32 remainders, or null).
cudaError_t launch_radius(const ProblemDesc& p, fpx_dtype dt, const void* k, const float* qbar,
                          const float* kbar, const float* qlo, const float* klo, float* qnorm,
                          float* radius, SeqTables t, cudaStream_t s);
// CTAs of the select kernels (each owns 8 rows); the workspace holds one int64 per CTA.
int select_ctas(const ProblemDesc& p);

// [T, H, D] tensor -> 3-D TMA map {D, H, T} with box {128 bytes, 1, 128 rows} and 128B swizzle
// (elem_bytes 1 = u8, 2 = bf16, 4 = fp32); false if the driver rejects it.
bool make_tmap_rows128(CUtensorMap* map, const void* base, int T, int H, int D, int elem_bytes);

// fpx_sparse_prefill: tile schedule, then one of the two attention kernels.
// `units`: schedule the tensor-core kernel's two-head units instead of single CSR rows.  The
// items are sorted by their kept-tile counts in row_ptr (heaviest first inside each KV head);
// *queue_head is reset to 0 for the persistent kernel's work queue.  nb_max = blocks of the
// longest sequence.
cudaError_t launch_order(const ProblemDesc& p, int nb_max, SeqTables t, const int32_t* row_ptr,
                         int32_t* order, int* queue_head, bool units, cudaStream_t s);
cudaError_t launch_attn_simt(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                             const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                             void* o, float* lse, SeqTables t, const int32_t* order,
                             StatusBlock* st, cudaStream_t s);
bool attn_tc_supported(const ProblemDesc& p, fpx_dtype dt);
// Returns cudaSuccess or the first error; `encode_failed` is set if a tensor map was rejected.
// vbits / sbits non-null: the vertical / slash token mask (uint32 [hq][words]) is applied.
cudaError_t launch_attn_tc(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                           const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                           void* o, float* lse, SeqTables t, const int32_t* order,
                           int* queue_head, const uint32_t* vbits, const uint32_t* sbits,
                           int words, StatusBlock* st, cudaStream_t s, bool* encode_failed);

// Query-probe vertical / slash discovery (fpx_probe.cu): zeroes and fills the two bitmasks
// (uint32 [hq][words]).  chunk_base: [num_seqs + 1] int32; partial: float2 [total_chunks * hkv *
// probe_tiles * 128]; bound: float2 [num_seqs * hq * n_probe].
int probe_tiles(const ProblemDesc& p, int n_probe);
size_t probe_smem(int tiles);
cudaError_t launch_probe(const ProblemDesc& p, fpx_dtype dt, const void* q, const void* k,
                         int n_probe, float alpha_v, float alpha_s, int chunk_blocks,
                         int total_chunks, SeqTables t, int32_t* chunk_base, float2* partial,
                         float2* bound, uint32_t* vbits, uint32_t* sbits, int words,
                         StatusBlock* st, cudaStream_t s, bool* encode_failed);
// Candidate key blocks of the vertical / slash attention into the select stage's keep bitmask
// and counts (then launch_select_finish builds the CSR).  vflag / sflag: uint8 [hq * NB] each.
cudaError_t launch_vs_count(const ProblemDesc& p, SeqTables t, const uint32_t* vbits,
                            const uint32_t* sbits, int words, uint8_t* vflag, uint8_t* sflag,
                            int32_t* counts, int64_t* cta_tot, uint32_t* mask, int mask_words,
                            cudaStream_t s);
// The scan and emit kernels of the select stage on counts / mask written by a count kernel.
cudaError_t launch_select_finish(const ProblemDesc& p, int32_t* row_ptr, int32_t* col_idx,
                                 int64_t capacity, int64_t* nnz_d, const int32_t* counts,
                                 int64_t* cta_tot, int* overflow, const uint32_t* mask,
                                 int mask_words, SeqTables t, StatusBlock* st, cudaStream_t s);

}  // namespace fpx
