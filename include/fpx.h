/*
 * fpx.h -- C ABI of the dynamic block-sparse pooled prefill attention library (sm_100a).
 *
 * The library runs, for one causal prefill (optionally a packed varlen batch), the three stages
 * of FlashPrefill ("FlashPrefill: Instantaneous Pattern Discovery and Thresholding for
 * Ultra-Fast Long-Context Prefilling", App. B "Detailed Implementation"):
 *
 *   fpx_block_scores   Instantaneous Pattern Discovery: mean-pool Q and K over B-token blocks
 *                      and score every pooled query block against every causally valid pooled
 *                      key block (§3 Method, "Block Approximation for Kernel Optimization").
 *   fpx_select         Max-based Dynamic Thresholding and Block Selection: keep block J of row I
 *                      iff its row-normalised score reaches alpha times the row maximum, OR the
 *                      sink / local-window masks, restricted to J <= I; compress to CSR (§3,
 *                      "Max-based Dynamic Thresholding"; App. B).
 *   fpx_sparse_prefill Block Sparse Attention: exact online-softmax attention over the kept
 *                      blocks only, token-causal inside the diagonal block; O and per-row LSE
 *                      (App. B, "Block Sparse Attention").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layouts.  Q is [T, Hq, D], K and V are [T, Hkv, D], row-major and contiguous ("packed THD"),
 *   base addresses 16-byte aligned (fp8 / bf16 / fp32 elements).  Query head h reads KV head
 *   h / (Hq / Hkv).  A packed batch is described by cu_seqlens (cu[0] = 0, non-decreasing,
 *   cu[S] = T); blocks restart at every sequence start and never cross a sequence boundary.
 *   nb_s = ceil(n_s / B) blocks per sequence, NB = sum_s nb_s, TRI = sum_s nb_s (nb_s + 1) / 2.
 * Scores.  fp32, triangular-packed, one row per (h, s, I): row (h, s, I) starts at element
 *   h * TRI + tri_base[s] + I (I + 1) / 2 and holds J = 0..I, where tri_base[s] is the sum of
 *   nb (nb + 1) / 2 over the sequences before s.
 * CSR.  Rows r = h * NB + block_base[s] + I (i.e. ordered (h, s, I)); row_ptr int32 [R + 1]
 *   with R = Hq * NB; col_idx int32 lists key-block indices local to the sequence, ascending.
 * Ownership.  The caller owns every buffer.  No entry point allocates, frees or synchronises
 *   (except fpx_query_status, which synchronises the stream it is given).  All work is enqueued
 *   on the caller's stream; the library keeps no state between calls and is re-entrant.
 *   Hence every entry point but fpx_query_status can be captured in a CUDA graph (stream
 *   capture) and replayed once it has run eagerly on the device (a first call resolves the
 *   driver's tensor-map encoder and, for fpx_select_noalloc, the scratch address); the
 *   kernels' programmatic dependent launches become graph edges.
 *   A replay reads the buffers' contents at replay time, so new inputs copied into the
 *   captured buffers give that input's result.
 * Workspaces.  Each entry point takes a device workspace of at least fpx_workspace_bytes()
 *   bytes (256-byte aligned).  Its first 256 bytes are a status block: kernels record the first
 *   device-side error there (bounded-wait timeout, malformed cu_seqlens or CSR, capacity); the
 *   record is sticky until fpx_clear_status().  One buffer of the largest size may serve all
 *   three stages on one stream.  Zero it (fpx_clear_status) before first use.
 * Errors.  Argument errors are found on the host before anything is launched and return a
 *   negative fpx_status; launch failures return FPX_ERR_CUDA.  Device-side conditions are read
 *   with fpx_query_status().  Nothing traps on the device and no exception crosses the ABI.
 */
#ifndef FPX_H_
#define FPX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* fpx_stream_t;

typedef enum {
  FPX_OK = 0,
  FPX_ERR_INVALID_ARG = -1,  /* null pointer, bad shape, bad cu_seqlens, NaN/negative alpha  */
  FPX_ERR_UNSUPPORTED = -2,  /* dtype / head dim / block size / index range not supported    */
  FPX_ERR_ALIGNMENT = -3,    /* a pointer is not aligned as documented                      */
  FPX_ERR_CAPACITY = -4,     /* workspace or col_idx capacity too small                      */
  FPX_ERR_CUDA = -5,         /* a CUDA runtime / driver call or a launch failed              */
  FPX_ERR_TIMEOUT = -6,      /* a bounded device-side wait expired (recorded in the status)  */
  FPX_ERR_DEVICE_INPUT = -7  /* device data was malformed (cu_seqlens, CSR index > row block) */
} fpx_status;

typedef enum { FPX_F32 = 0, FPX_BF16 = 1, FPX_E4M3 = 2 } fpx_dtype;

typedef struct {
  int32_t num_seqs;            /* >= 1 (1 when cu_seqlens_d is NULL)                           */
  const int32_t* cu_seqlens_d; /* device [num_seqs + 1]; NULL => one sequence of total_tokens   */
  const int32_t* cu_seqlens_h; /* host mirror of cu_seqlens_d (sizes grids and outputs); NULL
                                  iff cu_seqlens_d is NULL.  Must equal the device copy.        */
  int32_t total_tokens;        /* T >= 0                                                        */
  int32_t hq, hkv;             /* query / KV heads, hq % hkv == 0, both >= 1                    */
  int32_t d;                   /* head dim: 64 or 128                                           */
  int32_t block;               /* B: power of two in [16, 128]                                  */
  fpx_dtype dtype;             /* storage type of Q, K, V                                       */
  const float* q_scale_d;      /* FPX_E4M3 only: device fp32 [hq] dequantisation scales, else NULL */
  const float* k_scale_d;      /* FPX_E4M3 only: device fp32 [hkv]                              */
  const float* v_scale_d;      /* FPX_E4M3 only: device fp32 [hkv]                              */
  float softmax_scale;         /* scale of the dequantised dot products; <= 0 => 1/sqrt(d)      */
} fpx_problem;

/* Sizes.  Each returns 0 for an invalid problem. */
size_t fpx_num_blocks(const fpx_problem* p);   /* NB                                           */
size_t fpx_scores_elems(const fpx_problem* p); /* hq * TRI fp32 elements of the scores buffer  */
size_t fpx_rows(const fpx_problem* p);         /* R = hq * NB; row_ptr has R + 1 entries       */
size_t fpx_max_nnz(const fpx_problem* p);      /* hq * TRI: col_idx entries when alpha == 0    */

/* Workspace bytes for stage `which`: 0 = fpx_block_scores, 1 = fpx_select,
 * 2 = fpx_sparse_prefill, -1 = the maximum of the three. */
size_t fpx_workspace_bytes(const fpx_problem* p, int which);

/* Zero the status block of a workspace (async on `stream`). */
fpx_status fpx_clear_status(void* ws, fpx_stream_t stream);

/* Synchronise `stream`, then return the first device-side error recorded in the workspace's
 * status block (FPX_OK if none).  The record is left in place. */
fpx_status fpx_query_status(const void* ws, fpx_stream_t stream);

const char* fpx_status_string(fpx_status s);

/*
 * Stage 1 -- Instantaneous Pattern Discovery (FlashPrefill §3 "Instantaneous Pattern Discovery"
 * and "Block Approximation for Kernel Optimization"; App. B).
 *   q, k    device, [T, Hq, D] and [T, Hkv, D] in p->dtype (e4m3 codes for FPX_E4M3).
 *   scores  device fp32 [hq * TRI] (layout above):
 *           scores(h, s, I, J) = scale * <mean_{i in I} q_i, mean_{j in J} k_j>  for J <= I,
 *           means over the valid rows of each block (a tail block averages the rows it has),
 *           scale = softmax_scale (dequantised: times q_scale[h] * k_scale[h / g] for e4m3).
 *   ws      device workspace >= fpx_workspace_bytes(p, 0); holds the pooled vectors.
 */
fpx_status fpx_block_scores(const fpx_problem* p, const void* q, const void* k, float* scores,
                            void* ws, size_t ws_bytes, fpx_stream_t stream);

/*
 * Stage 2 -- Max-based Dynamic Thresholding and Block Selection (FlashPrefill §3 "Max-based
 * Dynamic Thresholding"; App. B "Dynamic Thresholding and Block Selection").
 *   For each row (h, s, I) with m = max_{J <= I} scores(h, s, I, J), key block J <= I is kept iff
 *     alpha == 0  or  expf(score - m) >= alpha  (the row-softmax ratio P_IJ / max_J P_IJ)
 *     or J < sink_blocks  or  J > I - window_blocks.
 *   alpha >= 0 (NaN rejected); sink_blocks, window_blocks >= 0.
 *   row_ptr   device int32 [R + 1], written (row_ptr[0] = 0, row_ptr[R] = nnz).
 *   col_idx   device int32 [col_capacity]; kept J per row, ascending.  If nnz > col_capacity
 *             nothing is written to col_idx, row_ptr is written all zero (an empty CSR, which
 *             fpx_sparse_prefill reads as rows with no key) and FPX_ERR_CAPACITY is recorded in
 *             the status.
 *   nnz_d     device int64 [1] (may be NULL): total kept blocks (on overflow: the capacity the
 *             selection needs).
 *   ws        device workspace >= fpx_workspace_bytes(p, 1).
 */
fpx_status fpx_select(const fpx_problem* p, const float* scores, float alpha,
                      int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                      int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d, void* ws,
                      size_t ws_bytes, fpx_stream_t stream);

/*
 * Stage 3 -- Block Sparse Attention (FlashPrefill App. B "Block Sparse Attention").
 *   For Q head h and query token i (local position, block I = i / B) of sequence s:
 *     l_j = scale * <q_i, k_j>  over key tokens j of the blocks listed in CSR row (h, s, I), j <= i
 *     lse_i = ln sum_j exp(l_j),   o_i = sum_j exp(l_j - lse_i) v_j
 *   (dequantised values for e4m3).  A row with no key gets o = 0 and lse = -inf.
 *   q, k, v   device, layouts above.
 *   row_ptr, col_idx  CSR as written by fpx_select (any CSR with indices in [0, I] and no
 *             duplicates is accepted; an index outside [0, I] is skipped and recorded as
 *             FPX_ERR_DEVICE_INPUT).
 *   o         device [T, Hq, D]: bf16 for FPX_BF16 and FPX_E4M3 inputs, fp32 for FPX_F32.
 *   lse       device fp32 [Hq, T], natural log (may be NULL).
 *   ws        device workspace >= fpx_workspace_bytes(p, 2) (holds the tile schedule).
 */
fpx_status fpx_sparse_prefill(const fpx_problem* p, const void* q, const void* k, const void* v,
                              const int32_t* row_ptr, const int32_t* col_idx, void* o,
                              float* lse, void* ws, size_t ws_bytes, fpx_stream_t stream);

/*
 * Paged K / V (FlashPrefill V2 abstract: native paged KV cache and continuous batching, as
 * inference servers keep the cache).  K and V live in a cache of fixed-size pages of `block`
 * tokens, [num_pages, block, hkv, d] in the problem's dtype (the same element layout as a
 * packed [num_pages * block, hkv, d] tensor, 16-byte aligned); Q stays packed by cu_seqlens.
 *   block_table_d  device int32 [num_seqs, pages_per_seq]: entry (s, J) is the page holding key
 *                  block J of sequence s (tokens J * block .. of that sequence); entries with
 *                  J >= nb_s are never read.  pages_per_seq >= the longest sequence's nb_s.
 *   num_pages      pages in the cache (num_pages * block <= INT32_MAX).
 * Rows of a sequence's last page beyond its length must hold finite values (they are multiplied
 * by zero).  A page index outside [0, num_pages) is recorded as FPX_ERR_DEVICE_INPUT and read as
 * zeros.  Same results as the packed entry points on the same data, bit for bit.
 */
typedef struct {
  const int32_t* block_table_d;
  int32_t pages_per_seq;
  int32_t num_pages;
} fpx_paged_kv;

/* fpx_block_scores with K read from the paged cache (any dtype / d / block). */
fpx_status fpx_block_scores_paged(const fpx_problem* p, const void* q, const void* k_cache,
                                  const fpx_paged_kv* kv, float* scores, void* ws,
                                  size_t ws_bytes, fpx_stream_t stream);

/* fpx_sparse_prefill with K and V read from the paged caches.  Tensor-core path only (bf16 or
 * e4m3, d = 128, block = 128; fpx_attention_path(p) == 1), else FPX_ERR_UNSUPPORTED. */
fpx_status fpx_sparse_prefill_paged(const fpx_problem* p, const void* q, const void* k_cache,
                                    const void* v_cache, const fpx_paged_kv* kv,
                                    const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                    float* lse, void* ws, size_t ws_bytes, fpx_stream_t stream);

/*
 * Radius rescue branch (the RBS-Attention abstract listed on the FlashPrefill page: a block
 * centroid may hide a highly relevant token -- "mean dilution"; a rescue branch driven by the
 * maximum key-block radius, thresholded independently and OR-ed with the centroid branch).  The
 * page gives no formula; this library implements the Cauchy-Schwarz reading:
 *   radius r_J = max over the valid tokens j of block J of || k_j - mean_J k ||_2 (per KV head),
 *   u_IJ = s_IJ + scale * || mean_I q ||_2 * r_J  >= scale * <mean_I q, k_j> for every j in J,
 *   rescue keep = alpha_rescue == 0 or exp(u_IJ - max_J' u_IJ') >= alpha_rescue (> 1: none),
 *   final keep = the fpx_select keep OR the rescue keep (J <= I).
 *
 * fpx_block_scores_rescue: fpx_block_scores (kv NULL: packed K, else the paged cache of
 *   fpx_block_scores_paged) that also writes qnorm fp32 [hq, NB] (h * NB + b: || mean q ||) and
 *   radius fp32 [hkv, NB] (kvh * NB + b), reading K a second time.  Workspace: stage 0.
 */
fpx_status fpx_block_scores_rescue(const fpx_problem* p, const void* q, const void* k,
                                   const fpx_paged_kv* kv, float* scores, float* qnorm,
                                   float* radius, void* ws, size_t ws_bytes,
                                   fpx_stream_t stream);

/* fpx_select with the rescue branch OR-ed in; alpha_rescue >= 0 (NaN: FPX_ERR_INVALID_ARG).
 * Same outputs, workspace (stage 1) and device-side conditions as fpx_select. */
fpx_status fpx_select_rescue(const fpx_problem* p, const float* scores, const float* qnorm,
                             const float* radius, float alpha, float alpha_rescue,
                             int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                             int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d, void* ws,
                             size_t ws_bytes, fpx_stream_t stream);

/*
 * Query-probe vertical / slash pattern discovery (FlashPrefill §3 Method, "Instantaneous Pattern
 * Discovery": uniformly distributed query probes find the vertical and slash patterns; §1
 * Introduction names the three pattern types).  The page gives no formula; the library
 * implements this reading, per sequence s of n tokens and Q head h:
 *   probes   m = min(n_probe, n) query tokens at pos_p = ceil((p + 1) n / m) - 1, p < m;
 *   A[p, j]  the exact causal softmax row of probe p: softmax over keys j <= pos_p of
 *            scale * <q_pos_p, k_j> (dequantised values for e4m3);
 *   Amax     max over p and j of A[p, j];
 *   vertical key j   iff alpha_v == 0 or max_p A[p, j] >= alpha_v * Amax;
 *   slash offset d   iff alpha_s == 0 or max_p A[p, pos_p - d] >= alpha_s * Amax
 *   (the page's max-based threshold, applied to the probes' attention).
 * Output, a token-granular index in bitmask form: vert_bits and slash_bits, device uint32
 *   [hq * words] each with words = fpx_pattern_words(p) = ceil(T / 32); bit b of head h is word
 *   h * words + b / 32, bit b % 32; bit cu[s] + x marks key token x (vert_bits) or offset x
 *   (slash_bits) of sequence s.  Both arrays are overwritten (bits of other sequences included).
 * Limits: bf16 or e4m3, d = 128, block = 128 (fpx_attention_path(p) == 1); 1 <= n_probe and
 *   (hq / hkv) * n_probe <= 512, else FPX_ERR_UNSUPPORTED.  alpha_v, alpha_s >= 0 (NaN:
 *   FPX_ERR_INVALID_ARG).
 * ws: device workspace >= fpx_vs_workspace_bytes(p, n_probe) (serves all three entry points of
 *   this path).
 */
size_t fpx_pattern_words(const fpx_problem* p);
size_t fpx_vs_workspace_bytes(const fpx_problem* p, int32_t n_probe);
fpx_status fpx_probe_patterns(const fpx_problem* p, const void* q, const void* k,
                              int32_t n_probe, float alpha_v, float alpha_s, uint32_t* vert_bits,
                              uint32_t* slash_bits, void* ws, size_t ws_bytes,
                              fpx_stream_t stream);

/*
 * Key-block candidates of the vertical / slash attention: CSR (same layout and capacity rules as
 * fpx_select) listing, for every row (h, s, I), the key blocks J <= I that can hold a key some
 * query of block I attends: J holds a vertical of head h, or a slash offset of head h lies in
 * [(I - J) B - B + 1, (I - J) B + B - 1].  Any bitmasks in the layout above are accepted.
 */
fpx_status fpx_vs_select(const fpx_problem* p, const uint32_t* vert_bits,
                         const uint32_t* slash_bits, int32_t* row_ptr, int32_t* col_idx,
                         int64_t col_capacity, int64_t* nnz_d, void* ws, size_t ws_bytes,
                         fpx_stream_t stream);

/*
 * Exact attention under the vertical / slash token mask: query token i (local) of sequence s,
 * Q head h attends key j <= i iff bit cu[s] + j of vert_bits[h] or bit cu[s] + (i - j) of
 * slash_bits[h] is set, among the key blocks its CSR row (h, s, i / B) lists (a list from
 * fpx_vs_select covers every such key).  O and LSE as fpx_sparse_prefill; a row that no key
 * reaches gets O = 0 and LSE = -inf.  Tensor-core path only (fpx_attention_path(p) == 1).
 */
fpx_status fpx_vs_prefill(const fpx_problem* p, const void* q, const void* k, const void* v,
                          const uint32_t* vert_bits, const uint32_t* slash_bits,
                          const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                          void* ws, size_t ws_bytes, fpx_stream_t stream);

/*
 * Allocation-free variant of fpx_select (the paper has no counterpart; it exists for callers).
 *   Some callers cannot allocate device memory where they run: a plugin whose host framework
 *   owns all device memory and offers no scratch buffer, or latency-critical code that must not
 *   call cudaMalloc because an allocation can synchronise the device.  This entry point takes no
 *   workspace: the stage's scratch lives in one fixed device array inside the library of
 *   fpx_select_noalloc_max_bytes() bytes (2 MiB), which every GPU that loads the library holds
 *   until the process exits.  The caller still owns scores, row_ptr, col_idx and nnz_d.
 *   Same arguments and results as fpx_select, without ws / ws_bytes.
 *   Limits: the problem's fpx_workspace_bytes(p, 1) must not exceed the array (9 + 4 *
 *   ceil(nb_max / 32) bytes per query-block row, nb_max = blocks of the longest sequence: about
 *   160,000 rows Hq * NB when no sequence exceeds 32 blocks, about 28,000 at 512 blocks);
 *   larger problems return FPX_ERR_CAPACITY before anything is launched.  An invalid or unsupported problem returns FPX_ERR_INVALID_ARG.
 *   Device-side conditions are visible through the outputs: nnz > col_capacity means nothing was
 *   written to col_idx and row_ptr is all zero; device cu_seqlens that disagree with the host
 *   mirror give an empty CSR with nnz 0.
 *   The first successful call on a device looks up the array's device address (with that device
 *   current) and keeps it for the life of the process; a failed lookup is retried by the next
 *   call.  Make that first call before any stream capture.  A cudaDeviceReset after it is not
 *   supported (the kept address would be stale).  All calls on a device share the array and each
 *   call re-zeroes the part that must start at zero: calls whose work overlaps on the GPU
 *   (unordered streams) race on it.
 */
fpx_status fpx_select_noalloc(const fpx_problem* p, const float* scores, float alpha,
                              int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d,
                              fpx_stream_t stream);
size_t fpx_select_noalloc_max_bytes(void);

/*
 * Diagnostic for failure detection (the paper has no counterpart).  Launches one CTA that waits,
 * with the same bounded-wait loop the pipeline barriers of fpx_sparse_prefill use, on an
 * mbarrier phase that nothing completes.  The wait gives up after limit_ns nanoseconds
 * (0 < limit_ns <= 2e9) and records FPX_ERR_TIMEOUT in the status block of `ws` (any workspace,
 * 256-byte aligned); the CUDA context stays usable.  Returns a launch status only.
 */
fpx_status fpx_diag_bounded_wait(void* ws, uint64_t limit_ns, fpx_stream_t stream);

/*
 * Diagnostic (the paper has no counterpart): y[i] = 2^x[i] evaluated with the FMA-pipe
 * exponential that fpx_sparse_prefill's softmax uses for a share of its elements (range
 * reduction x = n + f, |f| <= 1/2, a degree-3 minimax polynomial for 2^f, n added to the
 * exponent field).  Relative error <= 7.5e-5 for -125 <= x <= 8 (the softmax's range); x below
 * -125 gives 2^-125 * 2^0 (a vanishing weight).  x, y: device fp32 [n].  Returns a launch status.
 */
fpx_status fpx_diag_exp2(const float* x, float* y, int64_t n, fpx_stream_t stream);

/* Which attention kernel fpx_sparse_prefill uses for this problem: 1 = the tcgen05/TMEM
 * tensor-core mainloop (bf16 / e4m3, B = 128, D = 128), 0 = the CUDA-core kernel (fp32 and the
 * remaining shapes). */
int fpx_attention_path(const fpx_problem* p);

#ifdef __cplusplus
}
#endif

#endif /* FPX_H_ */
