// fpx_api.cu -- the C ABI declared in include/fpx.h: host-side validation, workspace layout and
// the launch sequence of every stage.  Nothing here allocates, frees or synchronises (except
// fpx_query_status, which synchronises the stream it is given).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "fpx_internal.h"

using namespace fpx;

namespace {

struct Sizes {
  int64_t nb = 0;      // NB
  int64_t tri = 0;     // TRI
  int64_t nb_max = 0;  // blocks of the longest sequence
};

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validates the problem description; fills sizes.  Everything here runs on the host.
fpx_status check_problem(const fpx_problem* p, Sizes* sz) {
  if (!p) return FPX_ERR_INVALID_ARG;
  if (p->dtype != FPX_F32 && p->dtype != FPX_BF16 && p->dtype != FPX_E4M3)
    return FPX_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return FPX_ERR_UNSUPPORTED;
  if (!is_pow2(p->block) || p->block < 16 || p->block > 128) return FPX_ERR_UNSUPPORTED;
  if (p->hq < 1 || p->hkv < 1 || p->hq % p->hkv != 0) return FPX_ERR_INVALID_ARG;
  if (p->total_tokens < 0 || p->num_seqs < 1) return FPX_ERR_INVALID_ARG;
  if ((p->cu_seqlens_d == nullptr) != (p->cu_seqlens_h == nullptr)) return FPX_ERR_INVALID_ARG;
  if (p->dtype == FPX_E4M3 && (!p->q_scale_d || !p->k_scale_d || !p->v_scale_d))
    return FPX_ERR_INVALID_ARG;
  if (std::isnan(p->softmax_scale) || std::isinf(p->softmax_scale)) return FPX_ERR_INVALID_ARG;
  Sizes s;
  if (!p->cu_seqlens_h) {
    if (p->num_seqs != 1) return FPX_ERR_INVALID_ARG;
    s.nb = (static_cast<int64_t>(p->total_tokens) + p->block - 1) / p->block;
    s.tri = s.nb * (s.nb + 1) / 2;
    s.nb_max = s.nb;
  } else {
    const int32_t* cu = p->cu_seqlens_h;
    if (cu[0] != 0 || cu[p->num_seqs] != p->total_tokens) return FPX_ERR_INVALID_ARG;
    for (int i = 0; i < p->num_seqs; ++i) {
      const int64_t n = static_cast<int64_t>(cu[i + 1]) - cu[i];
      if (n < 0) return FPX_ERR_INVALID_ARG;
      const int64_t nb = (n + p->block - 1) / p->block;
      s.nb += nb;
      s.tri += nb * (nb + 1) / 2;
      s.nb_max = std::max(s.nb_max, nb);
    }
  }
  // int32 CSR (row_ptr, col_idx) and int32 grid / row indices
  if (s.nb * p->hq >= INT32_MAX || s.tri * p->hq >= INT32_MAX) return FPX_ERR_UNSUPPORTED;
  *sz = s;
  return FPX_OK;
}

ProblemDesc make_desc(const fpx_problem* p, const Sizes& s) {
  ProblemDesc d;
  d.cu = p->cu_seqlens_d;
  d.num_seqs = p->num_seqs;
  d.total_tokens = p->total_tokens;
  d.hq = p->hq;
  d.hkv = p->hkv;
  d.group = p->hq / p->hkv;
  d.d = p->d;
  d.block = p->block;
  d.nb_total = static_cast<int32_t>(s.nb);
  d.tri_total = s.tri;
  d.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->d));
  const bool fp8 = p->dtype == FPX_E4M3;
  d.q_scale = fp8 ? p->q_scale_d : nullptr;
  d.k_scale = fp8 ? p->k_scale_d : nullptr;
  d.v_scale = fp8 ? p->v_scale_d : nullptr;
  d.page_table = nullptr;
  d.pages_per_seq = 0;
  d.num_pages = 0;
  return d;
}

// Host checks of a paged K / V description against the problem; fills the descriptor fields.
fpx_status apply_paged(const fpx_problem* p, const Sizes& s, const fpx_paged_kv* kv,
                       ProblemDesc* d) {
  if (!kv || !kv->block_table_d) return FPX_ERR_INVALID_ARG;
  if (kv->num_pages < 1 || kv->pages_per_seq < s.nb_max || kv->pages_per_seq < 1)
    return FPX_ERR_INVALID_ARG;
  if (static_cast<int64_t>(kv->num_pages) * p->block > INT32_MAX ||
      static_cast<int64_t>(kv->pages_per_seq) * p->num_seqs > INT32_MAX)
    return FPX_ERR_UNSUPPORTED;
  if (!aligned(kv->block_table_d, 4)) return FPX_ERR_ALIGNMENT;
  d->page_table = kv->block_table_d;
  d->pages_per_seq = kv->pages_per_seq;
  d->num_pages = kv->num_pages;
  return FPX_OK;
}

// Keep bitmask of the select stage: one 32-bit word per 32 key blocks of the longest row.
int64_t mask_words(const Sizes& s) { return (s.nb_max + 31) / 32; }

size_t scratch_bytes(const fpx_problem* p, const Sizes& s, int which) {
  const size_t R = static_cast<size_t>(s.nb) * p->hq;
  switch (which) {
    case 0:  // pooled Q and K, fp32 (twice: tf32 hi and lo parts for the tensor-core scores)
      return 2 * (align_up(sizeof(float) * s.nb * p->hq * p->d, 256) +
                  align_up(sizeof(float) * s.nb * p->hkv * p->d, 256));
    case 1:  // row max, keep counts, per-CTA totals, overflow flag, keep bitmask
      return align_up(sizeof(float) * R, 256) + align_up(sizeof(int32_t) * R, 256) +
             align_up(sizeof(int64_t) * (R / 8 + 1), 256) + 256 +
             align_up(sizeof(uint32_t) * R * mask_words(s), 256);
    case 2:  // tile schedule + the persistent kernel's work-queue head
      return align_up(sizeof(int32_t) * R, 256) + 256;
    default:
      return 0;
  }
}

size_t ws_bytes_for(const fpx_problem* p, const Sizes& s, int which) {
  return scratch_offset(p->num_seqs) + scratch_bytes(p, s, which);
}

// ---- query-probe vertical / slash path ---------------------------------------------------
constexpr int kProbeChunkBlocks = 8;  // key blocks of 128 per probe CTA

int pattern_words(const fpx_problem* p) { return (p->total_tokens + 31) / 32; }

int64_t probe_chunks(const fpx_problem* p) {
  // sum over sequences of ceil(nb_s / chunk) with nb_s counted in 128-key blocks
  int64_t c = 0;
  for (int i = 0; i < p->num_seqs; ++i) {
    const int64_t n = p->cu_seqlens_h ? static_cast<int64_t>(p->cu_seqlens_h[i + 1]) -
                                            p->cu_seqlens_h[i]
                                      : p->total_tokens;
    const int64_t nb = (n + 127) / 128;
    c += (nb + kProbeChunkBlocks - 1) / kProbeChunkBlocks;
  }
  return c;
}

struct ProbeLayout {
  size_t chunk_base, partial, bound, end;  // byte offsets inside the workspace
};

ProbeLayout probe_layout(const fpx_problem* p, int n_probe) {
  const int tiles = (p->hq / p->hkv * n_probe + 127) / 128;
  ProbeLayout L;
  L.chunk_base = scratch_offset(p->num_seqs);
  L.partial = L.chunk_base + align_up(sizeof(int32_t) * (p->num_seqs + 1), 256);
  L.bound = L.partial + align_up(sizeof(float) * 2 * static_cast<size_t>(probe_chunks(p)) *
                                     p->hkv * tiles * 128, 256);
  L.end = L.bound + align_up(sizeof(float) * 2 * static_cast<size_t>(p->num_seqs) * p->hq *
                                 n_probe, 256);
  return L;
}

// vs_select: the select stage's scratch followed by the two per-(head, block) flag arrays
size_t vs_select_bytes(const fpx_problem* p, const Sizes& s) {
  return ws_bytes_for(p, s, 1) + 2 * align_up(static_cast<size_t>(s.nb) * p->hq, 256);
}

fpx_status check_probe_args(const fpx_problem* p, int n_probe) {
  if (n_probe < 1 || static_cast<int64_t>(p->hq / p->hkv) * n_probe > 512)
    return FPX_ERR_UNSUPPORTED;
  return FPX_OK;
}

fpx_status check_ws(const fpx_problem* p, const Sizes& s, int which, void* ws, size_t ws_bytes) {
  if (!ws) return FPX_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return FPX_ERR_ALIGNMENT;
  if (ws_bytes < ws_bytes_for(p, s, which)) return FPX_ERR_CAPACITY;
  return FPX_OK;
}

}  // namespace

extern "C" {

size_t fpx_num_blocks(const fpx_problem* p) {
  Sizes s;
  return check_problem(p, &s) == FPX_OK ? static_cast<size_t>(s.nb) : 0;
}
size_t fpx_scores_elems(const fpx_problem* p) {
  Sizes s;
  return check_problem(p, &s) == FPX_OK ? static_cast<size_t>(s.tri) * p->hq : 0;
}
size_t fpx_rows(const fpx_problem* p) {
  Sizes s;
  return check_problem(p, &s) == FPX_OK ? static_cast<size_t>(s.nb) * p->hq : 0;
}
size_t fpx_max_nnz(const fpx_problem* p) { return fpx_scores_elems(p); }

size_t fpx_workspace_bytes(const fpx_problem* p, int which) {
  Sizes s;
  if (check_problem(p, &s) != FPX_OK) return 0;
  if (which >= 0 && which <= 2) return ws_bytes_for(p, s, which);
  if (which != -1) return 0;
  size_t m = 0;
  for (int w = 0; w <= 2; ++w) m = ws_bytes_for(p, s, w) > m ? ws_bytes_for(p, s, w) : m;
  return m;
}

fpx_status fpx_clear_status(void* ws, fpx_stream_t stream) {
  if (!ws) return FPX_ERR_INVALID_ARG;
  return cudaMemsetAsync(ws, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FPX_OK
             : FPX_ERR_CUDA;
}

fpx_status fpx_query_status(const void* ws, fpx_stream_t stream) {
  if (!ws) return FPX_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FPX_ERR_CUDA;
  StatusBlock h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return FPX_ERR_CUDA;
  return static_cast<fpx_status>(h.code);
}

const char* fpx_status_string(fpx_status s) {
  switch (s) {
    case FPX_OK: return "ok";
    case FPX_ERR_INVALID_ARG: return "invalid argument";
    case FPX_ERR_UNSUPPORTED: return "unsupported dtype, head dim, block size or size";
    case FPX_ERR_ALIGNMENT: return "misaligned pointer";
    case FPX_ERR_CAPACITY: return "capacity too small";
    case FPX_ERR_CUDA: return "CUDA error";
    case FPX_ERR_TIMEOUT: return "device-side wait timed out";
    case FPX_ERR_DEVICE_INPUT: return "malformed device input (cu_seqlens or CSR)";
  }
  return "unknown status";
}

int fpx_attention_path(const fpx_problem* p) {
  Sizes s;
  if (check_problem(p, &s) != FPX_OK) return -1;
  return attn_tc_supported(make_desc(p, s), p->dtype) ? 1 : 0;
}

static fpx_status block_scores_impl(const fpx_problem* p, const void* q, const void* k,
                                    const fpx_paged_kv* kv, float* scores, float* qnorm,
                                    float* radius, void* ws, size_t ws_bytes,
                                    fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if ((rc = check_ws(p, sz, 0, ws, ws_bytes)) != FPX_OK) return rc;
  if (p->total_tokens > 0 && (!q || !k || !scores)) return FPX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(scores, 4)) return FPX_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ProblemDesc d = make_desc(p, sz);
  if (kv && (rc = apply_paged(p, sz, kv, &d)) != FPX_OK) return rc;
  StatusBlock* st = static_cast<StatusBlock*>(ws);
  const SeqTables t = seq_tables_at(ws, p->num_seqs);
  char* scratch = static_cast<char*>(ws) + scratch_offset(p->num_seqs);
  const size_t qb = align_up(sizeof(float) * sz.nb * p->hq * p->d, 256);
  const size_t kb = align_up(sizeof(float) * sz.nb * p->hkv * p->d, 256);
  float* qbar = reinterpret_cast<float*>(scratch);
  float* kbar = reinterpret_cast<float*>(scratch + qb);
  const bool tc = score_tc_supported(d);
  float* qlo = tc ? reinterpret_cast<float*>(scratch + qb + kb) : nullptr;
  float* klo = tc ? reinterpret_cast<float*>(scratch + 2 * qb + kb) : nullptr;
  if (launch_plan(d, t, st, s) != cudaSuccess) return FPX_ERR_CUDA;
  if (sz.nb == 0) return FPX_OK;
  if (launch_pool(d, p->dtype, q, k, qbar, kbar, qlo, klo, t, st, s) != cudaSuccess)
    return FPX_ERR_CUDA;
  if (launch_score(d, p->dtype, qbar, kbar, qlo, klo, scores, t, st, s) != cudaSuccess)
    return FPX_ERR_CUDA;
  if (qnorm && launch_radius(d, p->dtype, k, qbar, kbar, qlo, klo, qnorm, radius, t, s) !=
                   cudaSuccess)
    return FPX_ERR_CUDA;
  return FPX_OK;
}

fpx_status fpx_block_scores(const fpx_problem* p, const void* q, const void* k, float* scores,
                            void* ws, size_t ws_bytes, fpx_stream_t stream) {
  return block_scores_impl(p, q, k, nullptr, scores, nullptr, nullptr, ws, ws_bytes, stream);
}

fpx_status fpx_block_scores_rescue(const fpx_problem* p, const void* q, const void* k,
                                   const fpx_paged_kv* kv, float* scores, float* qnorm,
                                   float* radius, void* ws, size_t ws_bytes,
                                   fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if (sz.nb > 0 && (!qnorm || !radius)) return FPX_ERR_INVALID_ARG;
  if (!aligned(qnorm, 4) || !aligned(radius, 4)) return FPX_ERR_ALIGNMENT;
  return block_scores_impl(p, q, k, kv, scores, qnorm, radius, ws, ws_bytes, stream);
}

fpx_status fpx_block_scores_paged(const fpx_problem* p, const void* q, const void* k_cache,
                                  const fpx_paged_kv* kv, float* scores, void* ws,
                                  size_t ws_bytes, fpx_stream_t stream) {
  if (!kv) return FPX_ERR_INVALID_ARG;
  return block_scores_impl(p, q, k_cache, kv, scores, nullptr, nullptr, ws, ws_bytes, stream);
}

static fpx_status select_impl(const fpx_problem* p, const float* scores, const float* qnorm,
                              const float* radius, float alpha, float alpha_rescue,
                              int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d, void* ws,
                              size_t ws_bytes, fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if ((rc = check_ws(p, sz, 1, ws, ws_bytes)) != FPX_OK) return rc;
  if (std::isnan(alpha) || alpha < 0.f) return FPX_ERR_INVALID_ARG;
  const bool rescue = qnorm != nullptr || radius != nullptr;
  if (rescue) {
    if (std::isnan(alpha_rescue) || alpha_rescue < 0.f) return FPX_ERR_INVALID_ARG;
    if (sz.tri > 0 && (!qnorm || !radius)) return FPX_ERR_INVALID_ARG;
    if (!aligned(qnorm, 4) || !aligned(radius, 4)) return FPX_ERR_ALIGNMENT;
  }
  if (sink_blocks < 0 || window_blocks < 0 || col_capacity < 0) return FPX_ERR_INVALID_ARG;
  if (!row_ptr) return FPX_ERR_INVALID_ARG;
  if (sz.tri > 0 && (!scores || (!col_idx && col_capacity > 0))) return FPX_ERR_INVALID_ARG;
  if (!aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(nnz_d, 8))
    return FPX_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const ProblemDesc d = make_desc(p, sz);
  StatusBlock* st = static_cast<StatusBlock*>(ws);
  const SeqTables t = seq_tables_at(ws, p->num_seqs);
  const size_t R = static_cast<size_t>(sz.nb) * p->hq;
  char* scratch = static_cast<char*>(ws) + scratch_offset(p->num_seqs);
  float* rowmax = reinterpret_cast<float*>(scratch);
  int32_t* counts = reinterpret_cast<int32_t*>(scratch + align_up(sizeof(float) * R, 256));
  int64_t* cta_tot = reinterpret_cast<int64_t*>(scratch + align_up(sizeof(float) * R, 256) +
                                                 align_up(sizeof(int32_t) * R, 256));
  int* overflow = reinterpret_cast<int*>(reinterpret_cast<char*>(cta_tot) +
                                         align_up(sizeof(int64_t) * (R / 8 + 1), 256));
  uint32_t* mask = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(overflow) + 256);
  if (launch_plan(d, t, st, s) != cudaSuccess) return FPX_ERR_CUDA;
  // window / sink beyond any row are equivalent to "all": clamp so the device compare stays
  // in range
  const int sink = sink_blocks > d.nb_total ? d.nb_total + 1 : sink_blocks;
  const int window = window_blocks > d.nb_total ? d.nb_total + 1 : window_blocks;
  if (launch_select(d, scores, alpha, sink, window, row_ptr, col_idx, col_capacity, nnz_d, rowmax,
                    counts, cta_tot, overflow, mask, static_cast<int>(mask_words(sz)),
                    rescue ? qnorm : nullptr, rescue ? radius : nullptr, alpha_rescue, t, st,
                    s) != cudaSuccess)
    return FPX_ERR_CUDA;
  return FPX_OK;
}

fpx_status fpx_select(const fpx_problem* p, const float* scores, float alpha, int32_t sink_blocks,
                      int32_t window_blocks, int32_t* row_ptr, int32_t* col_idx,
                      int64_t col_capacity, int64_t* nnz_d, void* ws, size_t ws_bytes,
                      fpx_stream_t stream) {
  return select_impl(p, scores, nullptr, nullptr, alpha, 0.f, sink_blocks, window_blocks, row_ptr,
                     col_idx, col_capacity, nnz_d, ws, ws_bytes, stream);
}

fpx_status fpx_select_rescue(const fpx_problem* p, const float* scores, const float* qnorm,
                             const float* radius, float alpha, float alpha_rescue,
                             int32_t sink_blocks, int32_t window_blocks, int32_t* row_ptr,
                             int32_t* col_idx, int64_t col_capacity, int64_t* nnz_d, void* ws,
                             size_t ws_bytes, fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if (sz.tri > 0 && (!qnorm || !radius)) return FPX_ERR_INVALID_ARG;
  return select_impl(p, scores, qnorm, radius, alpha, alpha_rescue, sink_blocks, window_blocks,
                     row_ptr, col_idx, col_capacity, nnz_d, ws, ws_bytes, stream);
}

static fpx_status sparse_prefill_impl(const fpx_problem* p, const void* q, const void* k,
                                      const void* v, const fpx_paged_kv* kv,
                                      const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                      float* lse, void* ws, size_t ws_bytes,
                                      fpx_stream_t stream, const uint32_t* vbits = nullptr,
                                      const uint32_t* sbits = nullptr) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if ((rc = check_ws(p, sz, 2, ws, ws_bytes)) != FPX_OK) return rc;
  if (p->total_tokens > 0 && (!q || !k || !v || !o || !row_ptr)) return FPX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4))
    return FPX_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ProblemDesc d = make_desc(p, sz);
  if (kv) {
    if ((rc = apply_paged(p, sz, kv, &d)) != FPX_OK) return rc;
    if (!attn_tc_supported(d, p->dtype)) return FPX_ERR_UNSUPPORTED;  // paged: tensor-core path
  }
  StatusBlock* st = static_cast<StatusBlock*>(ws);
  const SeqTables t = seq_tables_at(ws, p->num_seqs);
  char* scratch = static_cast<char*>(ws) + scratch_offset(p->num_seqs);
  int32_t* order = reinterpret_cast<int32_t*>(scratch);
  int* queue_head = reinterpret_cast<int*>(
      scratch + align_up(sizeof(int32_t) * static_cast<size_t>(sz.nb) * p->hq, 256));
  if (launch_plan(d, t, st, s) != cudaSuccess) return FPX_ERR_CUDA;
  if (sz.nb == 0) return FPX_OK;
  const bool tc = attn_tc_supported(d, p->dtype);
  if (launch_order(d, static_cast<int>(sz.nb_max), t, row_ptr, order, queue_head, tc, s) !=
      cudaSuccess)
    return FPX_ERR_CUDA;
  if (tc) {
    bool encode_failed = false;
    cudaError_t e = launch_attn_tc(d, p->dtype, q, k, v, row_ptr, col_idx, o, lse, t, order,
                                   queue_head, vbits, sbits, pattern_words(p), st, s,
                                   &encode_failed);
    if (encode_failed) return FPX_ERR_UNSUPPORTED;
    return e == cudaSuccess ? FPX_OK : FPX_ERR_CUDA;
  }
  return launch_attn_simt(d, p->dtype, q, k, v, row_ptr, col_idx, o, lse, t, order, st, s) == cudaSuccess
             ? FPX_OK
             : FPX_ERR_CUDA;
}

fpx_status fpx_sparse_prefill(const fpx_problem* p, const void* q, const void* k, const void* v,
                              const int32_t* row_ptr, const int32_t* col_idx, void* o,
                              float* lse, void* ws, size_t ws_bytes, fpx_stream_t stream) {
  return sparse_prefill_impl(p, q, k, v, nullptr, row_ptr, col_idx, o, lse, ws, ws_bytes, stream);
}

size_t fpx_pattern_words(const fpx_problem* p) {
  Sizes s;
  return check_problem(p, &s) == FPX_OK ? static_cast<size_t>(pattern_words(p)) : 0;
}

size_t fpx_vs_workspace_bytes(const fpx_problem* p, int32_t n_probe) {
  Sizes s;
  if (check_problem(p, &s) != FPX_OK || check_probe_args(p, n_probe) != FPX_OK) return 0;
  size_t m = probe_layout(p, n_probe).end;
  m = std::max(m, vs_select_bytes(p, s));
  return std::max(m, ws_bytes_for(p, s, 2));
}

fpx_status fpx_probe_patterns(const fpx_problem* p, const void* q, const void* k,
                              int32_t n_probe, float alpha_v, float alpha_s, uint32_t* vert_bits,
                              uint32_t* slash_bits, void* ws, size_t ws_bytes,
                              fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if ((rc = check_probe_args(p, n_probe)) != FPX_OK) return rc;
  ProblemDesc d = make_desc(p, sz);
  if (!attn_tc_supported(d, p->dtype)) return FPX_ERR_UNSUPPORTED;
  if (std::isnan(alpha_v) || std::isnan(alpha_s) || alpha_v < 0.f || alpha_s < 0.f)
    return FPX_ERR_INVALID_ARG;
  if (!ws) return FPX_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return FPX_ERR_ALIGNMENT;
  const ProbeLayout L = probe_layout(p, n_probe);
  if (ws_bytes < L.end) return FPX_ERR_CAPACITY;
  if (p->total_tokens > 0 && (!q || !k || !vert_bits || !slash_bits)) return FPX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(vert_bits, 4) || !aligned(slash_bits, 4))
    return FPX_ERR_ALIGNMENT;
  if (probe_chunks(p) >= INT32_MAX) return FPX_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  StatusBlock* st = static_cast<StatusBlock*>(ws);
  const SeqTables t = seq_tables_at(ws, p->num_seqs);
  char* base = static_cast<char*>(ws);
  if (launch_plan(d, t, st, s) != cudaSuccess) return FPX_ERR_CUDA;
  bool encode_failed = false;
  cudaError_t e = launch_probe(
      d, p->dtype, q, k, n_probe, alpha_v, alpha_s, kProbeChunkBlocks,
      static_cast<int>(probe_chunks(p)), t, reinterpret_cast<int32_t*>(base + L.chunk_base),
      reinterpret_cast<float2*>(base + L.partial), reinterpret_cast<float2*>(base + L.bound),
      vert_bits, slash_bits, pattern_words(p), st, s, &encode_failed);
  if (encode_failed) return FPX_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FPX_OK : FPX_ERR_CUDA;
}

fpx_status fpx_vs_select(const fpx_problem* p, const uint32_t* vert_bits,
                         const uint32_t* slash_bits, int32_t* row_ptr, int32_t* col_idx,
                         int64_t col_capacity, int64_t* nnz_d, void* ws, size_t ws_bytes,
                         fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  const ProblemDesc d = make_desc(p, sz);
  if (!attn_tc_supported(d, p->dtype)) return FPX_ERR_UNSUPPORTED;
  if (!ws) return FPX_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return FPX_ERR_ALIGNMENT;
  if (ws_bytes < vs_select_bytes(p, sz)) return FPX_ERR_CAPACITY;
  if (col_capacity < 0 || !row_ptr) return FPX_ERR_INVALID_ARG;
  if (p->total_tokens > 0 && (!vert_bits || !slash_bits || (!col_idx && col_capacity > 0)))
    return FPX_ERR_INVALID_ARG;
  if (!aligned(vert_bits, 4) || !aligned(slash_bits, 4) || !aligned(row_ptr, 4) ||
      !aligned(col_idx, 4) || !aligned(nnz_d, 8))
    return FPX_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  StatusBlock* st = static_cast<StatusBlock*>(ws);
  const SeqTables t = seq_tables_at(ws, p->num_seqs);
  const size_t R = static_cast<size_t>(sz.nb) * p->hq;
  char* scratch = static_cast<char*>(ws) + scratch_offset(p->num_seqs);
  int32_t* counts = reinterpret_cast<int32_t*>(scratch + align_up(sizeof(float) * R, 256));
  int64_t* cta_tot = reinterpret_cast<int64_t*>(scratch + align_up(sizeof(float) * R, 256) +
                                                 align_up(sizeof(int32_t) * R, 256));
  int* overflow = reinterpret_cast<int*>(reinterpret_cast<char*>(cta_tot) +
                                         align_up(sizeof(int64_t) * (R / 8 + 1), 256));
  uint32_t* mask = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(overflow) + 256);
  uint8_t* vflag = reinterpret_cast<uint8_t*>(ws) + ws_bytes_for(p, sz, 1);
  uint8_t* sflag = vflag + align_up(R, 256);
  if (launch_plan(d, t, st, s) != cudaSuccess) return FPX_ERR_CUDA;
  const int mw = static_cast<int>(mask_words(sz));
  if (launch_vs_count(d, t, vert_bits, slash_bits, pattern_words(p), vflag, sflag, counts,
                      cta_tot, mask, mw, s) != cudaSuccess)
    return FPX_ERR_CUDA;
  return launch_select_finish(d, row_ptr, col_idx, col_capacity, nnz_d, counts, cta_tot,
                              overflow, mask, mw, t, st, s) == cudaSuccess
             ? FPX_OK
             : FPX_ERR_CUDA;
}

fpx_status fpx_vs_prefill(const fpx_problem* p, const void* q, const void* k, const void* v,
                          const uint32_t* vert_bits, const uint32_t* slash_bits,
                          const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                          void* ws, size_t ws_bytes, fpx_stream_t stream) {
  Sizes sz;
  fpx_status rc = check_problem(p, &sz);
  if (rc != FPX_OK) return rc;
  if (!attn_tc_supported(make_desc(p, sz), p->dtype)) return FPX_ERR_UNSUPPORTED;
  if (p->total_tokens > 0 && (!vert_bits || !slash_bits)) return FPX_ERR_INVALID_ARG;
  if (!aligned(vert_bits, 4) || !aligned(slash_bits, 4)) return FPX_ERR_ALIGNMENT;
  return sparse_prefill_impl(p, q, k, v, nullptr, row_ptr, col_idx, o, lse, ws, ws_bytes, stream,
                             vert_bits, slash_bits);
}

fpx_status fpx_sparse_prefill_paged(const fpx_problem* p, const void* q, const void* k_cache,
                                    const void* v_cache, const fpx_paged_kv* kv,
                                    const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                    float* lse, void* ws, size_t ws_bytes, fpx_stream_t stream) {
  if (!kv) return FPX_ERR_INVALID_ARG;
  return sparse_prefill_impl(p, q, k_cache, v_cache, kv, row_ptr, col_idx, o, lse, ws, ws_bytes,
                             stream);
}

}  // extern "C"
