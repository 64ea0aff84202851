"""Python binding of the fpx C ABI (``include/fpx.h``): dynamic block-sparse pooled prefill
attention on B200.

Argument marshalling only: PyTorch supplies device memory and the current CUDA stream; every
step of the path (pooling, scoring, thresholding, CSR compression, sparse attention) runs in the
CUDA kernels of ``libfpx.so``.  There is no CPU fallback: if the library is missing, ``load()``
raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfpx.so")

F32, BF16, E4M3 = 0, 1, 2
_DTYPES = {torch.float32: F32, torch.bfloat16: BF16, torch.float8_e4m3fn: E4M3}

STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "misaligned pointer",
          -4: "capacity too small", -5: "CUDA error", -6: "device-side wait timed out",
          -7: "malformed device input"}

# every symbol include/fpx.h declares
EXPORTS = ("fpx_num_blocks", "fpx_scores_elems", "fpx_rows", "fpx_max_nnz", "fpx_workspace_bytes",
           "fpx_clear_status", "fpx_query_status", "fpx_status_string", "fpx_block_scores",
           "fpx_select", "fpx_sparse_prefill", "fpx_attention_path", "fpx_select_noalloc",
           "fpx_select_noalloc_max_bytes", "fpx_diag_bounded_wait", "fpx_block_scores_paged",
           "fpx_sparse_prefill_paged", "fpx_block_scores_rescue", "fpx_select_rescue",
           "fpx_diag_exp2", "fpx_pattern_words", "fpx_vs_workspace_bytes", "fpx_probe_patterns",
           "fpx_vs_select", "fpx_vs_prefill")


class FpxError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: fpx status {code} ({STATUS.get(code, 'unknown')})")
        self.code = code


class Problem(ctypes.Structure):
    """Mirror of ``fpx_problem``."""
    _fields_ = [("num_seqs", ctypes.c_int32), ("cu_seqlens_d", ctypes.c_void_p),
                ("cu_seqlens_h", ctypes.c_void_p), ("total_tokens", ctypes.c_int32),
                ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("block", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("q_scale_d", ctypes.c_void_p), ("k_scale_d", ctypes.c_void_p),
                ("v_scale_d", ctypes.c_void_p), ("softmax_scale", ctypes.c_float)]


class PagedKV(ctypes.Structure):
    """Mirror of ``fpx_paged_kv``."""
    _fields_ = [("block_table_d", ctypes.c_void_p), ("pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


def paged_kv(block_table: torch.Tensor, num_pages: int) -> PagedKV:
    """Describes a page table: device int32 [num_seqs, pages_per_seq] of page indices."""
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 [num_seqs, pages_per_seq] tensor")
    kv = PagedKV(block_table.data_ptr(), block_table.shape[1], int(num_pages))
    kv._keep = block_table  # the table must outlive the calls that use it
    return kv


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libfpx.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m dynamic_block_sparse_pooled_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Problem)
    vp, sz, i32, i64, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, \
        ctypes.c_float
    for name in ("fpx_num_blocks", "fpx_scores_elems", "fpx_rows", "fpx_max_nnz"):
        getattr(lib, name).argtypes = [P]
        getattr(lib, name).restype = sz
    lib.fpx_workspace_bytes.argtypes = [P, ctypes.c_int]
    lib.fpx_workspace_bytes.restype = sz
    lib.fpx_clear_status.argtypes = [vp, vp]
    lib.fpx_clear_status.restype = ctypes.c_int
    lib.fpx_query_status.argtypes = [vp, vp]
    lib.fpx_query_status.restype = ctypes.c_int
    lib.fpx_status_string.argtypes = [ctypes.c_int]
    lib.fpx_status_string.restype = ctypes.c_char_p
    lib.fpx_attention_path.argtypes = [P]
    lib.fpx_attention_path.restype = ctypes.c_int
    lib.fpx_block_scores.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.fpx_block_scores.restype = ctypes.c_int
    lib.fpx_select.argtypes = [P, vp, f32, i32, i32, vp, vp, i64, vp, vp, sz, vp]
    lib.fpx_select.restype = ctypes.c_int
    lib.fpx_sparse_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fpx_sparse_prefill.restype = ctypes.c_int
    lib.fpx_select_noalloc.argtypes = [P, vp, f32, i32, i32, vp, vp, i64, vp, vp]
    lib.fpx_select_noalloc.restype = ctypes.c_int
    lib.fpx_select_noalloc_max_bytes.argtypes = []
    lib.fpx_select_noalloc_max_bytes.restype = sz
    lib.fpx_diag_bounded_wait.argtypes = [vp, ctypes.c_uint64, vp]
    lib.fpx_diag_bounded_wait.restype = ctypes.c_int
    lib.fpx_diag_exp2.argtypes = [vp, vp, i64, vp]
    lib.fpx_diag_exp2.restype = ctypes.c_int
    lib.fpx_pattern_words.argtypes = [P]
    lib.fpx_pattern_words.restype = sz
    lib.fpx_vs_workspace_bytes.argtypes = [P, i32]
    lib.fpx_vs_workspace_bytes.restype = sz
    lib.fpx_probe_patterns.argtypes = [P, vp, vp, i32, f32, f32, vp, vp, vp, sz, vp]
    lib.fpx_probe_patterns.restype = ctypes.c_int
    lib.fpx_vs_select.argtypes = [P, vp, vp, vp, vp, i64, vp, vp, sz, vp]
    lib.fpx_vs_select.restype = ctypes.c_int
    lib.fpx_vs_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fpx_vs_prefill.restype = ctypes.c_int
    K = ctypes.POINTER(PagedKV)
    lib.fpx_block_scores_paged.argtypes = [P, vp, vp, K, vp, vp, sz, vp]
    lib.fpx_block_scores_paged.restype = ctypes.c_int
    lib.fpx_sparse_prefill_paged.argtypes = [P, vp, vp, vp, K, vp, vp, vp, vp, vp, sz, vp]
    lib.fpx_sparse_prefill_paged.restype = ctypes.c_int
    lib.fpx_block_scores_rescue.argtypes = [P, vp, vp, K, vp, vp, vp, vp, sz, vp]
    lib.fpx_block_scores_rescue.restype = ctypes.c_int
    lib.fpx_select_rescue.argtypes = [P, vp, vp, vp, f32, f32, i32, i32, vp, vp, i64, vp, vp, sz,
                                      vp]
    lib.fpx_select_rescue.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def check(code: int, where: str) -> None:
    if code != 0:
        raise FpxError(code, where)


@dataclass
class Prefill:
    """One prefill problem bound to device tensors (keeps the marshalled struct alive)."""
    struct: Problem
    cu_d: Optional[torch.Tensor]
    cu_h: Optional[np.ndarray]
    scales: tuple
    nb: int
    rows: int
    tri: int

    @property
    def ptr(self):
        return ctypes.byref(self.struct)


def problem(q: torch.Tensor, k: torch.Tensor, block: int,
            cu_seqlens: Optional[Sequence[int]] = None, softmax_scale: float = 0.0,
            q_scale: Optional[torch.Tensor] = None, k_scale: Optional[torch.Tensor] = None,
            v_scale: Optional[torch.Tensor] = None) -> Prefill:
    """Describes Q [T, Hq, D] / K [T, Hkv, D] (packed by cu_seqlens, host ints) to the library."""
    lib = load()
    t, hq, d = q.shape
    hkv = k.shape[1]
    if q.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {q.dtype}")
    s = Problem()
    cu_h = cu_d = None
    if cu_seqlens is not None:
        cu_h = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        cu_d = torch.from_numpy(cu_h).to(q.device)
        s.num_seqs = len(cu_h) - 1
        s.cu_seqlens_d = cu_d.data_ptr()
        s.cu_seqlens_h = cu_h.ctypes.data
    else:
        s.num_seqs = 1
    s.total_tokens, s.hq, s.hkv, s.d, s.block = t, hq, hkv, d, block
    s.dtype = _DTYPES[q.dtype]
    scales = (q_scale, k_scale, v_scale)
    if s.dtype == E4M3:
        s.q_scale_d, s.k_scale_d, s.v_scale_d = (x.data_ptr() for x in scales)
    s.softmax_scale = softmax_scale
    ref = ctypes.byref(s)
    nb, rows, tri = lib.fpx_num_blocks(ref), lib.fpx_rows(ref), lib.fpx_scores_elems(ref) // hq
    return Prefill(s, cu_d, cu_h, scales, nb, rows, tri)


def workspace(pf: Prefill, which: int = -1, device=None) -> torch.Tensor:
    """A zeroed device workspace (status block cleared) for stage `which` (-1: all stages)."""
    n = load().fpx_workspace_bytes(pf.ptr, which)
    if n == 0:
        raise FpxError(-1, "fpx_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device-side status recorded in `ws`."""
    return load().fpx_query_status(_ptr(ws), _stream(stream))


def clear_status(ws: torch.Tensor, stream=None) -> None:
    check(load().fpx_clear_status(_ptr(ws), _stream(stream)), "fpx_clear_status")


def attention_path(pf: Prefill) -> int:
    return load().fpx_attention_path(pf.ptr)


def block_scores(pf: Prefill, q: torch.Tensor, k: torch.Tensor, ws: torch.Tensor,
                 scores: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fpx_block_scores -> fp32 [Hq * TRI] triangular-packed pooled block scores."""
    if scores is None:
        scores = torch.empty(pf.struct.hq * pf.tri, dtype=torch.float32, device=q.device)
    check(load().fpx_block_scores(pf.ptr, _ptr(q), _ptr(k), _ptr(scores), _ptr(ws), ws.numel(),
                                  _stream(stream)), "fpx_block_scores")
    return scores


def _check_csr_outputs(pf: Prefill, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                       nnz: torch.Tensor, capacity: int) -> None:
    """The library writes up to `capacity` col_idx entries and R + 1 row_ptr entries: refuse
    buffers that cannot hold them (the device would write past the tensors)."""
    if row_ptr.dtype != torch.int32 or col_idx.dtype != torch.int32 or nnz.dtype != torch.int64:
        raise ValueError("row_ptr and col_idx must be int32 and nnz int64")
    if not (row_ptr.is_contiguous() and col_idx.is_contiguous()):
        raise ValueError("row_ptr and col_idx must be contiguous")
    if row_ptr.numel() < pf.rows + 1:
        raise ValueError(f"row_ptr holds {row_ptr.numel()} entries, needs {pf.rows + 1}")
    if capacity < 0 or capacity > col_idx.numel():
        raise ValueError(f"capacity {capacity} exceeds col_idx ({col_idx.numel()} entries)")
    if nnz.numel() < 1:
        raise ValueError("nnz needs one int64 entry")


def select(pf: Prefill, scores: torch.Tensor, alpha: float, ws: torch.Tensor,
           sink_blocks: int = 1, window_blocks: int = 1, row_ptr=None, col_idx=None,
           nnz=None, capacity: Optional[int] = None, stream=None):
    """fpx_select -> (row_ptr int32 [R+1], col_idx int32 [capacity], nnz int64 [1])."""
    dev = scores.device
    if row_ptr is None:
        row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        cap = pf.struct.hq * pf.tri if capacity is None else capacity
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    cap = col_idx.numel() if capacity is None else capacity
    if nnz is None:
        nnz = torch.empty(1, dtype=torch.int64, device=dev)
    _check_csr_outputs(pf, row_ptr, col_idx, nnz, cap)
    check(load().fpx_select(pf.ptr, _ptr(scores), float(alpha), sink_blocks, window_blocks,
                            _ptr(row_ptr), _ptr(col_idx), cap, _ptr(nnz), _ptr(ws), ws.numel(),
                            _stream(stream)), "fpx_select")
    return row_ptr, col_idx, nnz


def select_noalloc(pf: Prefill, scores: torch.Tensor, alpha: float, sink_blocks: int = 1,
                   window_blocks: int = 1, row_ptr=None, col_idx=None, nnz=None,
                   capacity: Optional[int] = None, stream=None):
    """fpx_select_noalloc: fpx_select for callers that cannot provide a workspace (the scratch
    is a fixed device array inside the library; concurrent calls on one device race on it)."""
    dev = scores.device
    if row_ptr is None:
        row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        cap = pf.struct.hq * pf.tri if capacity is None else capacity
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    cap = col_idx.numel() if capacity is None else capacity
    if nnz is None:
        nnz = torch.empty(1, dtype=torch.int64, device=dev)
    _check_csr_outputs(pf, row_ptr, col_idx, nnz, cap)
    check(load().fpx_select_noalloc(pf.ptr, _ptr(scores), float(alpha), sink_blocks,
                                    window_blocks, _ptr(row_ptr), _ptr(col_idx), cap, _ptr(nnz),
                                    _stream(stream)), "fpx_select_noalloc")
    return row_ptr, col_idx, nnz


def sparse_prefill(pf: Prefill, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   row_ptr: torch.Tensor, col_idx: torch.Tensor, ws: torch.Tensor,
                   o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   want_lse: bool = True, stream=None):
    """fpx_sparse_prefill -> (O [T, Hq, D] (bf16, fp32 for fp32 inputs), LSE fp32 [Hq, T])."""
    if o is None:
        odt = torch.float32 if q.dtype == torch.float32 else torch.bfloat16
        o = torch.empty(q.shape, dtype=odt, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    check(load().fpx_sparse_prefill(pf.ptr, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                                    _ptr(col_idx), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                    _stream(stream)), "fpx_sparse_prefill")
    return o, lse


def block_scores_paged(pf: Prefill, q: torch.Tensor, k_cache: torch.Tensor, kv: PagedKV,
                       ws: torch.Tensor, scores: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """fpx_block_scores_paged: K from the paged cache [num_pages, block, Hkv, D]."""
    if scores is None:
        scores = torch.empty(pf.struct.hq * pf.tri, dtype=torch.float32, device=q.device)
    check(load().fpx_block_scores_paged(pf.ptr, _ptr(q), _ptr(k_cache), ctypes.byref(kv),
                                        _ptr(scores), _ptr(ws), ws.numel(), _stream(stream)),
          "fpx_block_scores_paged")
    return scores


def sparse_prefill_paged(pf: Prefill, q: torch.Tensor, k_cache: torch.Tensor,
                         v_cache: torch.Tensor, kv: PagedKV, row_ptr: torch.Tensor,
                         col_idx: torch.Tensor, ws: torch.Tensor,
                         o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         stream=None):
    """fpx_sparse_prefill_paged: K and V from the paged caches -> (O, LSE)."""
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    check(load().fpx_sparse_prefill_paged(pf.ptr, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          ctypes.byref(kv), _ptr(row_ptr), _ptr(col_idx),
                                          _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                          _stream(stream)), "fpx_sparse_prefill_paged")
    return o, lse


def block_scores_rescue(pf: Prefill, q: torch.Tensor, k: torch.Tensor, ws: torch.Tensor,
                        kv: Optional[PagedKV] = None, stream=None):
    """fpx_block_scores_rescue -> (scores [Hq * TRI], qnorm [Hq, NB], radius [Hkv, NB])."""
    nb = pf.rows // pf.struct.hq
    scores = torch.empty(pf.struct.hq * pf.tri, dtype=torch.float32, device=q.device)
    qnorm = torch.empty((pf.struct.hq, nb), dtype=torch.float32, device=q.device)
    radius = torch.empty((pf.struct.hkv, nb), dtype=torch.float32, device=q.device)
    check(load().fpx_block_scores_rescue(pf.ptr, _ptr(q), _ptr(k),
                                         ctypes.byref(kv) if kv is not None else None,
                                         _ptr(scores), _ptr(qnorm), _ptr(radius), _ptr(ws),
                                         ws.numel(), _stream(stream)), "fpx_block_scores_rescue")
    return scores, qnorm, radius


def select_rescue(pf: Prefill, scores: torch.Tensor, qnorm: torch.Tensor, radius: torch.Tensor,
                  alpha: float, alpha_rescue: float, ws: torch.Tensor, sink_blocks: int = 1,
                  window_blocks: int = 1, stream=None):
    """fpx_select_rescue -> (row_ptr, col_idx, nnz) of the base OR rescue selection."""
    dev = scores.device
    row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=dev)
    cap = pf.struct.hq * pf.tri
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    nnz = torch.empty(1, dtype=torch.int64, device=dev)
    check(load().fpx_select_rescue(pf.ptr, _ptr(scores), _ptr(qnorm), _ptr(radius), float(alpha),
                                   float(alpha_rescue), sink_blocks, window_blocks, _ptr(row_ptr),
                                   _ptr(col_idx), cap, _ptr(nnz), _ptr(ws), ws.numel(),
                                   _stream(stream)), "fpx_select_rescue")
    return row_ptr, col_idx, nnz


def prefill(q, k, v, block: int, alpha: float, cu_seqlens=None, sink_blocks: int = 1,
            window_blocks: int = 1, softmax_scale: float = 0.0, q_scale=None, k_scale=None,
            v_scale=None, stream=None) -> dict:
    """The whole path on one stream: scores -> CSR -> O, LSE.  Raises on any recorded error."""
    pf = problem(q, k, block, cu_seqlens, softmax_scale, q_scale, k_scale, v_scale)
    ws = workspace(pf, -1, q.device)
    scores = block_scores(pf, q, k, ws, stream=stream)
    row_ptr, col_idx, nnz = select(pf, scores, alpha, ws, sink_blocks, window_blocks,
                                   stream=stream)
    o, lse = sparse_prefill(pf, q, k, v, row_ptr, col_idx, ws, stream=stream)
    check(status(ws, stream), "device status")
    return dict(problem=pf, scores=scores, row_ptr=row_ptr, col_idx=col_idx, nnz=nnz, o=o,
                lse=lse)


# ---- query-probe vertical / slash path ------------------------------------------------------

def pattern_words(pf: Prefill) -> int:
    """uint32 words per head of the vertical / slash bitmasks (ceil(T / 32))."""
    return load().fpx_pattern_words(pf.ptr)


def vs_workspace(pf: Prefill, n_probe: int, device=None) -> torch.Tensor:
    """A zeroed workspace for fpx_probe_patterns, fpx_vs_select and fpx_vs_prefill."""
    n = load().fpx_vs_workspace_bytes(pf.ptr, int(n_probe))
    if n == 0:
        raise FpxError(-2, "fpx_vs_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def probe_patterns(pf: Prefill, q: torch.Tensor, k: torch.Tensor, n_probe: int, alpha_v: float,
                   alpha_s: float, ws: torch.Tensor, vert=None, slash=None, stream=None):
    """fpx_probe_patterns -> (vert_bits, slash_bits): int32 [Hq, words] holding the uint32
    bitmasks (bit cu[s] + x of head h: key token / offset x of sequence s)."""
    shape = (pf.struct.hq, max(1, pattern_words(pf)))
    vert = torch.empty(shape, dtype=torch.int32, device=q.device) if vert is None else vert
    slash = torch.empty(shape, dtype=torch.int32, device=q.device) if slash is None else slash
    for t in (vert, slash):
        if t.dtype != torch.int32 or t.numel() < shape[0] * shape[1] or not t.is_contiguous():
            raise ValueError(f"bitmask must be a contiguous int32 tensor of {shape} words")
    check(load().fpx_probe_patterns(pf.ptr, _ptr(q), _ptr(k), int(n_probe), float(alpha_v),
                                    float(alpha_s), _ptr(vert), _ptr(slash), _ptr(ws), ws.numel(),
                                    _stream(stream)), "fpx_probe_patterns")
    return vert, slash


def vs_select(pf: Prefill, vert: torch.Tensor, slash: torch.Tensor, ws: torch.Tensor,
              row_ptr=None, col_idx=None, nnz=None, capacity: Optional[int] = None, stream=None):
    """fpx_vs_select -> (row_ptr, col_idx, nnz): key blocks that can hold an allowed key."""
    dev = vert.device
    if row_ptr is None:
        row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        cap = pf.struct.hq * pf.tri if capacity is None else capacity
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    cap = col_idx.numel() if capacity is None else capacity
    if nnz is None:
        nnz = torch.empty(1, dtype=torch.int64, device=dev)
    _check_csr_outputs(pf, row_ptr, col_idx, nnz, cap)
    check(load().fpx_vs_select(pf.ptr, _ptr(vert), _ptr(slash), _ptr(row_ptr), _ptr(col_idx), cap,
                               _ptr(nnz), _ptr(ws), ws.numel(), _stream(stream)), "fpx_vs_select")
    return row_ptr, col_idx, nnz


def vs_prefill(pf: Prefill, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               vert: torch.Tensor, slash: torch.Tensor, row_ptr: torch.Tensor,
               col_idx: torch.Tensor, ws: torch.Tensor, o=None, lse=None, stream=None):
    """fpx_vs_prefill -> (O, LSE) under the vertical / slash token mask."""
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    check(load().fpx_vs_prefill(pf.ptr, _ptr(q), _ptr(k), _ptr(v), _ptr(vert), _ptr(slash),
                                _ptr(row_ptr), _ptr(col_idx), _ptr(o), _ptr(lse), _ptr(ws),
                                ws.numel(), _stream(stream)), "fpx_vs_prefill")
    return o, lse


def vs_path(q, k, v, block: int, n_probe: int, alpha_v: float, alpha_s: float, cu_seqlens=None,
            softmax_scale: float = 0.0, q_scale=None, k_scale=None, v_scale=None,
            stream=None) -> dict:
    """The query-probe path on one stream: probes -> vertical / slash bitmasks -> candidate
    blocks -> masked attention.  Raises on any recorded device-side error."""
    pf = problem(q, k, block, cu_seqlens, softmax_scale, q_scale, k_scale, v_scale)
    ws = vs_workspace(pf, n_probe, q.device)
    vert, slash = probe_patterns(pf, q, k, n_probe, alpha_v, alpha_s, ws, stream=stream)
    row_ptr, col_idx, nnz = vs_select(pf, vert, slash, ws, stream=stream)
    o, lse = vs_prefill(pf, q, k, v, vert, slash, row_ptr, col_idx, ws, stream=stream)
    check(status(ws, stream), "device status")
    return dict(problem=pf, vert=vert, slash=slash, row_ptr=row_ptr, col_idx=col_idx, nnz=nnz,
                o=o, lse=lse)
