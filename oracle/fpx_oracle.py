"""Plain, slow fp64 CPU oracle for dynamic block-sparse pooled prefill attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import or run this module.  It shares no code with the CUDA
library (no kernels, headers, helpers or tables) and the CUDA library never imports it.

What it computes follows the FlashPrefill summary page (paperlayer.ai, "FlashPrefill:
Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context Prefilling"),
taking the steps of its three stages in order (App. B, "Detailed Implementation"):

1. Instantaneous Pattern Discovery (§3 Method; App. B): mean-pool every key block, mean-pool
   every query block ("secondary averaging across queries"), score each pooled query block
   against each causally valid pooled key block, and normalise each row (softmax over J <= I).
2. Max-based Dynamic Thresholding and Block Selection (§3 Method; App. B): keep key block J of
   query-block row I iff its normalised score is at least alpha times the row maximum; OR with
   the sink mask and the local-window mask; restrict to causal J <= I; compress to index lists.
3. Block Sparse Attention (App. B): exact softmax attention of every query token over the
   tokens of its kept blocks, with the token causal mask, returning O and the natural-log LSE.

Readings taken where the page is silent (each is listed with its reason in the design notes):
* the score is scale * <mean_I q, mean_J k> with scale = 1/sqrt(D) unless given; by linearity it
  equals the block mean of the token logits, i.e. the log geometric-mean proxy of §3;
* "global normalization" is a softmax over each query-block row's causal blocks J <= I, so
  P_IJ / max_J P_IJ = exp(s_IJ - max_J s_IJ): the threshold test is exp(s - m) >= alpha;
* the diagonal block is causally valid and scored with its full (all valid rows) mean;
* a partial tail block averages its valid rows only; blocks restart at each sequence start;
* alpha == 0 keeps every causal block by definition (not through the float test);
* sink = the first ``sink_blocks`` key blocks; window = the ``window_blocks`` blocks ending at
  the diagonal (J > I - window_blocks);
* Q head h reads KV head h // (Hq / Hkv); the pattern is chosen per Q head;
* a query row with no kept key gets O = 0 and LSE = -inf.

Every computation is fp64 on the dequantised input values.
"""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

NEAR_REL = 1e-3  # relative half-width of the near-threshold band


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int) -> float:
    return 1.0 / np.sqrt(d)


def seq_layout(cu_seqlens: Sequence[int], block: int) -> List[dict]:
    """Per sequence: token start, length n, block count nb = ceil(n/B), and the offsets of its
    blocks among all sequences' blocks (block_base) and of its causal block pairs (tri_base)."""
    cu = [int(c) for c in cu_seqlens]
    out, bb, tb = [], 0, 0
    for s in range(len(cu) - 1):
        n = cu[s + 1] - cu[s]
        nb = -(-n // block)
        out.append(dict(start=cu[s], n=n, nb=nb, block_base=bb, tri_base=tb))
        bb += nb
        tb += nb * (nb + 1) // 2
    return out


def total_blocks(cu_seqlens, block) -> int:
    return sum(L["nb"] for L in seq_layout(cu_seqlens, block))


def total_pairs(cu_seqlens, block) -> int:
    """TRI: the number of causal (I, J <= I) block pairs per head, summed over sequences."""
    return sum(L["nb"] * (L["nb"] + 1) // 2 for L in seq_layout(cu_seqlens, block))


# ---------------------------------------------------------------------------------------------
# Stage 1: Instantaneous Pattern Discovery
# ---------------------------------------------------------------------------------------------

def pool_blocks(x, start: int, n: int, block: int) -> np.ndarray:
    """Mean of every block of rows of one sequence: x [T, H, D] -> [nb, H, D] (fp64).

    Average-pooled key blocks are the proxies for their tokens and query blocks are averaged
    the same way (FlashPrefill §3, Instantaneous Pattern Discovery).  A tail block shorter than
    B averages the rows it has."""
    nb = -(-n // block)
    out = np.zeros((nb,) + tuple(x.shape[1:]), dtype=np.float64)
    for b in range(nb):
        rows = _f64(x[start + b * block:start + min((b + 1) * block, n)])
        out[b] = rows.sum(axis=0) / rows.shape[0]
    return out


def block_scores(q, k, cu_seqlens, block: int, scale: Optional[float] = None) -> List[np.ndarray]:
    """Pooled block scores per sequence: list of [Hq, nb, nb] fp64 arrays with
    s[h, I, J] = scale * <mean_I q_h, mean_J k_{h // g}> for J <= I and -inf above the diagonal
    (FlashPrefill §3 "Block Approximation for Kernel Optimization"; App. B compares query tiles
    with the causally valid pooled key blocks)."""
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    g = hq // hkv
    sc = default_scale(d) if scale is None or scale <= 0 else float(scale)
    out = []
    for L in seq_layout(cu_seqlens, block):
        nb = L["nb"]
        qb = pool_blocks(q, L["start"], L["n"], block)   # [nb, Hq, D]
        kb = pool_blocks(k, L["start"], L["n"], block)   # [nb, Hkv, D]
        s = np.full((hq, nb, nb), -np.inf, dtype=np.float64)
        for h in range(hq):
            full = sc * (qb[:, h, :] @ kb[:, h // g, :].T)  # [I, J]
            causal = np.tril(np.ones((nb, nb), dtype=bool))
            s[h][causal] = full[causal]
        out.append(s)
    return out


def normalise(scores: List[np.ndarray]) -> List[np.ndarray]:
    """Row softmax over the causal blocks J <= I of every query-block row (the "global
    normalization" of App. B, read per query-block row)."""
    out = []
    for s in scores:
        m = s.max(axis=2, keepdims=True) if s.shape[2] else s
        e = np.exp(s - m)
        out.append(e / e.sum(axis=2, keepdims=True) if s.shape[2] else e)
    return out


# ---------------------------------------------------------------------------------------------
# Stage 2: Max-based Dynamic Thresholding and Block Selection
# ---------------------------------------------------------------------------------------------

def select(scores: List[np.ndarray], alpha: float, sink_blocks: int = 1,
           window_blocks: int = 1) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Keep masks and near-threshold masks per sequence ([Hq, nb, nb] bool each).

    keep[I, J] = J <= I and (alpha == 0 or P_IJ >= alpha * max_J P_IJ or J < sink_blocks or
    J > I - window_blocks)  (FlashPrefill §3 "Max-based Dynamic Thresholding"; App. B combines
    the sink, window and causal masks with the score mask).  Because P is a row softmax,
    P_IJ / max_J P_IJ = exp(s_IJ - max_J s_IJ), which is the quantity compared with alpha.
    near[I, J] marks causal blocks that are not forced by sink/window and whose ratio lies
    within NEAR_REL * alpha of alpha (alpha > 0 only)."""
    keeps, nears = [], []
    for s in scores:
        hq, nb, _ = s.shape
        I = np.arange(nb)[:, None]
        J = np.arange(nb)[None, :]
        causal = J <= I
        forced = causal & ((J < sink_blocks) | (J > I - window_blocks))
        if nb == 0:
            keeps.append(np.zeros((hq, 0, 0), bool))
            nears.append(np.zeros((hq, 0, 0), bool))
            continue
        m = s.max(axis=2, keepdims=True)
        ratio = np.exp(s - m)
        if alpha == 0:
            keep = np.broadcast_to(causal, s.shape).copy()
            near = np.zeros(s.shape, bool)
        else:
            keep = causal & ((ratio >= alpha) | forced)
            near = causal & ~forced & (np.abs(ratio - alpha) <= NEAR_REL * alpha)
        keeps.append(keep)
        nears.append(near)
    return keeps, nears


def to_csr(keeps: List[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Compress the keep masks into CSR: rows r = (h, s, I) in that order (R = Hq * sum nb),
    each listing its kept key-block indices J (local to the sequence) ascending (App. B,
    "active-block indices are compressed")."""
    if not keeps:
        return np.zeros(1, np.int64), np.zeros(0, np.int32)
    hq = keeps[0].shape[0]
    counts, cols = [], []
    for h in range(hq):
        for kp in keeps:
            for I in range(kp.shape[1]):
                js = np.nonzero(kp[h, I])[0]
                counts.append(len(js))
                cols.append(js.astype(np.int32))
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate(cols) if cols else np.zeros(0, np.int32)
    return row_ptr, col_idx.astype(np.int32)


def csr_rows_to_sets(row_ptr, col_idx) -> List[np.ndarray]:
    return [np.asarray(col_idx[row_ptr[r]:row_ptr[r + 1]]) for r in range(len(row_ptr) - 1)]


def triangular_pack(scores: List[np.ndarray]) -> np.ndarray:
    """[Hq, TRI] layout: row (h, s, I) starts at tri_base[s] + I(I+1)/2 and holds J = 0..I."""
    if not scores:
        return np.zeros((0, 0))
    hq = scores[0].shape[0]
    parts = []
    for s in scores:
        nb = s.shape[1]
        idx = np.tril_indices(nb)
        parts.append(s[:, idx[0], idx[1]])
    return np.concatenate(parts, axis=1) if parts else np.zeros((hq, 0))


# ---------------------------------------------------------------------------------------------
# Stage 3: Block Sparse Attention
# ---------------------------------------------------------------------------------------------

def _row_index(layouts, hq, h, s, I) -> int:
    nbt = sum(L["nb"] for L in layouts)
    return h * nbt + layouts[s]["block_base"] + I


def attention(q, k, v, cu_seqlens, block: int, row_ptr, col_idx,
              scale: Optional[float] = None,
              rows: Optional[Iterable[Tuple[int, int]]] = None,
              blocks: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Exact softmax attention over the kept blocks (FlashPrefill App. B, Block Sparse
    Attention), token causal mask applied (key position <= query position, both local to the
    sequence).  For query token t of sequence s in block I, Q head h:
        l_j = scale * <q_t, k_j>  for j in the kept blocks of row (h, s, I), j <= t
        lse_t = log sum_j exp(l_j);  o_t = sum_j exp(l_j - lse_t) v_j.
    Returns (O [T, Hq, D], LSE [Hq, T]) in fp64 for every token; when ``rows`` lists (h, t)
    pairs, (O [n, D], LSE [n]) for those pairs only; when ``blocks`` lists (h, s, I) query
    blocks, a list of (O [rows, D], LSE [rows]) for the valid rows of each block."""
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    g = hq // hkv
    sc = default_scale(d) if scale is None or scale <= 0 else float(scale)
    layouts = seq_layout(cu_seqlens, block)
    row_ptr = np.asarray(row_ptr)
    col_idx = np.asarray(col_idx)
    starts = np.array([L["start"] for L in layouts], dtype=np.int64)

    def one_block(s, h, I, sel_rows):
        """Rows ``sel_rows`` (local positions inside block I) of head h in sequence s."""
        L = layouts[s]
        r = _row_index(layouts, hq, h, s, I)
        blocks = col_idx[row_ptr[r]:row_ptr[r + 1]]
        keys = [np.arange(J * block, min((J + 1) * block, L["n"])) for J in blocks]
        keys = np.concatenate(keys) if keys else np.zeros(0, np.int64)
        qpos = I * block + np.asarray(sel_rows)
        qt = _f64(q[L["start"] + qpos, h, :])                     # [r, D]
        if keys.size == 0:
            return np.zeros((len(qpos), d)), np.full(len(qpos), -np.inf)
        kt = _f64(k[L["start"] + keys, h // g, :])                # [n, D]
        vt = _f64(v[L["start"] + keys, h // g, :])
        logits = sc * (qt @ kt.T)                                  # [r, n]
        allowed = keys[None, :] <= qpos[:, None]
        logits = np.where(allowed, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(logits - m)
        ssum = e.sum(axis=1, keepdims=True)
        lse = (m + np.log(np.where(ssum > 0, ssum, 1.0)))[:, 0]
        o = (e @ vt) / np.where(ssum > 0, ssum, 1.0)
        lse[empty] = -np.inf
        o[empty] = 0.0
        return o, lse

    if blocks is not None:
        out = []
        for h, s, I in blocks:
            nrow = min(block, layouts[s]["n"] - I * block)
            out.append(one_block(s, h, I, np.arange(nrow)))
        return out

    if rows is None:
        t_total = int(cu_seqlens[-1])
        O = np.zeros((t_total, hq, d), dtype=np.float64)
        LSE = np.full((hq, t_total), -np.inf, dtype=np.float64)
        for s, L in enumerate(layouts):
            for h in range(hq):
                for I in range(L["nb"]):
                    nrow = min(block, L["n"] - I * block)
                    o, lse = one_block(s, h, I, np.arange(nrow))
                    t0 = L["start"] + I * block
                    O[t0:t0 + nrow, h] = o
                    LSE[h, t0:t0 + nrow] = lse
        return O, LSE

    rows = list(rows)
    O = np.zeros((len(rows), d), dtype=np.float64)
    LSE = np.zeros(len(rows), dtype=np.float64)
    for n, (h, t) in enumerate(rows):
        s = int(np.searchsorted(starts, t, side="right") - 1)
        while layouts[s]["n"] == 0 or t >= layouts[s]["start"] + layouts[s]["n"]:
            s += 1
        i = t - layouts[s]["start"]
        o, lse = one_block(s, h, i // block, [i % block])
        O[n], LSE[n] = o[0], lse[0]
    return O, LSE


# ---------------------------------------------------------------------------------------------
# The whole path
# ---------------------------------------------------------------------------------------------

def prefill(q, k, v, cu_seqlens, block: int, alpha: float, sink_blocks: int = 1,
            window_blocks: int = 1, scale: Optional[float] = None, rows=None) -> dict:
    """Pattern discovery -> thresholding/selection -> block-sparse attention, in that order."""
    s = block_scores(q, k, cu_seqlens, block, scale)
    keeps, nears = select(s, alpha, sink_blocks, window_blocks)
    row_ptr, col_idx = to_csr(keeps)
    o, lse = attention(q, k, v, cu_seqlens, block, row_ptr, col_idx, scale, rows)
    return dict(scores=s, keeps=keeps, nears=nears, row_ptr=row_ptr, col_idx=col_idx, o=o, lse=lse)
