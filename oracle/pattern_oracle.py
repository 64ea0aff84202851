"""Plain fp64 CPU oracle of query-probe vertical / slash pattern discovery (token granularity).

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` may import or run this module; it shares no code with
the CUDA library and the library never imports it.

FlashPrefill §3 ("Instantaneous Pattern Discovery") uses uniformly distributed query probes to
find vertical, slash and block-sparse patterns concurrently: vertical patterns are invariant
along the query axis (the same key columns matter to every query), slash patterns are invariant
under translation (the same query-key offsets matter everywhere).  The page gives no formula;
the reading taken here is the plainest one it supports, with the page's own max-based
thresholding (§3 "Max-based Dynamic Thresholding") as the selection rule:

* probes: n_probe query tokens spread uniformly over a sequence of n tokens, positions
  ceil((p + 1) n / n_probe) - 1 for p = 0 .. n_probe - 1 (distinct, always including the last);
* probe attention: A[p, j] = softmax over the causal keys j <= pos_p of scale * <q_pos_p, k_j>;
* vertical significance of key token j: v_j = max over probes with pos_p >= j of A[p, j];
  j is a vertical iff alpha_v == 0 or v_j >= alpha_v * max_j' v_j';
* slash significance of offset delta >= 0: d_delta = max over probes with pos_p >= delta of
  A[p, pos_p - delta]; delta is a slash iff alpha_s == 0 or d_delta >= alpha_s * max d;
* every query i then attends the keys j <= i with j a vertical or i - j a slash (per Q head).
"""
from __future__ import annotations

import math
from typing import List, Tuple

import numpy as np

from . import fpx_oracle as O


def probe_positions(n: int, n_probe: int) -> np.ndarray:
    """Uniformly spread probe query positions in [0, n), the last token always included."""
    if n == 0 or n_probe <= 0:
        return np.zeros(0, np.int64)
    m = min(n_probe, n)
    return np.unique(np.array([math.ceil((p + 1) * n / m) - 1 for p in range(m)], np.int64))


def probe_attention(q, k, start: int, n: int, pos: np.ndarray, scale: float, g: int
                    ) -> np.ndarray:
    """[Hq, P, n] fp64 causal softmax rows of the probe queries of one sequence."""
    hq = q.shape[1]
    a = np.zeros((hq, len(pos), n), np.float64)
    for h in range(hq):
        kk = np.asarray(k[start:start + n, h // g], np.float64)
        for p, i in enumerate(pos):
            logits = scale * (kk[:i + 1] @ np.asarray(q[start + i, h], np.float64))
            e = np.exp(logits - logits.max())
            a[h, p, :i + 1] = e / e.sum()
    return a


def probe_scores(a: np.ndarray, pos: np.ndarray) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Per Q head: v [n], the vertical significance of every key token (max over the probes that
    see it), and d [n], the slash significance of every offset (max over the probes of the
    probability that many tokens back)."""
    hq, _, n = a.shape
    vs, ds = [], []
    for h in range(hq):
        v = np.zeros(n)
        d = np.zeros(n)
        for p, i in enumerate(pos):
            v[:i + 1] = np.maximum(v[:i + 1], a[h, p, :i + 1])
            d[:i + 1] = np.maximum(d[:i + 1], a[h, p, i::-1])  # offset delta = i - j
        vs.append(v)
        ds.append(d)
    return vs, ds


def _select_max_based(x: np.ndarray, alpha: float) -> np.ndarray:
    if alpha == 0:
        return np.arange(x.size)
    if x.size == 0:
        return np.zeros(0, np.int64)
    return np.nonzero(x >= alpha * x.max())[0]


def vertical_slash(a: np.ndarray, pos: np.ndarray, alpha_v: float, alpha_s: float
                   ) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Per Q head: sorted vertical key tokens and sorted slash offsets of one sequence."""
    vs, ds = probe_scores(a, pos)
    verts = [_select_max_based(v, alpha_v) for v in vs]
    slashes = [_select_max_based(d, alpha_s) for d in ds]
    return verts, slashes


def near_threshold(x: np.ndarray, alpha: float) -> np.ndarray:
    """Indices whose significance lies within NEAR_REL * alpha * max of the selection threshold
    alpha * max (alpha > 0): decisions there may flip with rounding and are reported, not
    failed (the same rule as the block threshold's)."""
    if alpha == 0 or x.size == 0:
        return np.zeros(0, np.int64)
    thr = alpha * x.max()
    return np.nonzero(np.abs(x - thr) <= O.NEAR_REL * thr)[0]


def token_mask(n: int, verts: np.ndarray, slashes: np.ndarray) -> np.ndarray:
    """[n, n] bool: causal and (key is a vertical or the offset is a slash)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    isv = np.zeros(n, bool)
    isv[verts] = True
    iss = np.zeros(n, bool)
    iss[slashes] = True
    return (j <= i) & (isv[None, :] | iss[np.clip(i - j, 0, n - 1)])


def attention_token_mask(q, k, v, cu_seqlens, masks: List[np.ndarray], scale=None
                         ) -> Tuple[np.ndarray, np.ndarray]:
    """O [T, Hq, D] and LSE [Hq, T] (natural log) of exact attention under per-(sequence, head)
    token masks masks[s][h] ([n, n] bool); rows with no key get O = 0, LSE = -inf."""
    t_all, hq, d = q.shape
    g = hq // k.shape[1]
    sc = O.default_scale(d) if scale is None or scale <= 0 else float(scale)
    o = np.zeros((t_all, hq, v.shape[2]), np.float64)
    lse = np.full((hq, t_all), -np.inf)
    for s_, L in enumerate(O.seq_layout(cu_seqlens, 1)):
        a, n = L["start"], L["n"]
        if n == 0:  # an empty sequence has no rows
            continue
        for h in range(hq):
            qq = np.asarray(q[a:a + n, h], np.float64)
            kk = np.asarray(k[a:a + n, h // g], np.float64)
            vv = np.asarray(v[a:a + n, h // g], np.float64)
            logits = np.where(masks[s_][h], sc * (qq @ kk.T), -np.inf)
            m = logits.max(axis=1, keepdims=True)
            ok = np.isfinite(m[:, 0])
            e = np.where(ok[:, None], np.exp(logits - np.where(ok[:, None], m, 0.0)), 0.0)
            z = e.sum(axis=1)
            o[a:a + n, h][ok] = (e[ok] @ vv) / z[ok, None]
            lse[h, a:a + n][ok] = m[ok, 0] + np.log(z[ok])
    return o, lse


def discover(q, k, cu_seqlens, n_probe: int, alpha_v: float, alpha_s: float, scale=None,
             with_near: bool = False):
    """Per sequence: (verticals per head, slashes per head); with_near: also the near-threshold
    key tokens and offsets per head, (verts, slashes, near_verts, near_slashes)."""
    hq, d = q.shape[1], q.shape[2]
    g = hq // k.shape[1]
    sc = O.default_scale(d) if scale is None or scale <= 0 else float(scale)
    out = []
    for L in O.seq_layout(cu_seqlens, 1):
        pos = probe_positions(L["n"], n_probe)
        a = probe_attention(q, k, L["start"], L["n"], pos, sc, g)
        if not with_near:
            out.append(vertical_slash(a, pos, alpha_v, alpha_s))
            continue
        vs, ds = probe_scores(a, pos)
        out.append(([_select_max_based(v, alpha_v) for v in vs],
                     [_select_max_based(x, alpha_s) for x in ds],
                     [near_threshold(v, alpha_v) for v in vs],
                     [near_threshold(x, alpha_s) for x in ds]))
    return out


def attention_token_rows(q, k, v, cu_seqlens, verts, slashes, rows, scale=None):
    """O [len(rows), D] and LSE [len(rows)] of exact attention for the listed (h, t) pairs (t a
    global token index) under the vertical / slash token mask: query i of sequence s attends key
    j <= i iff j is in verts[s][h] or i - j is in slashes[s][h]; a row with no key gets O = 0,
    LSE = -inf.  The same definition as attention_token_mask, evaluated row by row."""
    hq, d = q.shape[1], q.shape[2]
    g = hq // k.shape[1]
    sc = O.default_scale(d) if scale is None or scale <= 0 else float(scale)
    lay = O.seq_layout(cu_seqlens, 1)
    starts = np.array([L["start"] for L in lay])
    o = np.zeros((len(rows), v.shape[2]))
    lse = np.full(len(rows), -np.inf)
    for r, (h, t) in enumerate(rows):
        s_ = int(np.searchsorted(starts, t, side="right") - 1)
        while lay[s_]["n"] == 0 or t >= lay[s_]["start"] + lay[s_]["n"]:
            s_ += 1
        a, n = lay[s_]["start"], lay[s_]["n"]
        i = t - a
        isv = np.zeros(n, bool)
        isv[np.asarray(verts[s_][h], np.int64)] = True
        iss = np.zeros(n, bool)
        iss[np.asarray(slashes[s_][h], np.int64)] = True
        j = np.arange(i + 1)
        keys = j[isv[j] | iss[i - j]]
        if keys.size == 0:
            continue
        logits = sc * (np.asarray(k[a + keys, h // g], np.float64) @
                       np.asarray(q[t, h], np.float64))
        m = logits.max()
        e = np.exp(logits - m)
        lse[r] = m + np.log(e.sum())
        o[r] = (e / e.sum()) @ np.asarray(v[a + keys, h // g], np.float64)
    return o, lse
