"""Plain fp64 CPU oracle of the rescue branch of radius-based block selection.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` may import or run this module; it shares no code with
the CUDA library and the library never imports it.

The RBS-Attention abstract (listed on the FlashPrefill page of thelatestinai.com; "a block centroid may
hide a highly relevant token among many irrelevant ones": mean dilution) describes two
independently thresholded selection branches whose masks are combined: a centroid base branch
(the FlashPrefill selection of ``fpx_oracle``) and a rescue branch driven by the maximum key-block
radius.  The page gives no formula; the reading taken here is the plainest one it supports:

* radius of key block J (per KV head): r_J = max over the block's valid tokens j of
  || k_j - mean_J k ||_2 (the largest distance of a key from its block centroid);
* rescue score of the pair (I, J): u_IJ = s_IJ + scale * || mean_I q ||_2 * r_J.  By
  Cauchy-Schwarz, u_IJ >= scale * <mean_I q, k_j> for every token j of block J, so u bounds the
  best single-key logit the centroid score s_IJ may hide;
* the rescue branch keeps J iff alpha_r == 0 or exp(u_IJ - max_J' u_IJ') >= alpha_r (the same
  max-based form as the base branch, its own threshold; alpha_r > 1 keeps nothing);
* the final mask is the base mask OR the rescue mask (then CSR as in the base selection).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import numpy as np

from . import fpx_oracle as O


def block_radius(k, cu_seqlens, block: int) -> List[np.ndarray]:
    """Per sequence: [nb, Hkv] fp64 radii r_J = max_j || k_j - mean_J k ||_2 over valid rows."""
    out = []
    for L in O.seq_layout(cu_seqlens, block):
        nb = L["nb"]
        r = np.zeros((nb, k.shape[1]), dtype=np.float64)
        for b in range(nb):
            rows = np.asarray(k[L["start"] + b * block:L["start"] + min((b + 1) * block, L["n"])],
                              dtype=np.float64)
            centre = rows.mean(axis=0)                      # [Hkv, D]
            r[b] = np.sqrt(((rows - centre) ** 2).sum(axis=2)).max(axis=0)
        out.append(r)
    return out


def query_norms(q, cu_seqlens, block: int) -> List[np.ndarray]:
    """Per sequence: [nb, Hq] fp64 norms || mean_I q ||_2 of the pooled query blocks."""
    return [np.sqrt((O.pool_blocks(q, L["start"], L["n"], block) ** 2).sum(axis=2))
            for L in O.seq_layout(cu_seqlens, block)]


def rescue_scores(q, k, cu_seqlens, block: int, scale: Optional[float] = None
                  ) -> List[np.ndarray]:
    """Per sequence: [Hq, nb, nb] fp64 u_IJ = s_IJ + scale * ||qbar_I|| * r_J (J <= I), -inf
    above the diagonal."""
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    g = hq // hkv
    sc = O.default_scale(d) if scale is None or scale <= 0 else float(scale)
    s_list = O.block_scores(q, k, cu_seqlens, block, scale)
    out = []
    for s, r, n in zip(s_list, block_radius(k, cu_seqlens, block),
                       query_norms(q, cu_seqlens, block)):
        u = s.copy()
        for h in range(hq):
            u[h] = s[h] + sc * n[:, h][:, None] * r[:, h // g][None, :]
        out.append(u)
    return out


def select_rescue(scores: List[np.ndarray], rescue: List[np.ndarray], alpha: float,
                  alpha_r: float, sink_blocks: int = 1, window_blocks: int = 1
                  ) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Keep and near-threshold masks of the combined selection (base OR rescue).  near marks
    causal blocks not forced by sink / window that lie within NEAR_REL of either threshold."""
    base_keep, base_near = O.select(scores, alpha, sink_blocks, window_blocks)
    keeps, nears = [], []
    for kb, nbase, u in zip(base_keep, base_near, rescue):
        hq, nb, _ = u.shape
        if nb == 0:
            keeps.append(kb)
            nears.append(nbase)
            continue
        I = np.arange(nb)[:, None]
        J = np.arange(nb)[None, :]
        causal = J <= I
        forced = causal & ((J < sink_blocks) | (J > I - window_blocks))
        ratio = np.exp(u - u.max(axis=2, keepdims=True))
        if alpha_r == 0:
            kr = np.broadcast_to(causal, u.shape).copy()
            nr = np.zeros(u.shape, bool)
        else:
            kr = causal & (ratio >= alpha_r)
            nr = causal & ~forced & (np.abs(ratio - alpha_r) <= O.NEAR_REL * alpha_r)
        keeps.append(kb | kr)
        nears.append(nbase | nr)
    return keeps, nears
