"""Threshold calibration and structural-retention presets for the max-based dynamic threshold
(FlashPrefill App. A, "Hyperparameter Configurations": alpha is the only hyperparameter; it is set
per model so that 4K-token sequences keep about 70 % of their blocks (computational density),
with block size 128 and an attention sink of 256 tokens plus a local window of 512 tokens
retained in addition to the blocks the threshold selects).

The kept fraction of blocks, density(alpha) = nnz / (Hq * TRI), is non-increasing in alpha: a
block kept at alpha is kept at every smaller alpha (the test is exp(s - m) >= alpha, OR-ed with
masks that do not depend on alpha).  calibrate_alpha() bisects alpha on the GPU selection itself
(fpx_select on the pooled scores of a reference prefill), so the calibrated alpha reproduces the
target density exactly as the kernels will see it.
"""
from __future__ import annotations

import math
from typing import Callable, Tuple

import torch

PAGES_SINK_TOKENS = 256
PAGES_WINDOW_TOKENS = 512
PAGES_TARGET_DENSITY_4K = 0.70


def retention_blocks(block: int, sink_tokens: int = PAGES_SINK_TOKENS,
                     window_tokens: int = PAGES_WINDOW_TOKENS) -> Tuple[int, int]:
    """(sink_blocks, window_blocks) that retain at least `sink_tokens` leading tokens and the
    `window_tokens` tokens before each query block (2 and 4 at block 128)."""
    if block <= 0:
        raise ValueError("block must be positive")
    return math.ceil(sink_tokens / block), math.ceil(window_tokens / block)


def bisect_alpha(density_of: Callable[[float], float], target: float, lo: float = 0.0,
                 hi: float = 1.0, iters: int = 30) -> Tuple[float, float]:
    """Largest alpha in [lo, hi] whose density is still >= target, for a non-increasing
    density_of; returns (alpha, density_of(alpha)).  A target at or below density_of(hi) gives
    hi; a target above density_of(lo) gives lo."""
    if not 0.0 <= target <= 1.0:
        raise ValueError("target density must lie in [0, 1]")
    d_hi = density_of(hi)
    if d_hi >= target:
        return hi, d_hi
    d_lo = density_of(lo)
    if d_lo < target:
        return lo, d_lo
    for _ in range(iters):  # invariant: density(lo) >= target > density(hi)
        mid = 0.5 * (lo + hi)
        d = density_of(mid)
        if d >= target:
            lo, d_lo = mid, d
        else:
            hi = mid
    return lo, d_lo


def calibrate_alpha(pf, scores: torch.Tensor, target: float, ws: torch.Tensor,
                    sink_blocks: int = 1, window_blocks: int = 1,
                    iters: int = 30) -> Tuple[float, float]:
    """alpha for which fpx_select keeps a fraction `target` of the causal blocks of the prefill
    described by `pf` (scores from fpx_block_scores); returns (alpha, density at alpha)."""
    from . import select

    total = pf.struct.hq * pf.tri
    if total == 0:
        return 0.0, 1.0
    row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=scores.device)
    col_idx = torch.empty(total, dtype=torch.int32, device=scores.device)
    nnz = torch.empty(1, dtype=torch.int64, device=scores.device)

    def density_of(alpha: float) -> float:
        select(pf, scores, alpha, ws, sink_blocks, window_blocks, row_ptr=row_ptr,
               col_idx=col_idx, nnz=nnz)
        return int(nnz.item()) / total

    return bisect_alpha(density_of, target, 0.0, 1.0, iters)
