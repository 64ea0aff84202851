"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI binding and compare
it with the CPU oracle on the same seeded inputs.

Tolerances (stated once, used everywhere):
* block indices: bit-exact, except blocks whose oracle ratio exp(s - m) lies within 1e-3 * alpha
  of alpha (both decisions are then correct; they are counted and reported);
* O: max-abs 2e-2 and mean-abs 2e-3 for bf16 (and fp32) inputs, 6e-2 / 6e-3 for e4m3;
* LSE: abs 1e-3 (natural log); rows with no key: O = 0 and LSE = -inf on both sides;
* pooled scores (fp32 on the GPU vs fp64): abs 2e-5 + 2e-5 * |s|.
"""
from __future__ import annotations

import numpy as np
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import dequantised
from oracle import fpx_oracle as O

TOL = {"bf16": (2e-2, 2e-3), "f32": (2e-2, 2e-3), "e4m3": (6e-2, 6e-3)}
LSE_TOL = 1e-3


def to_device(data: dict, device="cuda"):
    out = dict(data)
    for key in ("q", "k", "v", "q_scale", "k_scale", "v_scale"):
        if data.get(key) is not None:
            out[key] = data[key].to(device)
    return out


def oracle_inputs(data: dict):
    """fp64 numpy arrays holding exactly the values the stored tensors represent."""
    return (dequantised(data["q"], data.get("q_scale")), dequantised(data["k"], data.get("k_scale")),
            dequantised(data["v"], data.get("v_scale")))


def gpu_problem(dev: dict, block: int, softmax_scale: float = 0.0):
    return fpx.problem(dev["q"], dev["k"], block, dev["cu_seqlens"], softmax_scale,
                       dev.get("q_scale"), dev.get("k_scale"), dev.get("v_scale"))


def csr_sets(row_ptr, col_idx):
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx)
    return [ci[rp[r]:rp[r + 1]] for r in range(len(rp) - 1)]


def near_sets(nears, hq):
    out = []
    for h in range(hq):
        for nr in nears:
            for I in range(nr.shape[1]):
                out.append(set(np.nonzero(nr[h, I])[0].tolist()))
    return out


def compare_csr(gpu_rp, gpu_ci, ora_rp, ora_ci, nears, hq):
    """Returns the number of near-threshold disagreements; asserts everything else is equal."""
    g = csr_sets(gpu_rp, gpu_ci)
    o = csr_sets(ora_rp, ora_ci)
    assert len(g) == len(o)
    nr = near_sets(nears, hq)
    n_near = 0
    for r, (a, b) in enumerate(zip(g, o)):
        if np.array_equal(a, b):
            continue
        assert np.all(np.diff(a) > 0), f"row {r} not ascending"
        diff = set(a.tolist()) ^ set(b.tolist())
        bad = diff - nr[r]
        assert not bad, f"row {r}: blocks {sorted(bad)} differ outside the near-threshold band"
        n_near += len(diff)
    return n_near


def compare_attention(o_gpu, lse_gpu, o_ref, lse_ref, dtype: str):
    max_tol, mean_tol = TOL[dtype]
    og = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    lg = lse_gpu.detach().cpu().numpy().astype(np.float64)
    o_ref = np.asarray(o_ref)
    lse_ref = np.asarray(lse_ref)
    empty = ~np.isfinite(lse_ref)
    assert np.array_equal(empty, ~np.isfinite(lg)), "rows with no key differ"
    err = np.abs(og - o_ref)
    assert err.max() <= max_tol, f"O max-abs {err.max():.3e} > {max_tol}"
    assert err.mean() <= mean_tol, f"O mean-abs {err.mean():.3e} > {mean_tol}"
    if (~empty).any():
        lerr = np.abs(lg[~empty] - lse_ref[~empty])
        assert lerr.max() <= LSE_TOL, f"LSE max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean())


def oracle_triangular(q64, k64, cu, block, scale=None):
    return O.triangular_pack(O.block_scores(q64, k64, cu, block, scale))
