"""Radius rescue branch on the GPU (fpx_block_scores_rescue / fpx_select_rescue) against the
rescue oracle (oracle/rescue_oracle.py): pooled query norms and key-block radii, and the CSR of
the base OR rescue selection (bit-exact except blocks inside the near-threshold band of either
branch)."""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
from oracle import fpx_oracle as O
from oracle import rescue_oracle as R
import parity as PT

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama8b_bf16_n8192"]
CASES = {
    "tc_bf16_ragged": BASE.with_(seqlens=(1000,), hq=4, hkv=2, q_gain=40.0),
    "tc_bf16_varlen": BASE.with_(seqlens=(300, 0, 129, 640, 1, 128), hq=4, hkv=1, q_gain=20.0),
    "tc_e4m3": BASE.with_(seqlens=(900,), hq=2, hkv=1, dtype="e4m3", q_gain=20.0),
    "simt_bf16_d64": BASE.with_(seqlens=(400, 77), hq=2, hkv=2, d=64, q_gain=20.0),
}


def planted(seqlens, hq, hkv, d, block, seed, qmag, gain, every=3):
    """Inputs where the rescue branch matters: queries of a KV group share a strong direction, and
    every `every`-th key block of each sequence holds one key of norm `gain` pointing in a random
    direction -- a large radius that the block's centroid score does not show (mean dilution)."""
    rng = np.random.default_rng(seed)
    t_all, g = sum(seqlens), hq // hkv
    dirs = rng.standard_normal((hkv, d))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    q = 0.3 * rng.standard_normal((t_all, hq, d)) + qmag * dirs[np.arange(hq) // g][None]
    k = rng.standard_normal((t_all, hkv, d)) / np.sqrt(d)
    v = rng.standard_normal((t_all, hkv, d))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    for s_, n in enumerate(seqlens):
        for J in range(1, -(-n // block), every):
            for kvh in range(hkv):
                t = cu[s_] + J * block + rng.integers(0, min(block, n - J * block))
                u = rng.standard_normal(d)
                k[t, kvh] = gain * u / np.linalg.norm(u)
    bf = lambda x: torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)  # noqa: E731
    return dict(q=bf(q), k=bf(k), v=bf(v), cu_seqlens=cu, q_scale=None, k_scale=None,
                v_scale=None)


PLANTED = {  # (inputs, block, dtype, (alpha, alpha_rescue) pairs)
    "tc_bf16_planted": (lambda: planted((1000, 1500), 4, 2, 128, 128, 0, 150.0, 3.0), 128,
                        [(0.9, 0.1), (0.7, 0.1)]),
    "simt_bf16_d64_planted": (lambda: planted((400, 77), 4, 2, 64, 64, 0, 80.0, 4.0), 64,
                              [(0.9, 0.1)]),
}


def packed(per_seq):
    """Per-sequence [nb_s, H] arrays -> [H, NB] (the library's h * NB + b layout)."""
    cat = np.concatenate([x for x in per_seq if x.shape[0]], axis=0)
    return cat.T


def check(data, block, alpha, alpha_r):
    """GPU qnorm / radius / CSR against the rescue oracle; returns (rescued blocks, near)."""
    q64, k64, _ = PT.oracle_inputs(data)
    cu = data["cu_seqlens"]
    hq, hkv = q64.shape[1], k64.shape[1]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, block)
    ws = fpx.workspace(pf, -1)
    scores, qn, rad = fpx.block_scores_rescue(pf, dev["q"], dev["k"], ws)
    assert fpx.status(ws) == 0
    # norms and radii are in stored units (e4m3: codes); the oracle's are dequantised
    qs = data["q_scale"].numpy()[:, None] if data["q_scale"] is not None else 1.0
    ks = data["k_scale"].numpy()[:, None] if data["k_scale"] is not None else 1.0
    n_ref = packed(R.query_norms(q64, cu, block))
    r_ref = packed(R.block_radius(k64, cu, block))
    n_gpu = qn.cpu().numpy().astype(np.float64) * qs
    r_gpu = rad.cpu().numpy().astype(np.float64) * ks
    assert np.allclose(n_gpu, n_ref, rtol=2e-5, atol=2e-6), np.abs(n_gpu - n_ref).max()
    assert np.allclose(r_gpu, r_ref, rtol=2e-5, atol=2e-6), np.abs(r_gpu - r_ref).max()
    # combined selection
    s_list = O.block_scores(q64, k64, cu, block)
    u_list = R.rescue_scores(q64, k64, cu, block)
    keeps, nears = R.select_rescue(s_list, u_list, alpha, alpha_r)
    ora_rp, ora_ci = O.to_csr(keeps)
    rp, ci, nnz = fpx.select_rescue(pf, scores, qn, rad, alpha, alpha_r, ws)
    assert fpx.status(ws) == 0
    n_near = PT.compare_csr(rp.cpu().numpy(), ci.cpu().numpy(), ora_rp, ora_ci, nears, hq)
    base_keeps, _ = O.select(s_list, alpha)
    added = sum(int(k.sum()) for k in keeps) - sum(int(k.sum()) for k in base_keeps)
    return added, n_near


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("alpha,alpha_r", [(0.3, 0.05), (0.5, 0.3), (0.2, 2.0)])
def test_rescue_parity(name, alpha, alpha_r):
    w = CASES[name]
    added, n_near = check(generate(w, workers=4), w.block, alpha, alpha_r)
    print(name, alpha, alpha_r, "rescued blocks", added, "near", n_near)


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_rescue_parity_where_the_branch_adds_blocks(name):
    make, block, pairs = PLANTED[name]
    data = make()
    for alpha, alpha_r in pairs:
        added, n_near = check(data, block, alpha, alpha_r)
        assert added > 0  # the rescue branch changed the selection
        print(name, alpha, alpha_r, "rescued blocks", added, "near", n_near)


def test_rescue_off_equals_base_and_paged_equals_packed():
    w = CASES["tc_bf16_ragged"]
    data = generate(w, workers=4)
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores, qn, rad = fpx.block_scores_rescue(pf, dev["q"], dev["k"], ws)
    a = fpx.select(pf, scores, 0.3, ws)
    b = fpx.select_rescue(pf, scores, qn, rad, 0.3, 1.5, ws)  # alpha_rescue > 1: no rescue
    n = int(a[2].item())
    assert torch.equal(a[0], b[0]) and int(b[2].item()) == n and torch.equal(a[1][:n], b[1][:n])
    # the paged cache gives the same radii, bit for bit
    from test_gpu_paged import to_pages
    kc, table, npg = to_pages(dev["k"], data["cu_seqlens"], w.block, np.random.default_rng(5))
    s2, qn2, rad2 = fpx.block_scores_rescue(pf, dev["q"], kc, ws, kv=fpx.paged_kv(table, npg))
    assert fpx.status(ws) == 0
    assert torch.equal(scores, s2) and torch.equal(qn, qn2) and torch.equal(rad, rad2)
