"""Regression fixtures of the CPU oracle (tests/golden/oracle_small.json, written by
tests/golden/make_golden.py, which calls only the seeded generator and the oracle).

* not gpu: the oracle reproduces every stored value on the same seeded inputs (pooled scores,
  the CSR, the near-threshold count, O and LSE of sampled rows), so a change to the oracle's
  arithmetic cannot go unnoticed;
* gpu: the CUDA path through the C ABI matches the stored values at the parity tolerances
  (fp32 D = 64 B = 16 on the CUDA-core path; bf16 and e4m3 on the tensor-core path)."""
import json
import os

import numpy as np
import pytest
import torch

from gen import WORKLOADS, generate
from oracle import fpx_oracle as O
import parity as PT

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = json.load(open(os.path.join(HERE, "golden", "oracle_small.json")))
CASES = {c["name"]: c for c in GOLDEN["cases"]}


def workload(c):
    over = {k: (tuple(v) if isinstance(v, list) else v) for k, v in c["overrides"].items()}
    return WORKLOADS[c["workload"]].with_(**over)


@pytest.mark.parametrize("name", sorted(CASES))
def test_oracle_reproduces_the_fixtures(name):
    c = CASES[name]
    w = workload(c)
    data = generate(w)
    assert [int(x) for x in data["cu_seqlens"]] == c["cu_seqlens"]
    q, k, v = PT.oracle_inputs(data)
    rows = [tuple(r) for r in c["rows"]]
    r = O.prefill(q, k, v, data["cu_seqlens"], w.block, c["alpha"], c["sink_blocks"],
                  c["window_blocks"], rows=rows)
    np.testing.assert_allclose(O.triangular_pack(r["scores"]).reshape(-1), c["scores"],
                               rtol=1e-12, atol=1e-12)
    assert r["row_ptr"].tolist() == c["row_ptr"]
    assert r["col_idx"].tolist() == c["col_idx"]
    assert sum(int(n.sum()) for n in r["nears"]) == c["near"]
    np.testing.assert_allclose(r["o"], np.array(c["o_rows"]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(c["lse_rows"]), rtol=1e-12, atol=1e-12)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_cuda_path_matches_the_fixtures(name):
    import dynamic_block_sparse_pooled_b200 as fpx
    c = CASES[name]
    w = workload(c)
    data = generate(w)
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    ref = np.array(c["scores"])
    sg = scores.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sg - ref) <= 2e-5 + 2e-5 * np.abs(ref))
    row_ptr, col_idx, nnz = fpx.select(pf, scores, c["alpha"], ws, c["sink_blocks"],
                                       c["window_blocks"])
    assert fpx.status(ws) == 0
    assert c["near"] == 0  # every decision of these fixtures is away from the threshold band
    assert row_ptr.cpu().tolist() == c["row_ptr"]
    assert col_idx[:int(nnz.item())].cpu().tolist() == c["col_idx"]
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], row_ptr, col_idx, ws)
    assert fpx.status(ws) == 0
    rows = [tuple(r) for r in c["rows"]]
    o_g = torch.stack([o[t, h] for h, t in rows])
    l_g = torch.stack([lse[h, t] for h, t in rows])
    PT.compare_attention(o_g, l_g, np.array(c["o_rows"]), np.array(c["lse_rows"]), w.dtype)
