"""fpx_select_noalloc, the thresholding/CSR stage for callers that cannot allocate device memory
(e.g. a plugin whose host framework owns all device memory and gives it no scratch buffer, or
latency-critical code that must not call cudaMalloc because it can synchronise the device).

Its output must equal fpx_select's (block indices are integers: bit-exact) on two calls in a row,
since every call reuses the same library-owned scratch array left over from the previous call.
This file is collected last so that a failure here never hides the other tests' results.
"""
import ctypes

import numpy as np

import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
import parity as PT

pytestmark = pytest.mark.gpu


def test_noalloc_select_matches_workspace_select_twice():
    w = WORKLOADS["llama8b_bf16_n8192"].with_(seqlens=(1500, 0, 700), hq=4, hkv=2, q_gain=40.0)
    dev = PT.to_device(generate(w))
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    for alpha, sink, window in [(0.1, 1, 1), (0.5, 2, 3)]:  # two calls in a row
        rp_a, ci_a, n_a = fpx.select(pf, scores, alpha, ws, sink, window)
        rp_b, ci_b, n_b = fpx.select_noalloc(pf, scores, alpha, sink, window)
        torch.cuda.synchronize()
        assert fpx.status(ws) == 0
        assert torch.equal(rp_a, rp_b)
        assert torch.equal(n_a, n_b)
        n = int(n_a.item())
        assert torch.equal(ci_a[:n], ci_b[:n])


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = fpx.load()
    limit = lib.fpx_select_noalloc_max_bytes()
    assert limit == 2 << 20
    # 100 sequences of 12800 tokens, 32 heads: 320,000 query-block rows need ~2.6 MB of scratch
    cu = np.arange(101, dtype=np.int32) * 12800
    p = fpx.Problem()
    p.num_seqs, p.total_tokens, p.hq, p.hkv, p.d, p.block, p.dtype = 100, int(cu[-1]), 32, 8, 128, 128, 1
    p.cu_seqlens_h = cu.ctypes.data
    p.cu_seqlens_d = 0x1000  # never dereferenced: the size check comes first
    assert lib.fpx_workspace_bytes(ctypes.byref(p), 1) > limit
    a = 0x100000
    rc = lib.fpx_select_noalloc(ctypes.byref(p), a, 0.1, 1, 1, a, a, 10, a, None)
    assert rc == -4  # FPX_ERR_CAPACITY, nothing launched


def test_noalloc_reports_overflow_and_bad_cu_seqlens_through_its_outputs():
    # Both conditions depend on the per-call reset of the status held in the shared scratch: a
    # normal call after each must again equal fpx_select.
    w = WORKLOADS["llama8b_bf16_n8192"].with_(seqlens=(300, 0, 129, 640, 1, 128), hq=4, hkv=1,
                                              q_gain=20.0)
    dev = PT.to_device(generate(w))
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    rp_ref, ci_ref, n_ref = fpx.select(pf, scores, 0.1, ws)
    torch.cuda.synchronize()
    n = int(n_ref.item())

    def normal_call_matches():
        rp, ci, nn = fpx.select_noalloc(pf, scores, 0.1)
        torch.cuda.synchronize()
        assert torch.equal(rp, rp_ref) and torch.equal(nn, n_ref)
        assert torch.equal(ci[:n], ci_ref[:n])

    # (1) capacity 5 inside a sentinel-filled buffer: col_idx untouched, empty CSR, full count
    big = torch.full((64,), -7, dtype=torch.int32, device="cuda")
    rp, _, nn = fpx.select_noalloc(pf, scores, 0.1, col_idx=big, capacity=5)
    torch.cuda.synchronize()
    assert torch.all(big == -7)
    assert torch.all(rp == 0)
    assert int(nn.item()) == n
    normal_call_matches()
    # (2) device cu_seqlens that disagree with the host mirror: empty CSR, nnz 0
    cu_good = pf.cu_d.clone()
    pf.cu_d[2] += 1
    rp, _, nn = fpx.select_noalloc(pf, scores, 0.1)
    torch.cuda.synchronize()
    assert torch.all(rp == 0) and int(nn.item()) == 0
    pf.cu_d.copy_(cu_good)
    normal_call_matches()
