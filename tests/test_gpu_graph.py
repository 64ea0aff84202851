"""The whole path (fpx_block_scores -> fpx_select -> fpx_sparse_prefill) can be captured in a
CUDA graph (no host synchronisation, no allocation, no host-side read of device results inside
the calls; programmatic dependent launches become graph edges) and replayed: the replays give
the eager results bit for bit, also after new inputs are copied into the captured buffers."""
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
import parity as PT

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama8b_bf16_n8192"]


def eager(dev, w, alpha):
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    sc = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    rp, ci, nnz = fpx.select(pf, sc, alpha, ws)
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, ci, ws)
    torch.cuda.synchronize()
    assert fpx.status(ws) == 0
    return o, lse, rp, ci[:int(nnz.item())], nnz


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_path_replays_from_a_cuda_graph(dtype):
    w = BASE.with_(seqlens=(1500, 700), hq=4, hkv=2, dtype=dtype, q_gain=30.0)
    alpha = 0.1
    data = [generate(w.with_(seed=s), workers=4) for s in (0, 1)]
    devs = [PT.to_device(d) for d in data]
    want = [eager(d, w, alpha) for d in devs]
    # static buffers, filled with the first inputs; everything else allocated before capture
    tensors = [k for k in ("q", "k", "v", "q_scale", "k_scale", "v_scale")
               if devs[0].get(k) is not None]
    st = {k: devs[0][k].clone() for k in tensors}
    for k in ("q_scale", "k_scale", "v_scale"):
        st.setdefault(k, None)
    st["cu_seqlens"] = devs[0]["cu_seqlens"]
    pf = PT.gpu_problem(st, w.block)
    ws = fpx.workspace(pf, -1)
    sc = torch.empty(w.hq * pf.tri, dtype=torch.float32, device="cuda")
    rp = torch.empty(pf.rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(w.hq * pf.tri, dtype=torch.int32, device="cuda")
    nnz = torch.empty(1, dtype=torch.int64, device="cuda")
    o = torch.empty(st["q"].shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.hq, w.total_tokens), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # one eager pass on the capture stream first
        fpx.block_scores(pf, st["q"], st["k"], ws, scores=sc)
        fpx.select(pf, sc, alpha, ws, row_ptr=rp, col_idx=ci, nnz=nnz)
        fpx.sparse_prefill(pf, st["q"], st["k"], st["v"], rp, ci, ws, o=o, lse=lse)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fpx.block_scores(pf, st["q"], st["k"], ws, scores=sc)
        fpx.select(pf, sc, alpha, ws, row_ptr=rp, col_idx=ci, nnz=nnz)
        fpx.sparse_prefill(pf, st["q"], st["k"], st["v"], rp, ci, ws, o=o, lse=lse)
    for i in (0, 1, 0):
        for k in tensors:
            st[k].copy_(devs[i][k])
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert fpx.status(ws) == 0
        wo, wl, wrp, wci, wn = want[i]
        n = int(nnz.item())
        assert n == int(wn.item())
        assert torch.equal(rp, wrp) and torch.equal(ci[:n], wci)
        assert torch.equal(o.view(torch.int16), wo.view(torch.int16))
        assert torch.equal(lse, wl)
    del g
