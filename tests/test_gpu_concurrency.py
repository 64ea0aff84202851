"""The library holds no state between calls (apart from the documented scratch of the
allocation-free select): two problems run at once on two CUDA streams, each with its own
workspace, give bit-identical results to the same problems run one after the other, and a
third problem launched from a second host thread meanwhile does too."""
import threading

import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
import parity as PT

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama8b_bf16_n8192"]
PROBLEMS = [
    (BASE.with_(seqlens=(1500,), hq=4, hkv=2, q_gain=30.0), 0.1),
    (BASE.with_(seqlens=(700, 0, 300), hq=4, hkv=1, q_gain=20.0), 0.2),
    (BASE.with_(seqlens=(900,), hq=2, hkv=1, dtype="e4m3", q_gain=20.0), 0.1),
]


class Run:
    def __init__(self, w, alpha):
        self.w, self.alpha = w, alpha
        self.dev = PT.to_device(generate(w, workers=4))
        self.pf = PT.gpu_problem(self.dev, w.block)

    def path(self, stream=None):
        d, pf = self.dev, self.pf
        ws = fpx.workspace(pf, -1)  # zero-filled on the current stream, ahead of the launches
        sc = fpx.block_scores(pf, d["q"], d["k"], ws, stream=stream)
        rp, ci, nnz = fpx.select(pf, sc, self.alpha, ws, stream=stream)
        o, lse = fpx.sparse_prefill(pf, d["q"], d["k"], d["v"], rp, ci, ws, stream=stream)
        return ws, (sc, rp, ci, nnz, o, lse)


def same(a, b):
    sa, rpa, cia, na, oa, la = a
    sb, rpb, cib, nb, ob, lb = b
    n = int(na.item())
    assert n == int(nb.item())
    assert torch.equal(sa, sb) and torch.equal(rpa, rpb) and torch.equal(cia[:n], cib[:n])
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
    assert torch.equal(la, lb)


def test_streams_and_threads_give_the_sequential_results():
    runs = [Run(w, a) for w, a in PROBLEMS]
    ref = []
    for r in runs:
        ws, out = r.path()
        torch.cuda.synchronize()
        assert fpx.status(ws) == 0
        ref.append(out)
    s0, s1, s2 = (torch.cuda.Stream() for _ in range(3))
    got = [None] * 3

    def third():
        with torch.cuda.stream(s2):
            got[2] = runs[2].path(stream=s2)

    th = threading.Thread(target=third)
    th.start()
    with torch.cuda.stream(s0):
        got[0] = runs[0].path(stream=s0)
    with torch.cuda.stream(s1):
        got[1] = runs[1].path(stream=s1)
    th.join()
    torch.cuda.synchronize()
    for (ws, out), r in zip(got, ref):
        assert fpx.status(ws) == 0
        same(out, r)
