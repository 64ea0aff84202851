"""GPU parity at the full workload sizes, in the launch configuration the benchmark times
(fpx_block_scores -> fpx_select -> fpx_sparse_prefill on one stream, one shared workspace).

Checked against the CPU oracle on the same seeded inputs:
* every pooled block score (fp32 GPU vs fp64 oracle);
* every CSR row: bit-exact except blocks in the near-threshold band (counted);
* attention given the oracle's mask, on sampled whole query blocks that the oracle evaluates one
  by one: for every head, the heaviest block of the longest sequence and one seeded random block,
  plus block 0 of every sequence for head 0.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, default_workers, generate
from oracle import fpx_oracle as O
import parity as PT

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny_fp32_n2048", None, 1.0),
    ("llama8b_bf16_n8192", None, 1.0),
    ("llama8b_bf16_n32768", 0.0, 1.0),
    ("llama8b_bf16_n32768", 0.05, 1.0),
    ("llama8b_bf16_n32768", 0.1, 1.0),
    ("llama8b_bf16_n32768", 0.2, 1.0),
    ("llama8b_bf16_n131072", None, 1.0),
    ("llama8b_e4m3_n131072", None, 1.0),
    ("varlen8_bf16_t264192", None, 1.0),
    # The sparse regime (labelled supplementary workloads): the same layers with Q multiplied by
    # q_gain, which widens the pooled-score spread the way trained models' larger logits do; at
    # alpha = 0.1 the 131072-token layer then keeps about 50 %, 20 % and 5 % of its causal blocks.
    ("llama8b_bf16_n131072", None, 290.0),
    ("llama8b_bf16_n131072", None, 340.0),
    ("llama8b_bf16_n131072", None, 415.0),
    ("llama8b_e4m3_n131072", None, 340.0),
    ("varlen8_bf16_t264192", None, 340.0),
    # one 1 048 576-token sequence (8192 blocks per row: the index arithmetic of every stage well
    # past the other layers'), two heads, in the sparse regime so that the oracle's CSR stays small
    ("llama8b_bf16_n131072", None, 415.0, dict(seqlens=(1048576,), hq=2, hkv=1)),
]


def oracle_arrays(data):
    """Oracle inputs: fp32 for fp32/bf16 storage (exact), fp64 for e4m3 codes x scales."""
    if data["q_scale"] is None:
        return tuple(data[k].float().numpy() for k in ("q", "k", "v"))
    return PT.oracle_inputs(data)


def sample_blocks(w, cu, rng):
    lay = O.seq_layout(cu, w.block)
    longest = int(np.argmax([L["n"] for L in lay]))
    picks = []
    for h in range(w.hq):
        nb = lay[longest]["nb"]
        picks.append((h, longest, nb - 1))
        picks.append((h, longest, int(rng.integers(0, nb))))
    for s, L in enumerate(lay):
        if L["nb"]:
            picks.append((0, s, 0))
    return sorted(set(picks)), lay


CASES = [c if len(c) == 4 else (*c, None) for c in CASES]


@pytest.mark.parametrize("name,alpha,q_gain,over", CASES,
                         ids=[f"{n}-a{a}-g{g:g}" + ("-" + "-".join(f"{k}{v[0] if isinstance(v, tuple) else v}"
                                                                    for k, v in o.items()) if o else "")
                              for n, a, g, o in CASES])
def test_full_size_parity(name, alpha, q_gain, over):
    w = WORKLOADS[name].with_(q_gain=q_gain, **(over or {}))
    if alpha is not None:
        w = w.with_(alpha=alpha)
    data = generate(w, workers=default_workers())
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)

    # GPU path, exactly as the benchmark calls it
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    row_ptr, col_idx, nnz = fpx.select(pf, scores, w.alpha, ws, w.sink_blocks, w.window_blocks)
    assert fpx.status(ws) == 0

    q, k, v = oracle_arrays(data)
    del data
    # 1) all pooled scores
    s_list = O.block_scores(q, k, cu, w.block)
    s_ref = O.triangular_pack(s_list)
    sg = scores.cpu().numpy().reshape(w.hq, -1).astype(np.float64)
    err = np.abs(sg - s_ref)
    assert np.all(err <= 2e-5 + 2e-5 * np.abs(s_ref)), f"scores max err {err.max():.3e}"
    # 2) all CSR rows
    keeps, nears = O.select(s_list, w.alpha, w.sink_blocks, w.window_blocks)
    ora_rp, ora_ci = O.to_csr(keeps)
    n_near = PT.compare_csr(row_ptr.cpu().numpy(), col_idx.cpu().numpy(), ora_rp, ora_ci, nears,
                            w.hq)
    # 3) attention given the oracle's mask, sampled query blocks
    rp_d = torch.from_numpy(ora_rp.astype(np.int32)).cuda()
    ci_d = torch.from_numpy(ora_ci.astype(np.int32)).cuda()
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp_d, ci_d, ws)
    assert fpx.status(ws) == 0
    picks, lay = sample_blocks(w, cu, np.random.default_rng(1234))
    outs = O.attention(q, k, v, cu, w.block, ora_rp, ora_ci, blocks=picks)
    o_g, l_g, o_r, l_r = [], [], [], []
    for (h, s, I), (ob, lb) in zip(picks, outs):
        t0 = lay[s]["start"] + I * w.block
        n = ob.shape[0]
        o_g.append(o[t0:t0 + n, h].float().cpu().numpy())
        l_g.append(lse[h, t0:t0 + n].cpu().numpy())
        o_r.append(ob)
        l_r.append(lb)
    err_max, err_mean = PT.compare_attention(torch.from_numpy(np.concatenate(o_g)),
                                             torch.from_numpy(np.concatenate(l_g)),
                                             np.concatenate(o_r), np.concatenate(l_r), w.dtype)
    density = len(ora_ci) / (w.hq * O.total_pairs(cu, w.block))
    if q_gain > 1.0:  # the supplementary workloads must really be sparse
        assert density < 0.75, density
    print(f"{name} alpha={w.alpha} q_gain={q_gain:g}: density={density:.4f} "
          f"near-threshold={n_near} sampled blocks={len(picks)} "
          f"O max/mean err={err_max:.2e}/{err_mean:.2e}")
