"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle on small seeded
workloads that span several tiles and a ragged tail, for every attention kernel and dtype."""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
from oracle import fpx_oracle as O
import parity as PT

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama8b_bf16_n8192"]

CASES = {
    # tensor-core path: bf16 / e4m3, B = 128, D = 128
    "tc_bf16_ragged": BASE.with_(seqlens=(1000,), hq=4, hkv=2),
    "tc_bf16_sparse": BASE.with_(seqlens=(1500,), hq=4, hkv=2, q_gain=40.0),
    "tc_bf16_varlen": BASE.with_(seqlens=(300, 0, 129, 640, 1, 128), hq=4, hkv=1, q_gain=20.0),
    "tc_bf16_gqa8": BASE.with_(seqlens=(777,), hq=8, hkv=1),
    # odd GQA group (the last unit of each KV head holds one tile) and plain MHA (every unit
    # holds one tile)
    "tc_bf16_gqa3": BASE.with_(seqlens=(650, 129), hq=6, hkv=2, q_gain=30.0),
    "tc_e4m3_mha": BASE.with_(seqlens=(400,), hq=2, hkv=2, dtype="e4m3", q_gain=20.0),
    "tc_e4m3": BASE.with_(seqlens=(900,), hq=2, hkv=1, dtype="e4m3", q_gain=20.0),
    # CUDA-core path
    "simt_f32_tiny": WORKLOADS["tiny_fp32_n2048"].with_(seqlens=(333,)),
    "simt_bf16_b64": BASE.with_(seqlens=(500,), hq=4, hkv=2, block=64, q_gain=30.0),
    "simt_bf16_d64": BASE.with_(seqlens=(400, 77), hq=2, hkv=2, d=64),
    "simt_e4m3_b32": BASE.with_(seqlens=(260,), hq=2, hkv=1, block=32, dtype="e4m3"),
}


def run_case(w, alpha, sink=1, window=1, data=None):
    if data is None:
        data = generate(w, workers=4)
    q64, k64, v64 = PT.oracle_inputs(data)
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    # stage 1: scores
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    s_ref = PT.oracle_triangular(q64, k64, cu, w.block)
    sg = scores.cpu().numpy().reshape(w.hq, -1).astype(np.float64)
    assert np.all(np.abs(sg - s_ref) <= 2e-5 + 2e-5 * np.abs(s_ref)), \
        f"scores max err {np.abs(sg - s_ref).max():.3e}"
    # stage 2: selection
    scl = O.block_scores(q64, k64, cu, w.block)
    keeps, nears = O.select(scl, alpha, sink, window)
    ora_rp, ora_ci = O.to_csr(keeps)
    row_ptr, col_idx, nnz = fpx.select(pf, scores, alpha, ws, sink, window)
    assert fpx.status(ws) == 0
    n_near = PT.compare_csr(row_ptr.cpu().numpy(), col_idx.cpu().numpy(), ora_rp, ora_ci,
                            nears, w.hq)
    assert int(nnz.item()) == int(row_ptr[-1].item())
    # stage 3: attention given the oracle's mask
    rp_d = torch.from_numpy(ora_rp.astype(np.int32)).cuda()
    ci_d = torch.from_numpy(ora_ci.astype(np.int32) if ora_ci.size else np.zeros(1, np.int32)).cuda()
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp_d, ci_d, ws)
    assert fpx.status(ws) == 0
    o_ref, lse_ref = O.attention(q64, k64, v64, cu, w.block, ora_rp, ora_ci)
    err = PT.compare_attention(o, lse, o_ref, lse_ref, w.dtype)
    density = len(ora_ci) / max(1, w.hq * O.total_pairs(cu, w.block))
    return dict(near=n_near, err=err, density=density, path=fpx.attention_path(pf))


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("alpha", [0.0, 0.1, 0.5])
def test_parity(name, alpha):
    w = CASES[name]
    res = run_case(w, alpha)
    want_path = 1 if name.startswith("tc_") else 0
    assert res["path"] == want_path
    print(name, alpha, res)


@pytest.mark.parametrize("sink,window,alpha", [(2, 4, 0.2), (0, 1, 0.9), (3, 0, 0.3), (0, 0, 2.0)])
def test_structural_masks(sink, window, alpha):
    # includes a case with empty rows (no sink, no window, alpha > 1): O = 0, LSE = -inf
    res = run_case(CASES["tc_bf16_varlen"], alpha, sink, window)
    print(sink, window, alpha, res)


def test_full_causal_equals_library_dense_attention():
    # alpha = 0 keeps every causal block: the sparse kernel must match dense causal attention
    w = CASES["tc_bf16_ragged"]
    data = PT.to_device(generate(w))
    out = fpx.prefill(data["q"], data["k"], data["v"], w.block, 0.0, data["cu_seqlens"])
    q = data["q"].transpose(0, 1)[None].float()
    k = data["k"].transpose(0, 1)[None].float().repeat_interleave(w.hq // w.hkv, 1)
    v = data["v"].transpose(0, 1)[None].float().repeat_interleave(w.hq // w.hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    err = (out["o"].float() - ref[0].transpose(0, 1)).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


def test_whole_path_matches_oracle():
    w = CASES["tc_bf16_sparse"]
    data = generate(w)
    dev = PT.to_device(data)
    out = fpx.prefill(dev["q"], dev["k"], dev["v"], w.block, 0.1, dev["cu_seqlens"])
    q64, k64, v64 = PT.oracle_inputs(data)
    ref = O.prefill(q64, k64, v64, data["cu_seqlens"], w.block, 0.1)
    n_near = PT.compare_csr(out["row_ptr"].cpu().numpy(), out["col_idx"].cpu().numpy(),
                            ref["row_ptr"], ref["col_idx"], ref["nears"], w.hq)
    if n_near == 0:  # same mask: the whole path's own attention output must match
        PT.compare_attention(out["o"], out["lse"], ref["o"], ref["lse"], w.dtype)
    # always: the attention stage on the oracle's mask
    pf = out["problem"]
    ws = fpx.workspace(pf, -1)
    rp_d = torch.from_numpy(ref["row_ptr"].astype(np.int32)).cuda()
    ci_d = torch.from_numpy(ref["col_idx"].astype(np.int32)).cuda()
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp_d, ci_d, ws)
    assert fpx.status(ws) == 0
    PT.compare_attention(o, lse, ref["o"], ref["lse"], w.dtype)


def test_deterministic():
    w = CASES["tc_bf16_sparse"]
    dev = PT.to_device(generate(w))
    a = fpx.prefill(dev["q"], dev["k"], dev["v"], w.block, 0.1, dev["cu_seqlens"])
    b = fpx.prefill(dev["q"], dev["k"], dev["v"], w.block, 0.1, dev["cu_seqlens"])
    for key in ("scores", "row_ptr", "o", "lse"):
        assert torch.equal(a[key], b[key]), key
    n = int(a["nnz"].item())
    assert torch.equal(a["col_idx"][:n], b["col_idx"][:n])


def test_device_side_errors_are_recorded():
    w = CASES["tc_bf16_ragged"]
    dev = PT.to_device(generate(w))
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    # col_idx capacity too small: nothing is written, row_ptr is an empty CSR, FPX_ERR_CAPACITY
    # recorded, nnz reports the count needed.  The capacity is a 5-entry slice of a larger
    # sentinel-filled buffer, so a write past the slice would show.
    big = torch.full((64,), -7, dtype=torch.int32, device="cuda")
    rp, _, nnz = fpx.select(pf, scores, 0.0, ws, col_idx=big, capacity=5)
    assert fpx.status(ws) == -4
    assert torch.all(big == -7)
    assert torch.all(rp == 0)
    assert int(nnz.item()) == w.hq * pf.tri
    # the empty CSR is safe to attend: every row has no key (O = 0, LSE = -inf), nothing read
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, big, ws)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    assert torch.all(big == -7)
    # an index beyond the row's diagonal block: skipped and FPX_ERR_DEVICE_INPUT recorded
    fpx.clear_status(ws)
    rp, ci, _ = fpx.select(pf, scores, 0.0, ws)
    assert fpx.status(ws) == 0
    ci_bad = ci.clone()
    ci_bad[0] = 5  # row 0 is query block 0: only block 0 is valid
    o, lse = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, ci_bad, ws)
    assert fpx.status(ws) == -7
    # the context stays usable
    fpx.clear_status(ws)
    o2, lse2 = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, ci, ws)
    assert fpx.status(ws) == 0
    torch.cuda.synchronize()


def test_device_cu_seqlens_mismatch_is_recorded():
    w = CASES["tc_bf16_varlen"]
    dev = PT.to_device(generate(w))
    pf = PT.gpu_problem(dev, w.block)
    pf.cu_d[2] += 1  # device copy no longer matches the host mirror
    ws = fpx.workspace(pf, -1)
    fpx.block_scores(pf, dev["q"], dev["k"], ws)
    assert fpx.status(ws) == -7


def test_empty_problem():
    q = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    out = fpx.prefill(q, k, k, 128, 0.1)
    assert out["o"].shape == (0, 4, 128) and int(out["nnz"].item()) == 0


def rising_maxima_data(dtype, pattern="block"):
    """Logits that rise by ~12 log2 units per key block for about half of the query rows (the
    sign of a fixed query component drawn per row and head, so mixed inside every warp of 32
    rows) and fall for the rest: a rising row's block maximum passes the lazy-rescale threshold
    (2^8) at every block after its first, a falling row's never does.  pattern "block" raises
    whole blocks (the first 64 keys of a block already pass the threshold); "second_half"
    raises only keys 64-127 of every block (the first 64 stay at the bottom), so the maximum
    moves the reference in the second half of every block after the first."""
    w = BASE.with_(seqlens=(1000, 700), hq=4, hkv=2)
    data = generate(w, workers=4)
    cu = data["cu_seqlens"]
    q, k, v = data["q"].float(), data["k"].float(), data["v"].float()
    g = torch.Generator().manual_seed(1234)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        pos = torch.arange(b - a, dtype=torch.float32)
        blk = (pos // w.block).view(-1, 1)
        if pattern == "block":
            k[a:b, :, 0] = 8.0 * blk
        else:
            upper = ((pos % w.block) >= w.block // 2).float().view(-1, 1)
            k[a:b, :, 0] = 8.0 * (blk + 1.0) * upper
        sign = torch.where(torch.rand(b - a, w.hq, generator=g) < 0.5, -1.0, 1.0)
        q[a:b, :, 0] = 12.0 * sign
    if dtype == "bf16":
        data.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16))
    else:
        from gen.synthetic import _quant_e4m3
        w = w.with_(dtype="e4m3")
        (q8, qs), (k8, ks), (v8, vs) = _quant_e4m3(q), _quant_e4m3(k), _quant_e4m3(v)
        data.update(q=q8, k=k8, v=v8, q_scale=qs, k_scale=ks, v_scale=vs)
    data["workload"] = w
    return w, data


@pytest.mark.parametrize("pattern", ["block", "second_half"])
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("alpha", [0.0, 0.3])
def test_rising_maxima_rescale_mid_row(dtype, alpha, pattern):
    w, data = rising_maxima_data(dtype, pattern)
    res = run_case(w, alpha, data=data)
    assert res["path"] == 1
    print(dtype, alpha, res)
