"""GPU parity of the query-probe vertical / slash path (fpx_probe_patterns -> fpx_vs_select ->
fpx_vs_prefill, through the C ABI) against the CPU oracle (oracle/pattern_oracle.py) on the same
seeded inputs.

* Vertical and slash sets: equal to the oracle's except tokens / offsets whose significance lies
  within 1e-3 relative of the selection threshold (the oracle's near sets; counted).
* Candidate blocks (fpx_vs_select): every key that some query of a block row may attend under the
  oracle's sets lies in a listed block.
* Attention: O / LSE under the oracle's sets against the oracle's token-masked attention, at the
  bf16 / e4m3 tolerances of the block path; rows that no key reaches: O = 0, LSE = -inf.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, default_workers, generate
from oracle import fpx_oracle as O
from oracle import pattern_oracle as PO
import parity as PT

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama8b_bf16_n8192"]


def bits_to_sets(bits: torch.Tensor, cu, hq):
    """[hq, words] bitmask -> per sequence, per head: sorted local indices x with bit cu[s] + x."""
    b = bits.cpu().numpy().view(np.uint32)
    flat = np.unpackbits(b.view(np.uint8).reshape(hq, -1), axis=1, bitorder="little")
    out = []
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        out.append([np.nonzero(flat[h, a:e])[0] for h in range(hq)])
    tail = flat[:, int(cu[-1]):]
    assert not tail.any(), "bits set past the last token"
    return out


def sets_to_bits(sets, cu, hq, words, device="cuda"):
    flat = np.zeros((hq, words * 32), np.uint8)
    for s, per_head in enumerate(sets):
        for h in range(hq):
            idx = np.asarray(per_head[h], np.int64)
            flat[h, int(cu[s]) + idx] = 1
    b = np.packbits(flat, axis=1, bitorder="little").view(np.uint32).reshape(hq, words)
    return torch.from_numpy(b.view(np.int32).copy()).to(device)


def compare_sets(gpu, ora, near, what):
    n_near = 0
    for s, (gs, os_, ns) in enumerate(zip(gpu, ora, near)):
        for h, (a, b, nr) in enumerate(zip(gs, os_, ns)):
            diff = set(np.asarray(a).tolist()) ^ set(np.asarray(b).tolist())
            bad = diff - set(np.asarray(nr).tolist())
            assert not bad, f"{what} seq {s} head {h}: {sorted(bad)[:10]} differ outside the band"
            n_near += len(diff)
    return n_near


def check_candidates_cover(rp, ci, verts, slashes, cu, hq, block):
    """Every (query, key) pair the token mask allows lies in a listed block of its row."""
    rp, ci = rp.cpu().numpy(), ci.cpu().numpy()
    lay = O.seq_layout(cu, block)
    nbt = sum(L["nb"] for L in lay)
    for s, L in enumerate(lay):
        n = L["n"]
        if n == 0:
            continue
        for h in range(hq):
            mask = PO.token_mask(n, np.asarray(verts[s][h], np.int64),
                                 np.asarray(slashes[s][h], np.int64))
            for I in range(L["nb"]):
                r = h * nbt + L["block_base"] + I
                listed = set(ci[rp[r]:rp[r + 1]].tolist())
                rows = mask[I * block:min((I + 1) * block, n)]
                need = set((np.nonzero(rows.any(axis=0))[0] // block).tolist())
                assert need <= listed, f"row (h={h}, s={s}, I={I}) misses blocks {need - listed}"
                assert all(J <= I for J in listed)


def run_case(w, n_probe, alpha_v, alpha_s):
    data = generate(w, workers=4)
    q64, k64, v64 = PT.oracle_inputs(data)
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.vs_workspace(pf, n_probe)
    # 1) pattern discovery
    vert, slash = fpx.probe_patterns(pf, dev["q"], dev["k"], n_probe, alpha_v, alpha_s, ws)
    assert fpx.status(ws) == 0
    found = PO.discover(q64, k64, cu, n_probe, alpha_v, alpha_s, with_near=True)
    ov = [f[0] for f in found]
    os_ = [f[1] for f in found]
    near_v = compare_sets(bits_to_sets(vert, cu, w.hq), ov, [f[2] for f in found], "verticals")
    near_s = compare_sets(bits_to_sets(slash, cu, w.hq), os_, [f[3] for f in found], "slashes")
    # 2) candidate blocks and 3) attention, both on the oracle's sets
    words = fpx.pattern_words(pf)
    vb = sets_to_bits(ov, cu, w.hq, words)
    sb = sets_to_bits(os_, cu, w.hq, words)
    rp, ci, nnz = fpx.vs_select(pf, vb, sb, ws)
    assert fpx.status(ws) == 0
    check_candidates_cover(rp, ci, ov, os_, cu, w.hq, w.block)
    o, lse = fpx.vs_prefill(pf, dev["q"], dev["k"], dev["v"], vb, sb, rp, ci, ws)
    assert fpx.status(ws) == 0
    masks = [[PO.token_mask(L["n"], np.asarray(ov[s][h], np.int64),
                            np.asarray(os_[s][h], np.int64)) for h in range(w.hq)]
             for s, L in enumerate(O.seq_layout(cu, 1))]
    o_ref, lse_ref = PO.attention_token_mask(q64, k64, v64, cu, masks)
    err = PT.compare_attention(o, lse, o_ref, lse_ref, w.dtype)
    # 4) the whole path on its own sets, when they agree with the oracle's
    if near_v == 0 and near_s == 0:
        out = fpx.vs_path(dev["q"], dev["k"], dev["v"], w.block, n_probe, alpha_v, alpha_s, cu,
                          q_scale=dev.get("q_scale"), k_scale=dev.get("k_scale"),
                          v_scale=dev.get("v_scale"))
        PT.compare_attention(out["o"], out["lse"], o_ref, lse_ref, w.dtype)
    n_v = sum(len(x) for per in ov for x in per)
    n_s = sum(len(x) for per in os_ for x in per)
    return dict(near=(near_v, near_s), verts=n_v, slashes=n_s, err=err,
                cand_density=int(nnz.item()) / max(1, w.hq * O.total_pairs(cu, w.block)))


CASES = {
    # (workload, n_probe, alpha_v, alpha_s)
    "gqa2_n1500": (BASE.with_(seqlens=(1500,), hq=4, hkv=2, q_gain=40.0), 32, 0.01, 0.01),
    "varlen_zero_len": (BASE.with_(seqlens=(300, 0, 129, 700, 1, 128), hq=4, hkv=1, q_gain=20.0),
                        16, 0.02, 0.05),
    "e4m3": (BASE.with_(seqlens=(900,), hq=2, hkv=1, dtype="e4m3", q_gain=20.0), 32, 0.01, 0.01),
    "one_tile_group1": (BASE.with_(seqlens=(1100,), hq=2, hkv=2, q_gain=40.0), 64, 0.05, 0.02),
    "three_tiles": (BASE.with_(seqlens=(1300,), hq=4, hkv=1, q_gain=40.0), 96, 0.01, 0.01),
    # odd group: 3 x 48 probe rows = one full tile and 16 rows; the attention's last unit of
    # each KV head holds one tile
    "gqa3_partial_tile": (BASE.with_(seqlens=(800, 333), hq=6, hkv=2, q_gain=40.0), 48, 0.01,
                          0.01),
    "four_tiles_gqa8": (BASE.with_(seqlens=(1000,), hq=8, hkv=1, q_gain=40.0), 64, 0.01, 0.01),
    "alpha_zero_is_dense": (BASE.with_(seqlens=(700,), hq=2, hkv=1), 8, 0.0, 0.0),
    "alpha_above_one_is_empty": (BASE.with_(seqlens=(500, 300), hq=2, hkv=1, q_gain=40.0), 8,
                                 1.5, 2.0),
    "verticals_only": (BASE.with_(seqlens=(1200,), hq=2, hkv=1, q_gain=40.0), 32, 0.01, 1.5),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_pattern_path_matches_oracle(name):
    w, n_probe, av, as_ = CASES[name]
    res = run_case(w, n_probe, av, as_)
    print(name, res)
    if name == "alpha_above_one_is_empty":
        assert res["verts"] == 0 and res["slashes"] == 0 and res["cand_density"] == 0


def test_alpha_zero_equals_dense_causal_attention():
    w = BASE.with_(seqlens=(900,), hq=4, hkv=2)
    dev = PT.to_device(generate(w))
    out = fpx.vs_path(dev["q"], dev["k"], dev["v"], w.block, 16, 0.0, 0.0, dev["cu_seqlens"])
    assert int(out["nnz"].item()) == w.hq * out["problem"].tri  # every causal block
    q = dev["q"].transpose(0, 1)[None].float()
    k = dev["k"].transpose(0, 1)[None].float().repeat_interleave(2, 1)
    v = dev["v"].transpose(0, 1)[None].float().repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    err = (out["o"].float() - ref[0].transpose(0, 1)).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


def test_pattern_entry_points_reject_bad_arguments():
    lib = fpx.load()
    w = BASE.with_(seqlens=(300,), hq=8, hkv=1)
    dev = PT.to_device(generate(w))
    pf = PT.gpu_problem(dev, w.block)
    assert lib.fpx_vs_workspace_bytes(pf.ptr, 65) == 0   # 8 heads x 65 probes > 512 rows
    assert lib.fpx_vs_workspace_bytes(pf.ptr, 0) == 0
    ws = fpx.vs_workspace(pf, 64)
    vb = torch.zeros((8, fpx.pattern_words(pf)), dtype=torch.int32, device="cuda")
    sb = torch.zeros_like(vb)
    call = lambda n, av, as_, size=ws.numel(): lib.fpx_probe_patterns(  # noqa: E731
        pf.ptr, dev["q"].data_ptr(), dev["k"].data_ptr(), n, av, as_, vb.data_ptr(),
        sb.data_ptr(), ws.data_ptr(), size, None)
    assert call(65, 0.1, 0.1) == -2
    assert call(64, float("nan"), 0.1) == -1
    assert call(64, 0.1, -0.5) == -1
    assert call(64, 0.1, 0.1, 16) == -4
    wf = BASE.with_(seqlens=(300,), hq=2, hkv=1, d=64)  # head dim 64: not on this path
    devf = PT.to_device(generate(wf))
    pff = PT.gpu_problem(devf, wf.block)
    assert lib.fpx_probe_patterns(pff.ptr, devf["q"].data_ptr(), devf["k"].data_ptr(), 8, 0.1,
                                  0.1, vb.data_ptr(), sb.data_ptr(), ws.data_ptr(), ws.numel(),
                                  None) == -2


FULL = [("llama8b_bf16_n32768", 64, 0.01, 0.01), ("llama8b_bf16_n131072", 64, 0.01, 0.01)]


@pytest.mark.parametrize("name,n_probe,av,as_", FULL, ids=[f[0] for f in FULL])
def test_pattern_path_full_size(name, n_probe, av, as_):
    """Full layer (q_gain 40, the labelled sparse-regime knob): every head's vertical and slash
    sets, and sampled attention rows (every head: the last token and two seeded random ones) on
    the oracle's sets."""
    w = WORKLOADS[name].with_(q_gain=40.0)
    data = generate(w, workers=default_workers())
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.vs_workspace(pf, n_probe)
    vert, slash = fpx.probe_patterns(pf, dev["q"], dev["k"], n_probe, av, as_, ws)
    words = fpx.pattern_words(pf)
    q, k, v = (data[x].float().numpy() for x in ("q", "k", "v"))
    found = PO.discover(q, k, cu, n_probe, av, as_, with_near=True)
    ov = [f[0] for f in found]
    os_ = [f[1] for f in found]
    near_v = compare_sets(bits_to_sets(vert, cu, w.hq), ov, [f[2] for f in found], "verticals")
    near_s = compare_sets(bits_to_sets(slash, cu, w.hq), os_, [f[3] for f in found], "slashes")
    vb = sets_to_bits(ov, cu, w.hq, words)
    sb = sets_to_bits(os_, cu, w.hq, words)
    rp, ci, nnz = fpx.vs_select(pf, vb, sb, ws)
    o, lse = fpx.vs_prefill(pf, dev["q"], dev["k"], dev["v"], vb, sb, rp, ci, ws)
    assert fpx.status(ws) == 0
    rng = np.random.default_rng(7)
    n = w.total_tokens
    rows = [(h, t) for h in range(w.hq) for t in [n - 1] + rng.integers(0, n, 2).tolist()]
    o_ref, lse_ref = PO.attention_token_rows(q, k, v, cu, ov, os_, rows)
    o_g = torch.stack([o[t, h] for h, t in rows])
    l_g = torch.stack([lse[h, t] for h, t in rows])
    err = PT.compare_attention(o_g, l_g, o_ref, lse_ref, w.dtype)
    n_v = sum(len(x) for per in ov for x in per)
    n_s = sum(len(x) for per in os_ for x in per)
    print(f"{name}: verticals={n_v} slashes={n_s} near={near_v}/{near_s} "
          f"candidate density={int(nnz.item()) / (w.hq * O.total_pairs(cu, w.block)):.4f} "
          f"O err={err}")
