"""Paged K / V (FlashPrefill V2 abstract: native paged KV cache).  The packed K and V blocks are
scattered into a zero-filled cache of 128-token pages in a seeded random order; the paged entry
points must give scores and O / LSE identical, bit for bit, to the packed entry points on the same
data (same tiles, same arithmetic), and O / LSE must match the oracle on the packed K / V."""
import math

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
    "bf16_varlen": BASE.with_(seqlens=(300, 0, 129, 640, 1, 128), hq=4, hkv=1, q_gain=20.0),
    "bf16_gqa": BASE.with_(seqlens=(1000, 777), hq=8, hkv=2),
    "e4m3": BASE.with_(seqlens=(900, 260), hq=2, hkv=1, dtype="e4m3", q_gain=20.0),
}


def to_pages(x, cu, block, rng, spare=3):
    """Packed [T, H, D] -> (cache [num_pages * block, H, D], table [S, pages_per_seq], pages);
    unused table entries are -1 (never read)."""
    nbs = [math.ceil((cu[i + 1] - cu[i]) / block) for i in range(len(cu) - 1)]
    pps = max(1, max(nbs))
    num_pages = sum(nbs) + spare
    perm = rng.permutation(num_pages)
    cache = torch.zeros((num_pages * block,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    table = np.full((len(nbs), pps), -1, np.int32)
    k = 0
    for s, nb in enumerate(nbs):
        for J in range(nb):
            pg = int(perm[k])
            k += 1
            table[s, J] = pg
            a = int(cu[s]) + J * block
            b = min(int(cu[s + 1]), a + block)
            cache[pg * block: pg * block + (b - a)] = x[a:b]
    return cache, torch.from_numpy(table).cuda(), num_pages


@pytest.mark.parametrize("name", sorted(CASES))
def test_paged_equals_packed_and_oracle(name):
    w = CASES[name]
    data = generate(w, workers=4)
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    rng = np.random.default_rng(7)
    kc, table, npg = to_pages(dev["k"], cu, w.block, rng)
    vc, _, _ = to_pages(dev["v"], cu, w.block, np.random.default_rng(7))
    kv = fpx.paged_kv(table, npg)

    s_a = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    s_b = fpx.block_scores_paged(pf, dev["q"], kc, kv, ws)
    assert fpx.status(ws) == 0
    assert torch.equal(s_a, s_b)

    rp, ci, _ = fpx.select(pf, s_a, 0.1, ws)
    o_a, l_a = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, ci, ws)
    o_b, l_b = fpx.sparse_prefill_paged(pf, dev["q"], kc, vc, kv, rp, ci, ws)
    assert fpx.status(ws) == 0
    assert torch.equal(o_a, o_b) and torch.equal(l_a, l_b)

    q64, k64, v64 = PT.oracle_inputs(data)
    o_ref, lse_ref = O.attention(q64, k64, v64, cu, w.block, rp.cpu().numpy(), ci.cpu().numpy())
    PT.compare_attention(o_b, l_b, o_ref, lse_ref, w.dtype)


def test_paged_page_index_outside_the_cache_is_recorded():
    w = CASES["bf16_gqa"]
    data = generate(w, workers=4)
    cu = data["cu_seqlens"]
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    kc, table, npg = to_pages(dev["k"], cu, w.block, np.random.default_rng(3))
    vc, _, _ = to_pages(dev["v"], cu, w.block, np.random.default_rng(3))
    bad = table.clone()
    bad[0, 1] = npg + 5
    kv = fpx.paged_kv(bad, npg)
    s = fpx.block_scores_paged(pf, dev["q"], kc, kv, ws)
    assert fpx.status(ws) == -7
    fpx.clear_status(ws)
    rp, ci, _ = fpx.select(pf, s, 0.0, ws)
    o, lse = fpx.sparse_prefill_paged(pf, dev["q"], kc, vc, kv, rp, ci, ws)
    assert fpx.status(ws) == -7
    # the context stays usable and the good table still gives the packed result
    fpx.clear_status(ws)
    good = fpx.paged_kv(table, npg)
    o2, _ = fpx.sparse_prefill_paged(pf, dev["q"], kc, vc, good, rp, ci, ws)
    o3, _ = fpx.sparse_prefill(pf, dev["q"], dev["k"], dev["v"], rp, ci, ws)
    assert fpx.status(ws) == 0
    assert torch.equal(o2, o3)
