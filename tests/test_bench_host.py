"""Host-side logic of bench.py without a GPU: the max-over-ranks reduction and the weak-scaling
aggregate on world_size-2 gloo process groups, and the reference arm's contract (rank 0 prints
one JSON line, other ranks exit 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port():
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
        val = bench.aggregate_value(1e12, world, got[0])
        q.put((rank, got, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p_ in procs:
        p_.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p_ in procs:
        p_.join(timeout=60)
        assert p_.exitcode == 0
    for rank, got, val in res:
        assert got == [11.0, 5.0]          # max over ranks, element-wise
        assert val == pytest.approx(2 * 1e12 / 11e-3 / 1e12)  # whole-job aggregate


def test_single_process_identity():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.aggregate_value(2e12, 1, 1000.0) == pytest.approx(2.0)


def run_ref(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny_fp32_n2048", "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)


def test_reference_arm_rank_contract():
    r1 = run_ref(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = run_ref(0)
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_traffic_is_reported_only_for_the_measured_sources(monkeypatch):
    # sources with the recorded digest: the measured bytes; a workload never measured: null
    monkeypatch.setattr(bench, "ATTN_TRAFFIC_DIGEST", bench.attn_sources_digest())
    assert bench.attn_traffic("llama8b_bf16_n131072") == bench.ATTN_TRAFFIC["llama8b_bf16_n131072"]
    assert bench.attn_traffic("varlen8_bf16_t264192") is None
    # kernel sources that differ from the captured ones: null
    monkeypatch.setattr(bench, "ATTN_TRAFFIC_DIGEST", "0" * 64)
    assert bench.attn_traffic("llama8b_bf16_n131072") is None


@pytest.mark.parametrize("alpha,sink,window", [(1.0, 1, 1), (1.0, 0, 2), (0.0, 1, 1)])
def test_selection_stats_match_the_oracle(alpha, sink, window):
    """bench.selection_stats on a varlen problem (a ragged tail and a zero-length sequence, odd
    GQA group): the near-threshold count equals the oracle's near mask, and the K/V tile loads
    equal the brute-force union of each unit's two heads' kept blocks."""
    import numpy as np
    from oracle import fpx_oracle as O
    rng = np.random.default_rng(7)
    seqlens, hq, hkv, d, block = (70, 0, 33, 128), 6, 2, 16, 16
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    t = int(cu[-1])
    q = rng.standard_normal((t, hq, d)) * 3.0
    k = rng.standard_normal((t, hkv, d))
    sc = O.block_scores(q, k, cu, block)
    if alpha > 0:
        # put alpha beside the ratio of an unforced causal block so that the band is not empty
        s0 = sc[0][1]  # sequence 0, Q head 1: [nb, nb]
        I = s0.shape[0] - 1
        J = I - window if sink <= I - window else 0
        alpha = float(np.exp(s0[I, J] - s0[I, :I + 1].max())) * (1 + 4e-4)
    keeps, nears = O.select(sc, alpha, sink, window)
    if alpha > 0:
        assert sum(int(n.sum()) for n in nears) >= 1
    rp, ci = O.to_csr(keeps)
    scores = torch.from_numpy(O.triangular_pack(sc).astype(np.float32).reshape(-1))
    st = bench.selection_stats(scores, torch.from_numpy(rp.astype(np.int32)),
                               torch.from_numpy(ci.astype(np.int32) if ci.size else
                                                np.zeros(1, np.int32)),
                               cu, hq, hkv, block, alpha, sink, window)
    assert st["near_threshold_blocks"] == sum(int(n.sum()) for n in nears)
    g = hq // hkv
    loads = 0
    for kp in keeps:  # [hq, nb, nb] per sequence
        for kvh in range(hkv):
            for h0 in range(kvh * g, (kvh + 1) * g, 2):
                u = kp[h0] | kp[h0 + 1] if h0 + 1 < (kvh + 1) * g else kp[h0]
                loads += int(u.sum())
    assert st["kv_tile_loads"] == loads
    assert st["union_excess_tiles"] == 0
