"""alpha calibration and retention presets (FlashPrefill App. A, "Hyperparameter
Configurations").  Host logic on CPU; the GPU test bisects on fpx_select itself and checks the
result against the oracle's selection."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_pooled_b200 import calibrate as CAL


def test_retention_blocks_match_the_pages_at_block_128():
    assert CAL.retention_blocks(128) == (2, 4)
    assert CAL.retention_blocks(64) == (4, 8)
    assert CAL.retention_blocks(100) == (3, 6)  # rounded up: at least 256 / 512 tokens kept


def test_bisect_finds_the_largest_alpha_meeting_the_target():
    steps = np.linspace(0.0, 1.0, 1001)

    def density_of(a):  # non-increasing step function, density(0) = 1
        return float(1.0 - 0.9 * steps[np.searchsorted(steps, a, side="right") - 1])

    for target in (0.95, 0.7, 0.31, 0.1):
        a, d = CAL.bisect_alpha(density_of, target)
        assert d >= target and d == density_of(a)
        assert density_of(a + 2e-3) < target  # one step further drops below the target


def test_bisect_edges():
    f = lambda a: 1.0 - 0.5 * a  # noqa: E731
    assert CAL.bisect_alpha(f, 1.0) == (0.0, 1.0)
    assert CAL.bisect_alpha(f, 0.4) == (1.0, 0.5)  # below the floor at alpha = 1
    with pytest.raises(ValueError):
        CAL.bisect_alpha(f, 1.5)


@pytest.mark.gpu
def test_calibrated_alpha_reproduces_the_target_density():
    import dynamic_block_sparse_pooled_b200 as fpx
    from gen import WORKLOADS, generate
    from oracle import fpx_oracle as O
    import parity as PT

    # a 4096-token bf16 layer with a logit gain that makes the selection genuinely sparse
    w = WORKLOADS["llama8b_bf16_n8192"].with_(seqlens=(4096,), q_gain=300.0)
    data = generate(w)
    dev = PT.to_device(data)
    pf = PT.gpu_problem(dev, w.block)
    ws = fpx.workspace(pf, -1)
    scores = fpx.block_scores(pf, dev["q"], dev["k"], ws)
    sink, window = CAL.retention_blocks(w.block)
    alpha, dens = CAL.calibrate_alpha(pf, scores, CAL.PAGES_TARGET_DENSITY_4K, ws, sink, window)
    assert fpx.status(ws) == 0
    assert dens >= CAL.PAGES_TARGET_DENSITY_4K
    # the oracle's selection at the calibrated alpha has the same density (up to blocks in the
    # near-threshold band)
    q, k = (data[x].float().numpy() for x in ("q", "k"))
    s_list = O.block_scores(q, k, data["cu_seqlens"], w.block)
    keeps, nears = O.select(s_list, alpha, sink, window)
    kept = sum(int(np.sum(kp)) for kp in keeps)
    near = sum(int(np.sum(nr)) for nr in nears)
    total = w.hq * O.total_pairs(data["cu_seqlens"], w.block)
    assert abs(kept - dens * total) <= near
    print(f"alpha={alpha:.5f} density={dens:.4f} oracle={kept / total:.4f} near={near}")
