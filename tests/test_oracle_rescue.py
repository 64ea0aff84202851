"""Pins of the rescue-branch oracle (oracle/rescue_oracle.py) against facts fixed by the
mathematics: Cauchy-Schwarz bound on every token logit, closed-form radii, reductions to the base
selection, monotonicity."""
import numpy as np

from oracle import fpx_oracle as O
from oracle import rescue_oracle as R


def _rand(seed, t, hq, hkv, d):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((t, hq, d)), rng.standard_normal((t, hkv, d))


def check_rescue_score_bounds_every_token_logit_of_the_block(R=R):
    q, k = _rand(0, 23, 4, 2, 8)
    cu, block, g = [0, 9, 23], 4, 2
    sc = O.default_scale(8)
    for s_i, (L, u) in enumerate(zip(O.seq_layout(cu, block), R.rescue_scores(q, k, cu, block))):
        qb = O.pool_blocks(q, L["start"], L["n"], block)
        for h in range(4):
            for I in range(L["nb"]):
                for J in range(I + 1):
                    a = L["start"] + J * block
                    b = L["start"] + min((J + 1) * block, L["n"])
                    best = max(sc * float(qb[I, h] @ k[j, h // g]) for j in range(a, b))
                    assert u[h, I, J] >= best - 1e-12
                    if b - a == 1:  # one key: radius 0, the bound is the logit itself
                        assert abs(u[h, I, J] - best) <= 1e-12


def check_radius_closed_forms(R=R):
    d = 5
    rng = np.random.default_rng(1)
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    k = np.stack([a, b])[:, None, :]
    assert np.isclose(R.block_radius(k, [0, 2], 2)[0][0, 0], np.linalg.norm(a - b) / 2)
    # three keys at 0, 0, 3e along one axis: centroid e, distances 1, 1, 2 -> radius 2 (the max)
    e = np.zeros(d)
    e[2] = 1.0
    k3 = np.stack([0 * e, 0 * e, 3 * e])[:, None, :]
    assert np.isclose(R.block_radius(k3, [0, 3], 4)[0][0, 0], 2.0)
    # identical keys: radius 0; translation invariance; |c| scaling
    same = np.repeat(a[None, None, :], 4, axis=0)
    assert R.block_radius(same, [0, 4], 4)[0][0, 0] == 0.0
    kk = rng.standard_normal((8, 2, d))
    r0 = R.block_radius(kk, [0, 8], 4)[0]
    assert np.allclose(R.block_radius(kk + rng.standard_normal(d), [0, 8], 4)[0], r0)
    assert np.allclose(R.block_radius(-2.5 * kk, [0, 8], 4)[0], 2.5 * r0)


def check_query_norm_is_the_pooled_query_norm(R=R):
    # antipodal query tokens pool to zero: no rescue bonus, u == s
    d = 6
    rng = np.random.default_rng(2)
    v = rng.standard_normal(d)
    q = np.stack([v, -v, v, -v])[:, None, :]
    k = rng.standard_normal((4, 1, d))
    assert np.isclose(R.query_norms(q, [0, 4], 4)[0][0, 0], 0.0)
    u = R.rescue_scores(q, k, [0, 4], 4)[0]
    s = O.block_scores(q, k, [0, 4], 4)[0]
    assert np.allclose(u[np.isfinite(s)], s[np.isfinite(s)])


def check_reductions_to_the_base_selection(R=R):
    q, k = _rand(3, 40, 2, 1, 8)
    cu, block = [0, 40], 4
    s = O.block_scores(q, k, cu, block)
    u = R.rescue_scores(q, k, cu, block)
    base, _ = O.select(s, 0.3)
    off, _ = R.select_rescue(s, u, 0.3, 1.5)            # alpha_r > 1: the branch keeps nothing
    assert all(np.array_equal(x, y) for x, y in zip(base, off))
    # every block's keys identical (radius 0) -> u == s and the branches coincide at alpha_r = alpha
    kk = np.repeat(k[::4], 4, axis=0)
    s0 = O.block_scores(q, kk, cu, block)
    u0 = R.rescue_scores(q, kk, cu, block)
    assert all(np.allclose(a[np.isfinite(a)], b[np.isfinite(b)]) for a, b in zip(s0, u0))
    b0, _ = O.select(s0, 0.3)
    c0, _ = R.select_rescue(s0, u0, 0.3, 0.3)
    assert all(np.array_equal(x, y) for x, y in zip(b0, c0))


def check_union_and_monotonicity(R=R):
    q, k = _rand(4, 64, 2, 2, 8)
    cu, block = [0, 25, 64], 4
    s = O.block_scores(q, k, cu, block)
    u = R.rescue_scores(q, k, cu, block)
    base, _ = O.select(s, 0.5)
    lo, _ = R.select_rescue(s, u, 0.5, 0.2)
    hi, _ = R.select_rescue(s, u, 0.5, 0.6)
    for b_, l_, h_ in zip(base, lo, hi):
        assert np.all(l_ >= b_) and np.all(h_ >= b_) and np.all(l_ >= h_)
    assert sum(int(x.sum()) for x in lo) > sum(int(x.sum()) for x in base)


def check_bound_is_tight_when_the_far_key_points_along_the_query(R=R):
    # two keys c +- delta * qhat per block: centroid c, radius delta, and the best token logit
    # is exactly scale * (<qbar, c> + delta * |qbar|) = u (per KV head, different deltas)
    rng = np.random.default_rng(5)
    d, hq, hkv = 8, 4, 2
    qdir = rng.standard_normal((hkv, d))
    q = np.zeros((2, hq, d))
    for h in range(hq):
        q[:, h] = (h + 1.0) * qdir[h // 2]
    k = np.zeros((2, hkv, d))
    for kvh, delta in enumerate((0.7, 1.9)):
        c = rng.standard_normal(d)
        qhat = qdir[kvh] / np.linalg.norm(qdir[kvh])
        k[0, kvh], k[1, kvh] = c + delta * qhat, c - delta * qhat
    u = R.rescue_scores(q, k, [0, 2], 2)[0]
    sc = O.default_scale(d)
    for h in range(hq):
        best = max(sc * float(q[0, h] @ k[j, h // 2]) for j in range(2))
        assert np.isclose(u[h, 0, 0], best, rtol=1e-12, atol=1e-12)


def check_only_the_far_key_block_is_rescued(R=R):
    # four key blocks with the same centroid (equal centroid scores); block 2 hides one far key
    rng = np.random.default_rng(6)
    d = 8
    c = rng.standard_normal(d)
    q = np.tile(rng.standard_normal(d), (16, 1))[:, None, :]
    k = np.tile(c, (16, 1))[:, None, :].copy()
    far = rng.standard_normal(d)
    k[8, 0] = c + 3.0 * far
    k[9, 0] = c - 3.0 * far  # keeps the block's centroid at c
    s = O.block_scores(q, k, [0, 16], 4)
    u = R.rescue_scores(q, k, [0, 16], 4)
    keep, _ = R.select_rescue(s, u, 2.0, 0.99, sink_blocks=0, window_blocks=0)
    assert keep[0][0, 3].tolist() == [False, False, True, False]


ALL_CHECKS = [check_rescue_score_bounds_every_token_logit_of_the_block, check_radius_closed_forms,
              check_query_norm_is_the_pooled_query_norm, check_reductions_to_the_base_selection,
              check_union_and_monotonicity,
              check_bound_is_tight_when_the_far_key_points_along_the_query,
              check_only_the_far_key_block_is_rescued]


def test_rescue_score_bounds_every_token_logit_of_the_block():
    check_rescue_score_bounds_every_token_logit_of_the_block()


def test_radius_closed_forms():
    check_radius_closed_forms()


def test_query_norm_is_the_pooled_query_norm():
    check_query_norm_is_the_pooled_query_norm()


def test_reductions_to_the_base_selection():
    check_reductions_to_the_base_selection()


def test_union_and_monotonicity():
    check_union_and_monotonicity()


def test_bound_is_tight_when_the_far_key_points_along_the_query():
    check_bound_is_tight_when_the_far_key_points_along_the_query()


def test_only_the_far_key_block_is_rescued():
    check_only_the_far_key_block_is_rescued()
