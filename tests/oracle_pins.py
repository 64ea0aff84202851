"""Pins for the CPU oracle: checks against facts the FlashPrefill summary and plain mathematics
fix, each independent of the oracle's own code path.  Every check takes the oracle module as an
argument so that ``test_oracle_mutations.py`` can run the same checks on copies of the oracle
with a planted mistake and confirm that some check catches each one.

Sources of truth used here:
* library special cases: with alpha = 0 every causal block is kept, so the result must be dense
  causal attention -> torch's CPU scaled-dot-product attention in fp64 (with its LSE output);
  with an explicit block mask -> the same routine with an additive token mask;
* brute force on tiny inputs: block size 1 turns pooled block scores into token logits and the
  block threshold into a token threshold (pure-Python loops);
* linearity: a pooled score equals the block mean of token logits (compute-then-pool form);
* closed-form properties of the max-based threshold (FlashPrefill §3 and App. B): rows of the
  normalised scores sum to 1; alpha > 1 keeps exactly sink and window; alpha = 1 keeps exactly
  the row argmax plus sink and window; alpha = 0 keeps every causal block; the diagonal and sink
  are always kept with the default masks; a constant added to every key and a permutation of the
  tokens inside a block leave the selection unchanged;
* packing: a packed varlen batch equals running every sequence alone.
"""
from __future__ import annotations

import math

import numpy as np
import torch

F64 = torch.float64


def rand_problem(seqlens, hq, hkv, d, seed=0, scale_q=1.0):
    rng = np.random.default_rng(seed)
    t = int(sum(seqlens))
    q = rng.standard_normal((t, hq, d)) * scale_q
    k = rng.standard_normal((t, hkv, d))
    v = rng.standard_normal((t, hkv, d))
    cu = np.zeros(len(seqlens) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(seqlens)
    return q, k, v, cu


def sdpa_with_lse(q, k, v, scale, mask=None, causal=False):
    """torch CPU SDPA (fp64) for one sequence; q [n, Hq, D], k/v [n, Hkv, D] -> O [n,Hq,D], LSE
    [Hq, n].  GQA by repeating each KV head over its Q-head group."""
    hq, hkv = q.shape[1], k.shape[1]
    g = hq // hkv
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None].to(F64)
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None].to(F64)
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None].to(F64)
    kt = kt.repeat_interleave(g, dim=1)
    vt = vt.repeat_interleave(g, dim=1)
    kw = dict(scale=scale)
    if mask is not None:
        kw["attn_mask"] = torch.from_numpy(mask)[None].to(F64)
    o, lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(qt, kt, vt, 0.0, causal,
                                                                         **kw)
    return o[0].numpy().transpose(1, 0, 2), lse[0].numpy()


# ---------------------------------------------------------------------------------------------

def check_alpha0_is_dense_causal(O):
    seqlens = [77, 130]
    q, k, v, cu = rand_problem(seqlens, 4, 2, 16, seed=1)
    block = 32
    scale = 1 / math.sqrt(16)
    res = O.prefill(q, k, v, cu, block, alpha=0.0)
    # every causal block is kept
    for kp in res["keeps"]:
        nb = kp.shape[1]
        assert np.array_equal(kp, np.broadcast_to(np.tril(np.ones((nb, nb), bool)), kp.shape))
    for s in range(len(seqlens)):
        a, b = cu[s], cu[s + 1]
        o_ref, lse_ref = sdpa_with_lse(q[a:b], k[a:b], v[a:b], scale, causal=True)
        assert np.abs(res["o"][a:b] - o_ref).max() < 1e-10
        assert np.abs(res["lse"][:, a:b] - lse_ref).max() < 1e-10


def check_block1_bruteforce(O):
    n, hq, hkv, d = 19, 2, 1, 8
    q, k, v, cu = rand_problem([n], hq, hkv, d, seed=2, scale_q=2.0)
    scale = 0.37
    for alpha, sink, window in [(0.3, 1, 1), (0.05, 2, 3), (0.6, 0, 1), (2.0, 1, 2)]:
        res = O.prefill(q, k, v, cu, 1, alpha, sink, window, scale=scale)
        for h in range(hq):
            for i in range(n):
                logit = [scale * sum(q[i, h, c] * k[j, h // (hq // hkv), c] for c in range(d))
                         for j in range(i + 1)]
                for j in range(i + 1):
                    assert abs(res["scores"][0][h, i, j] - logit[j]) < 1e-12
                mx = max(logit)
                keep = []
                for j in range(i + 1):
                    ratio = math.exp(logit[j] - mx)
                    if abs(ratio - alpha) <= 1e-9:
                        continue  # tie with the threshold: rounding decides
                    want = ratio >= alpha or j < sink or j > i - window
                    assert bool(res["keeps"][0][h, i, j]) == want, (alpha, h, i, j)
                    if want:
                        keep.append(j)
                ls = [logit[j] for j in keep]
                m2 = max(ls)
                z = sum(math.exp(x - m2) for x in ls)
                lse = m2 + math.log(z)
                assert abs(res["lse"][h, i] - lse) < 1e-12
                for c in range(d):
                    oc = sum(math.exp(logit[j] - lse) * v[j, h // (hq // hkv), c] for j in keep)
                    assert abs(res["o"][i, h, c] - oc) < 1e-12


def check_pooled_score_is_block_mean_of_token_logits(O):
    seqlens = [150]
    hq, hkv, d, block = 4, 2, 8, 32
    q, k, v, cu = rand_problem(seqlens, hq, hkv, d, seed=3)
    scale = 0.5
    s = O.block_scores(q, k, cu, block, scale)[0]
    n = seqlens[0]
    nb = -(-n // block)
    for h in range(hq):
        tok = scale * (q[:, h, :] @ k[:, h // (hq // hkv), :].T)  # compute-then-pool form
        for I in range(nb):
            for J in range(nb):
                if J > I:
                    assert s[h, I, J] == -np.inf
                    continue
                blk = tok[I * block:min((I + 1) * block, n), J * block:min((J + 1) * block, n)]
                assert abs(s[h, I, J] - blk.mean()) < 1e-12


def check_normalised_rows_sum_to_one(O):
    q, k, v, cu = rand_problem([200, 64], 2, 1, 8, seed=4, scale_q=3.0)
    p = O.normalise(O.block_scores(q, k, cu, 16))
    for ps in p:
        nb = ps.shape[1]
        assert np.abs(ps.sum(axis=2) - 1.0).max() < 1e-12
        assert np.all(ps[:, ~np.tril(np.ones((nb, nb), bool))] == 0)
        assert np.all(ps >= 0)


def check_selection_special_cases(O):
    q, k, v, cu = rand_problem([300], 3, 1, 8, seed=5, scale_q=4.0)
    sc = O.block_scores(q, k, cu, 16)
    s = sc[0]
    nb = s.shape[1]
    I = np.arange(nb)[:, None]
    J = np.arange(nb)[None, :]
    causal = J <= I
    for sink, window in [(1, 1), (2, 3), (0, 1)]:
        keep = O.select(sc, 1.5, sink, window)[0][0]
        assert np.array_equal(keep, np.broadcast_to(causal & ((J < sink) | (J > I - window)),
                                                     keep.shape))
        keep = O.select(sc, 1.0, sink, window)[0][0]
        argmax = s == s.max(axis=2, keepdims=True)
        assert np.array_equal(keep, causal & (argmax | (J < sink) | (J > I - window)))
        keep = O.select(sc, 0.0, sink, window)[0][0]
        assert np.array_equal(keep, np.broadcast_to(causal, keep.shape))
    for alpha in [0.01, 0.3, 0.9, 5.0]:
        keep = O.select(sc, alpha)[0][0]
        diag = keep[:, np.arange(nb), np.arange(nb)]
        assert diag.all()
        assert keep[:, :, 0].all()
        assert not keep[:, ~causal].any()
    # CSR compression lists exactly the kept blocks, ascending, rows (h, s, I)
    keeps = O.select(sc, 0.3, 1, 1)[0]
    rp, ci = O.to_csr(keeps)
    r = 0
    for h in range(3):
        for I_ in range(nb):
            got = ci[rp[r]:rp[r + 1]]
            assert np.array_equal(got, np.nonzero(keeps[0][h, I_])[0])
            r += 1
    assert r == len(rp) - 1


def check_selection_invariances(O):
    q, k, v, cu = rand_problem([256], 2, 1, 8, seed=6, scale_q=5.0)
    block = 32
    alpha = 0.25
    sc = O.block_scores(q, k, cu, block)
    keep0, near0 = O.select(sc, alpha)
    # constant vector added to every key: row I shifts by scale * qbar_I . c
    c = np.random.default_rng(7).standard_normal(8) * 3.0
    sc_c = O.block_scores(q, k + c[None, None, :], cu, block)
    keep_c, _ = O.select(sc_c, alpha)
    ok = ~near0[0]
    assert np.array_equal(keep0[0][ok], keep_c[0][ok])
    # permuting tokens inside each block leaves the pooled scores unchanged
    perm = np.concatenate([b * block + np.random.default_rng(b).permutation(block)
                           for b in range(256 // block)])
    sc_p = O.block_scores(q[perm], k[perm], cu, block)
    assert np.abs(sc_p[0][np.isfinite(sc[0])] - sc[0][np.isfinite(sc[0])]).max() < 1e-12
    assert np.array_equal(O.select(sc_p, alpha)[0][0][ok], keep0[0][ok])
    # the score is linear in q: doubling q doubles every score
    sc_2 = O.block_scores(2 * q, k, cu, block)
    fin = np.isfinite(sc[0])
    assert np.abs(sc_2[0][fin] - 2 * sc[0][fin]).max() < 1e-12


def check_attention_given_mask(O):
    seqlens = [100, 57]
    hq, hkv, d, block = 4, 2, 16, 16
    q, k, v, cu = rand_problem(seqlens, hq, hkv, d, seed=8)
    scale = 0.3
    rng = np.random.default_rng(9)
    lay = O.seq_layout(cu, block)
    keeps = []
    for L in lay:
        nb = L["nb"]
        kp = (rng.random((hq, nb, nb)) < 0.5) & np.tril(np.ones((nb, nb), bool))
        kp[0, 1, :] = False  # one row with no kept block at all
        keeps.append(kp)
    rp, ci = O.to_csr(keeps)
    o, lse = O.attention(q, k, v, cu, block, rp, ci, scale)
    for s, L in enumerate(lay):
        a, b, n = L["start"], L["start"] + L["n"], L["n"]
        pos = np.arange(n)
        for h in range(hq):
            blockmask = keeps[s][h][pos[:, None] // block, pos[None, :] // block]
            allowed = blockmask & (pos[None, :] <= pos[:, None])
            mask = np.where(allowed, 0.0, -np.inf)[None].repeat(hq, 0)
            o_ref, lse_ref = sdpa_with_lse(q[a:b], k[a:b], v[a:b], scale, mask=mask)
            rows = allowed.any(axis=1)
            assert np.abs(o[a:b][rows, h] - o_ref[rows, h]).max() < 1e-10
            assert np.abs(lse[h, a:b][rows] - lse_ref[h][rows]).max() < 1e-10
            assert np.all(o[a:b][~rows, h] == 0)
            assert np.all(lse[h, a:b][~rows] == -np.inf)
        # sampled-row evaluation agrees with the full evaluation
    picks = [(0, 0), (3, 99), (1, 100), (2, 156), (0, 17)]
    o_s, lse_s = O.attention(q, k, v, cu, block, rp, ci, scale, rows=picks)
    for n_, (h, t) in enumerate(picks):
        assert np.abs(o_s[n_] - o[t, h]).max() < 1e-12
        assert lse_s[n_] == lse[h, t] or abs(lse_s[n_] - lse[h, t]) < 1e-12


def check_varlen_equals_separate(O):
    seqlens = [45, 0, 96, 33]
    hq, hkv, d, block = 2, 1, 8, 16
    q, k, v, cu = rand_problem(seqlens, hq, hkv, d, seed=10, scale_q=4.0)
    alpha = 0.2
    packed = O.prefill(q, k, v, cu, block, alpha)
    lay = O.seq_layout(cu, block)
    nbt = sum(L["nb"] for L in lay)
    for s, L in enumerate(lay):
        a, b = L["start"], L["start"] + L["n"]
        alone = O.prefill(q[a:b], k[a:b], v[a:b], np.array([0, L["n"]]), block, alpha)
        assert np.array_equal(packed["keeps"][s], alone["keeps"][0])
        assert np.abs(packed["o"][a:b] - alone["o"]).max() < 1e-12 if L["n"] else True
        for h in range(hq):
            for I in range(L["nb"]):
                r = h * nbt + L["block_base"] + I
                r1 = h * L["nb"] + I
                got = packed["col_idx"][packed["row_ptr"][r]:packed["row_ptr"][r + 1]]
                want = alone["col_idx"][alone["row_ptr"][r1]:alone["row_ptr"][r1 + 1]]
                assert np.array_equal(got, want)
                assert got.size == 0 or (got.min() >= 0 and got.max() <= I)


ALL_CHECKS = [
    check_alpha0_is_dense_causal,
    check_block1_bruteforce,
    check_pooled_score_is_block_mean_of_token_logits,
    check_normalised_rows_sum_to_one,
    check_selection_special_cases,
    check_selection_invariances,
    check_attention_given_mask,
    check_varlen_equals_separate,
]


def check_block_evaluation_matches_full(O):
    seqlens = [90, 200]
    q, k, v, cu = rand_problem(seqlens, 2, 1, 8, seed=11, scale_q=3.0)
    res = O.prefill(q, k, v, cu, 32, 0.3)
    picks = [(0, 0, 2), (1, 1, 6), (1, 0, 0)]
    out = O.attention(q, k, v, cu, 32, res["row_ptr"], res["col_idx"], blocks=picks)
    lay = O.seq_layout(cu, 32)
    for (h, s, I), (o, lse) in zip(picks, out):
        t0 = lay[s]["start"] + I * 32
        n = o.shape[0]
        assert np.abs(o - res["o"][t0:t0 + n, h]).max() < 1e-12
        with np.errstate(invalid="ignore"):  # -inf - -inf in a planted mistake: NaN fails below
            assert np.abs(lse - res["lse"][h, t0:t0 + n]).max() < 1e-12


ALL_CHECKS.append(check_block_evaluation_matches_full)


def check_near_band_is_exactly_the_unforced_ratios_within_the_band(O):
    """Hand-made score rows with known ratios exp(s - m): the near-threshold band must be exactly
    the causal, not forced (sink / window) blocks whose ratio lies within 1e-3 * alpha of alpha
    (the reporting rule for blocks whose decision rounding may flip).  Ratios sit at +-5e-4,
    -9e-4 (inside) and +-2e-3 (outside) relative to alpha; the sink and diagonal blocks are put
    inside the band to show that forced blocks are never reported."""
    nb, hq = 8, 2
    inside = {2: 1 + 5e-4, 3: 1 - 9e-4, 6: 1 - 5e-4}
    outside = {4: 1 + 2e-3, 5: 1 - 2e-3}
    for alpha in (0.05, 0.3, 0.9):
        s = np.full((hq, nb, nb), -np.inf)
        for h in range(hq):
            c = 0.37 - 1.3 * h  # a per-row offset cancels in s - max s
            for I in range(nb):
                for J in range(I + 1):
                    if J == I and I >= 2:
                        r = alpha * (1 + 1e-4)        # diagonal: forced, inside the band
                    elif J == 0 and I >= 1:
                        r = alpha * (1 - 1e-4)        # sink: forced, inside the band
                    elif J == 1 or I == 0:
                        r = 1.0                       # the row maximum
                    else:
                        r = alpha * {**inside, **outside}[J]
                    s[h, I, J] = c + math.log(r)
        keeps, nears = O.select([s], alpha, 1, 1)
        for h in range(hq):
            for I in range(nb):
                want_near = sorted(J for J in inside if J < I)
                want_keep = sorted({0, 1, I} & set(range(I + 1)) | {J for J in (2, 4) if J < I})
                assert np.nonzero(nears[0][h, I])[0].tolist() == want_near, (alpha, h, I)
                assert np.nonzero(keeps[0][h, I])[0].tolist() == want_keep, (alpha, h, I)
    keeps, nears = O.select([s], 0.0, 1, 1)  # alpha = 0: every causal block, nothing near
    assert not nears[0].any()
    assert np.array_equal(keeps[0], np.broadcast_to(np.tril(np.ones((nb, nb), bool)), s.shape))


def check_triangular_pack_matches_the_layout_formula(O):
    """Element (h, s, I, J <= I) of the packed scores sits at h * TRI + tri_base[s] + I (I + 1) / 2
    + J, tri_base[s] = sum over earlier sequences of nb (nb + 1) / 2 (the C ABI's score layout),
    checked on a varlen batch with ragged tails and a zero-length sequence."""
    seqlens, block, hq = [130, 0, 64, 1, 257], 64, 3
    nbs = [-(-n // block) for n in seqlens]
    tri_base, acc = [], 0
    for nb in nbs:
        tri_base.append(acc)
        acc += nb * (nb + 1) // 2
    tri = acc
    sc = []
    for si, nb in enumerate(nbs):
        a = np.full((hq, nb, nb), -np.inf)
        for h in range(hq):
            for I in range(nb):
                for J in range(I + 1):
                    a[h, I, J] = h * 1e6 + si * 1e4 + I * 100 + J
        sc.append(a)
    flat = np.asarray(O.triangular_pack(sc)).reshape(-1)
    assert flat.size == hq * tri
    seen = 0
    for h in range(hq):
        for si, nb in enumerate(nbs):
            for I in range(nb):
                for J in range(I + 1):
                    idx = h * tri + tri_base[si] + I * (I + 1) // 2 + J
                    assert flat[idx] == h * 1e6 + si * 1e4 + I * 100 + J, (h, si, I, J)
                    seen += 1
    assert seen == flat.size


ALL_CHECKS += [check_near_band_is_exactly_the_unforced_ratios_within_the_band,
               check_triangular_pack_matches_the_layout_formula]
