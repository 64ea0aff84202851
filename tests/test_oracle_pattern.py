"""Pins of the query-probe vertical / slash oracle (oracle/pattern_oracle.py): probe placement,
the dense limit against a library attention, planted vertical and slash structure, brute force
of token-masked attention, threshold edge cases."""
import numpy as np
import torch

from oracle import fpx_oracle as O
from oracle import pattern_oracle as PO


def check_probe_positions_are_uniform_and_end_at_the_last_token(PO=PO):
    assert PO.probe_positions(100, 4).tolist() == [24, 49, 74, 99]
    assert PO.probe_positions(5, 10).tolist() == [0, 1, 2, 3, 4]  # at most one probe per token
    assert PO.probe_positions(7, 1).tolist() == [6]
    assert PO.probe_positions(0, 4).size == 0


def check_alpha_zero_is_dense_causal_attention(PO=PO):
    rng = np.random.default_rng(0)
    t, hq, hkv, d = 40, 2, 1, 8
    q, k, v = (rng.standard_normal((t, h, d)) for h in (hq, hkv, hkv))
    cu = [0, 15, 40]
    found = PO.discover(q, k, cu, 4, 0.0, 0.5)
    masks = [[PO.token_mask(n, vs[h], ss[h]) for h in range(hq)]
             for n, (vs, ss) in zip([15, 25], found)]
    o, lse = PO.attention_token_mask(q, k, v, cu, masks)
    for a, b in ((0, 15), (15, 40)):
        qq = torch.from_numpy(q[a:b]).permute(1, 0, 2)[None]
        kk = torch.from_numpy(np.repeat(k[a:b], hq // hkv, axis=1)).permute(1, 0, 2)[None]
        vv = torch.from_numpy(np.repeat(v[a:b], hq // hkv, axis=1)).permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
        assert np.allclose(o[a:b], ref[0].permute(1, 0, 2).numpy(), atol=1e-12)


def check_planted_vertical_and_slash_are_found(PO=PO):
    rng = np.random.default_rng(1)
    n, d, star, delta = 64, 16, 5, 3
    base = rng.standard_normal(d)
    q = (4.0 * base + 0.1 * rng.standard_normal((n, d)))[:, None, :]
    k = 0.1 * rng.standard_normal((n, 1, d))
    k[star, 0] = 3.0 * base  # every query attends token `star`
    verts, _ = PO.discover(q, k, [0, n], 8, 0.5, 2.0)[0]
    assert star in verts[0]
    # slash: key j points at query j + delta, so every query's best key sits `delta` back
    q2 = rng.standard_normal((n, 1, d)) * 3.0
    k2 = 0.1 * rng.standard_normal((n, 1, d))
    k2[:n - delta, 0] = q2[delta:, 0]
    _, slashes = PO.discover(q2, k2, [0, n], 8, 2.0, 0.9)[0]
    assert delta in slashes[0]
    mask = PO.token_mask(n, np.zeros(0, int), slashes[0])
    assert all(mask[i, i - delta] for i in range(delta, n))
    assert not any(mask[i, i + 1] for i in range(n - 1))  # causal


def check_token_masked_attention_matches_brute_force(PO=PO):
    rng = np.random.default_rng(2)
    n, d = 12, 4
    q, k, v = (rng.standard_normal((n, 1, d)) for _ in range(3))
    verts, slashes = np.array([0, 7]), np.array([0, 2])
    mask = PO.token_mask(n, verts, slashes)
    o, lse = PO.attention_token_mask(q, k, v, [0, n], [[mask]])
    sc = 1.0 / np.sqrt(d)
    for i in range(n):
        js = [j for j in range(i + 1) if j in verts or (i - j) in slashes]
        lg = np.array([sc * q[i, 0] @ k[j, 0] for j in js])
        w = np.exp(lg - lg.max())
        assert np.allclose(o[i, 0], (w[:, None] * v[js, 0]).sum(0) / w.sum())
        assert np.isclose(lse[0, i], lg.max() + np.log(w.sum()))


def check_threshold_edges(PO=PO):
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((20, 2, 4)), rng.standard_normal((20, 1, 4))
    verts, slashes = PO.discover(q, k, [0, 20], 5, 1.5, 1.5)[0]
    assert all(x.size == 0 for x in verts) and all(x.size == 0 for x in slashes)
    verts, slashes = PO.discover(q, k, [0, 20], 5, 1.0, 1.0)[0]
    assert all(x.size >= 1 for x in verts) and all(x.size >= 1 for x in slashes)  # the maxima


def check_aggregation_over_probes_is_the_max(PO=PO):
    # probe rows given directly: key 0 gets 0.6 from one probe, key 1 gets 0.35 from three;
    # the max reading keeps key 0 (a sum would prefer key 1); offsets likewise
    a = np.zeros((1, 3, 4))
    a[0, 0, :2] = [0.6, 0.4]            # probe at position 1
    a[0, 1, :3] = [0.3, 0.35, 0.35]     # probe at position 2
    a[0, 2, :4] = [0.3, 0.35, 0.0, 0.35]  # probe at position 3
    verts, slashes = PO.vertical_slash(a, np.array([1, 2, 3]), 0.9, 0.9)
    assert verts[0].tolist() == [0]
    # slash offsets: probe 1 -> {0: 0.4, 1: 0.6}; probe 2 -> {0: .35, 1: .35, 2: .3};
    # probe 3 -> {0: .35, 1: 0, 2: .35, 3: .3}: max per offset 0.4, 0.6, 0.35, 0.3
    assert slashes[0].tolist() == [1]


def check_near_threshold_band(PO=PO):
    # significances placed at known distances from alpha * max: inside the 1e-3 relative band
    # (+-5e-4, -9e-4 of the threshold) and outside it (+-2e-3)
    for alpha in (0.05, 0.3, 0.9):
        x = np.array([1.0, alpha * (1 + 5e-4), alpha * (1 - 9e-4), alpha * (1 + 2e-3),
                      alpha * (1 - 2e-3), alpha * (1 - 5e-4), 0.0]) * 0.37
        assert PO.near_threshold(x, alpha).tolist() == [1, 2, 5]
        assert PO._select_max_based(x, alpha).tolist() == [0, 1, 3]
    assert PO.near_threshold(x, 0.0).size == 0
    assert PO.near_threshold(np.zeros(0), 0.5).size == 0


def check_token_rows_equal_full_token_mask_attention(PO=PO):
    rng = np.random.default_rng(4)
    t, hq, hkv, d = 50, 2, 1, 8
    q, k, v = (rng.standard_normal((t, h, d)) for h in (hq, hkv, hkv))
    cu = [0, 21, 21, 50]
    verts = [[np.array([0, 5]), np.array([3])], [[], []], [np.array([1, 20]), np.array([])]]
    slashes = [[np.array([0, 2]), np.array([4])], [[], []], [np.array([0]), np.array([1, 7])]]
    masks = [[PO.token_mask(n, np.asarray(vs[h], int), np.asarray(ss[h], int)) for h in range(hq)]
             for n, vs, ss in zip([21, 0, 29], verts, slashes)]
    o, lse = PO.attention_token_mask(q, k, v, cu, masks)
    # includes rows whose next key is a vertical (0, 4) and (1, 2): a non-causal row would see it
    rows = [(0, 0), (1, 0), (1, 3), (0, 20), (1, 21), (0, 49), (1, 30), (0, 25), (0, 4), (1, 2)]
    o_r, lse_r = PO.attention_token_rows(q, k, v, cu, verts, slashes, rows)
    for n_, (h, t_) in enumerate(rows):
        assert lse_r[n_] == lse[h, t_] or abs(lse_r[n_] - lse[h, t_]) < 1e-12
        assert np.abs(o_r[n_] - o[t_, h]).max() < 1e-12
    assert np.isneginf(lse_r[1]) and not o_r[1].any()  # head 1, token 0: no key at all


def check_probe_rows_are_causal_softmax_rows(PO=PO):
    # the probe rows are exact causal attention rows (FlashPrefill §3, query probes): against
    # torch's softmax of the masked logits, with GQA (Q head h reads KV head h / (Hq / Hkv)) and
    # a sequence that starts inside the token array
    rng = np.random.default_rng(5)
    t, hq, hkv, d, start, n, sc = 30, 4, 2, 8, 3, 25, 0.37
    q, k = rng.standard_normal((t, hq, d)), rng.standard_normal((t, hkv, d))
    pos = PO.probe_positions(n, 5)
    a = PO.probe_attention(q, k, start, n, pos, sc, hq // hkv)
    causal = torch.ones(n, n, dtype=torch.bool).tril()
    for h in range(hq):
        qq = torch.from_numpy(q[start:start + n, h])
        kk = torch.from_numpy(k[start:start + n, h * hkv // hq])
        ref = torch.softmax((sc * qq @ kk.T).masked_fill(~causal, float("-inf")), dim=-1)
        assert np.allclose(a[h], ref[torch.from_numpy(pos)].numpy(), atol=1e-12)


ALL_CHECKS = [check_probe_rows_are_causal_softmax_rows, check_near_threshold_band, check_token_rows_equal_full_token_mask_attention,
              check_probe_positions_are_uniform_and_end_at_the_last_token,
              check_alpha_zero_is_dense_causal_attention, check_planted_vertical_and_slash_are_found,
              check_token_masked_attention_matches_brute_force, check_threshold_edges,
              check_aggregation_over_probes_is_the_max]


def test_probe_positions_are_uniform_and_end_at_the_last_token():
    check_probe_positions_are_uniform_and_end_at_the_last_token()


def test_alpha_zero_is_dense_causal_attention():
    check_alpha_zero_is_dense_causal_attention()


def test_planted_vertical_and_slash_are_found():
    check_planted_vertical_and_slash_are_found()


def test_token_masked_attention_matches_brute_force():
    check_token_masked_attention_matches_brute_force()


def test_threshold_edges():
    check_threshold_edges()


def test_aggregation_over_probes_is_the_max():
    check_aggregation_over_probes_is_the_max()


def test_near_threshold_band():
    check_near_threshold_band()


def test_probe_rows_are_causal_softmax_rows():
    check_probe_rows_are_causal_softmax_rows()


def test_token_rows_equal_full_token_mask_attention():
    check_token_rows_equal_full_token_mask_attention()
