"""Planted mistakes in the rescue-branch and query-probe oracles: each test copies the oracle,
plants one plausible mistake in the copy (on the CPU) and checks that at least one of that
oracle's pins rejects the copy."""
import importlib.util
import types

import pytest

import test_oracle_pattern as PP
import test_oracle_rescue as RP

MUTATIONS = {
    "rescue": ("oracle.rescue_oracle", RP, {
        "radius_mean_not_max": ("np.sqrt(((rows - centre) ** 2).sum(axis=2)).max(axis=0)",
                                "np.sqrt(((rows - centre) ** 2).sum(axis=2)).mean(axis=0)"),
        "radius_squared": ("np.sqrt(((rows - centre) ** 2).sum(axis=2)).max(axis=0)",
                           "((rows - centre) ** 2).sum(axis=2).max(axis=0)"),
        "radius_from_origin": ("(rows - centre) ** 2", "rows ** 2"),
        "bonus_sign": ("u[h] = s[h] + sc *", "u[h] = s[h] - sc *"),
        "bonus_unscaled": ("u[h] = s[h] + sc *", "u[h] = s[h] + 1.0 *"),
        "norm_of_mean_of_norms": (
            "return [np.sqrt((O.pool_blocks(q, L[\"start\"], L[\"n\"], block) ** 2).sum(axis=2))",
            "return [O.pool_blocks(np.sqrt((np.asarray(q, np.float64) ** 2).sum(axis=2, keepdims=True))"
            "[..., 0:1], L[\"start\"], L[\"n\"], block)[..., 0]"),
        "rescue_kv_head_modulo": ("r[:, h // g][None, :]", "r[:, h % hkv][None, :]"),
        "rescue_replaces_base": ("keeps.append(kb | kr)", "keeps.append(kr)"),
        "rescue_threshold_on_s": ("ratio = np.exp(u - u.max(axis=2, keepdims=True))",
                                  "ratio = np.exp(s_ - s_.max(axis=2, keepdims=True))"),
    }),
    "pattern": ("oracle.pattern_oracle", PP, {
        "probes_skip_last": ("math.ceil((p + 1) * n / m) - 1", "math.ceil(p * n / m)"),
        "vertical_sum_not_max": ("v[:i + 1] = np.maximum(v[:i + 1], a[h, p, :i + 1])",
                                 "v[:i + 1] = v[:i + 1] + a[h, p, :i + 1]"),
        "slash_reversed": ("a[h, p, i::-1]", "a[h, p, :i + 1]"),
        "slash_mask_offset_sign": ("iss[np.clip(i - j, 0, n - 1)]", "iss[np.clip(j - i, 0, n - 1)]"),
        "mask_not_causal": ("return (j <= i) & (", "return (j >= 0) & ("),
        "probe_not_causal": ("logits = scale * (kk[:i + 1] @", "logits = scale * (kk[:i + 2] @"),
        "attn_scale_dropped": ("logits = np.where(masks[s_][h], sc * (qq @ kk.T), -np.inf)",
                               "logits = np.where(masks[s_][h], (qq @ kk.T), -np.inf)"),
        "threshold_inverted": ("np.nonzero(x >= alpha * x.max())", "np.nonzero(x <= alpha * x.max())"),
        "near_band_x10": ("np.abs(x - thr) <= O.NEAR_REL * thr", "np.abs(x - thr) <= 10 * O.NEAR_REL * thr"),
        "near_band_absolute": ("np.abs(x - thr) <= O.NEAR_REL * thr", "np.abs(x - thr) <= O.NEAR_REL"),
        "token_rows_offset_sign": ("keys = j[isv[j] | iss[i - j]]", "keys = j[isv[j] | iss[j]]"),
        "token_rows_not_causal": ("j = np.arange(i + 1)", "j = np.arange(min(i + 2, n))"),
        "probe_kv_head_modulo": ("k[start:start + n, h // g]", "k[start:start + n, h % k.shape[1]]"),
        "probe_scale_dropped": ("logits = scale * (kk[:i + 1] @", "logits = (kk[:i + 1] @"),
        "probe_rows_not_normalised": ("a[h, p, :i + 1] = e / e.sum()", "a[h, p, :i + 1] = e"),
    }),
}

CASES = [(o, n) for o, (_, _, muts) in MUTATIONS.items() for n in sorted(muts)]


def mutated(modname, old, new, tag):
    src = open(importlib.util.find_spec(modname).origin).read()
    src = src.replace("from . import fpx_oracle as O", "from oracle import fpx_oracle as O")
    if tag == "rescue_threshold_on_s":
        src = src.replace("for kb, nbase, u in zip(base_keep, base_near, rescue):",
                          "for kb, nbase, u, s_ in zip(base_keep, base_near, rescue, scores):")
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType(f"mutant_{tag}")
    exec(compile(src.replace(old, new), f"<mutant {tag}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("oracle,name", CASES, ids=[f"{o}-{n}" for o, n in CASES])
def test_planted_mistake_is_caught(oracle, name):
    modname, pins, muts = MUTATIONS[oracle]
    old, new = muts[name]
    mod = mutated(modname, old, new, name)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, ValueError, IndexError, FloatingPointError, TypeError):
            caught.append(check.__name__)
    assert caught, f"no pin rejects the planted mistake {oracle}/{name}"
