"""Planted mistakes: each test copies the oracle, plants one plausible mistake in the copy (on
the CPU, never in the CUDA path) and checks that at least one pin rejects the copy."""
import importlib.util
import types

import pytest

import oracle_pins as P

SRC = importlib.util.find_spec("oracle.fpx_oracle").origin

MUTATIONS = {
    "kv_head_modulo": ("kb[:, h // g, :]", "kb[:, h % hkv, :]"),
    "scores_transposed": ("full = sc * (qb[:, h, :] @ kb[:, h // g, :].T)",
                          "full = (sc * (qb[:, h, :] @ kb[:, h // g, :].T)).T"),
    "score_scale_dropped": ("full = sc * (qb", "full = 1.0 * (qb"),
    "pool_divides_by_block": ("rows.sum(axis=0) / rows.shape[0]", "rows.sum(axis=0) / block"),
    "threshold_strict": ("(ratio >= alpha)", "(ratio > alpha)"),
    "threshold_on_probability": ("ratio = np.exp(s - m)",
                                 "ratio = np.exp(s - m) / np.exp(s - m).sum(axis=2, keepdims=True)"),
    "window_off_by_one": ("(J > I - window_blocks)", "(J >= I - window_blocks)"),
    "sink_off_by_one": ("(J < sink_blocks)", "(J <= sink_blocks)"),
    "token_mask_strict": ("keys[None, :] <= qpos[:, None]", "keys[None, :] < qpos[:, None]"),
    "token_mask_dropped": ("logits = np.where(allowed, logits, -np.inf)", "pass"),
    "lse_drops_max": ("lse = (m + np.log(", "lse = (0 * m + np.log("),
    "attn_kv_head_modulo": ("kt = _f64(k[L[\"start\"] + keys, h // g, :])",
                            "kt = _f64(k[L[\"start\"] + keys, h % hkv, :])"),
    "v_from_k": ("vt = _f64(v[", "vt = _f64(k["),
    "csr_row_order_seq_major": ("    for h in range(hq):\n        for kp in keeps:",
                                "    for kp in keeps:\n        for h in range(hq):"),
    "attn_scale_dropped": ("logits = sc * (qt @ kt.T)", "logits = (qt @ kt.T)"),
    "no_renormalise": ("o = (e @ vt) / np.where(ssum > 0, ssum, 1.0)", "o = (e @ vt)"),
    "near_band_x10": ("NEAR_REL = 1e-3", "NEAR_REL = 1e-2"),
    "near_band_on_score_difference": ("(np.abs(ratio - alpha) <= NEAR_REL * alpha)",
                                      "(np.abs((s - m) - alpha) <= NEAR_REL * alpha)"),
    "near_band_includes_forced": ("near = causal & ~forced & (", "near = causal & ("),
    "tri_pack_upper_triangle": ("parts.append(s[:, idx[0], idx[1]])",
                                "parts.append(s[:, idx[1], idx[0]])"),
    "tri_pack_column_major": ("idx = np.tril_indices(nb)", "idx = np.triu_indices(nb)[::-1]"),
}


def mutated(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType(f"oracle_mut_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    mod = mutated(name)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"
