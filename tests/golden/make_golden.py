"""Writes tests/golden/oracle_small.json: regression fixtures of the CPU oracle on small seeded
workloads.  Test infrastructure only: this script calls the seeded generator (gen/) and the
oracle (oracle/) and nothing else.

The pages print no worked example with values (no formula body, no listing, no table of
outputs), so no fixture here is the pages' own; these are the oracle's results on the seeded
inputs, stored so that any later change to the oracle's arithmetic shows up as a diff of this
file (and must then name the passage that justifies it).  They are not pins: the oracle's pins
are the checks in tests/oracle_pins.py and tests/test_oracle_*.py.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from gen import WORKLOADS, generate  # noqa: E402
from oracle import fpx_oracle as O  # noqa: E402

# (name, base workload, overrides, alpha, sink_blocks, window_blocks, sampled (h, t) rows)
CASES = [
    ("fp32_varlen_b16", "tiny_fp32_n2048",
     dict(seqlens=(70, 0, 33), hq=4, hkv=2, d=64, block=16, q_gain=60.0),
     0.3, 1, 1, [(0, 0), (1, 15), (2, 16), (3, 69), (0, 70), (3, 102), (1, 88)]),
    ("bf16_ragged_b128", "llama8b_bf16_n8192", dict(seqlens=(700,), hq=2, hkv=1, q_gain=300.0),
     0.2, 1, 1, [(0, 0), (1, 127), (0, 128), (1, 255), (0, 699), (1, 640), (0, 511)]),
    ("e4m3_sparse_b128", "llama8b_bf16_n8192",
     dict(seqlens=(520,), hq=2, hkv=1, dtype="e4m3", q_gain=400.0), 0.2, 0, 1,
     [(0, 5), (1, 130), (0, 300), (1, 519), (0, 400)]),
]


def oracle_inputs(data):
    import torch
    out = []
    for key, sc in (("q", "q_scale"), ("k", "k_scale"), ("v", "v_scale")):
        a = data[key].to(torch.float64)
        if data.get(sc) is not None:
            a = a * data[sc].to(torch.float64).view(1, -1, 1)
        out.append(a.numpy())
    return out


def case_record(name, base, over, alpha, sink, window, rows):
    w = WORKLOADS[base].with_(**over)
    data = generate(w)
    q, k, v = oracle_inputs(data)
    cu = data["cu_seqlens"]
    r = O.prefill(q, k, v, cu, w.block, alpha, sink, window, rows=rows)
    tri = O.triangular_pack(r["scores"])
    return {
        "name": name, "workload": base, "overrides": {k_: (list(v_) if isinstance(v_, tuple) else v_)
                                                      for k_, v_ in over.items()},
        "alpha": alpha, "sink_blocks": sink, "window_blocks": window,
        "cu_seqlens": [int(x) for x in cu],
        "scores": [float(x) for x in tri.reshape(-1)],
        "row_ptr": [int(x) for x in r["row_ptr"]],
        "col_idx": [int(x) for x in r["col_idx"]],
        "near": int(sum(int(n.sum()) for n in r["nears"])),
        "rows": [list(x) for x in rows],
        "o_rows": [[float(x) for x in row] for row in r["o"]],
        "lse_rows": [float(x) for x in r["lse"]],
    }


def main():
    out = {"what": "CPU-oracle results on small seeded workloads (regression fixtures; the pages "
                   "print no worked example)",
           "cases": [case_record(*c) for c in CASES]}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print(path, os.path.getsize(path), "bytes")


if __name__ == "__main__":
    main()
