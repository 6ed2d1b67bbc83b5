"""Write tests/golden/oracle_small.json from the CPU oracle alone.

The pages print no worked example for PISA, so this fixture is a regression
record of the oracle on a small seeded case (causal GQA, ragged block count),
not an independent pin: it makes any later change to the oracle's arithmetic
visible. Run from the repository root: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

CASE = dict(batch=1, heads_q=4, heads_kv=2, seq=37 * 16, head_dim=32, block=16, factor=4, topk=5, causal=1, seed=4242)


def compute():
    c = CASE
    w = workloads.Workload("golden", c["batch"], c["heads_q"], c["heads_kv"], c["seq"], c["seq"], c["head_dim"],
                           c["block"], c["factor"], c["topk"], c["causal"], "iid", c["seed"])
    q, k, v = workloads.qkv_f32(w)
    res = oracle.forward(q, k, v, w.block, w.factor, w.topk, True)
    return {
        "case": c,
        "idx": res["idx"].tolist(),
        "o_row_sums": [float(x) for x in res["O"].astype(np.float64).sum(axis=-1).reshape(-1)[::7]],
        "lse": [float(x) for x in res["lse"].reshape(-1)[::7]],
        "pyramid_top": res["pyramid"][0][1][-1].astype(np.float64).tolist(),
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=None, separators=(",", ":"))
    print("wrote", out)
