"""Writes tests/golden/oracle_tiny.json from the oracle alone.

The source pages print no worked numeric example of routing, re-selection
or the expert FFN, so the stored values here are the oracle's, recorded once
so that any later change to the oracle's arithmetic shows up as a diff.
Inputs: the tiny layer (d=256, E=16, k=4, d_ff=128, bias N(0, 0.5)),
seeds 0..2, B=4; rules NONE, OEA k0=2, XShare budgets 4/6/8, Lynx
affinity binning, hierarchical XShare (2 tokens per request, budgets 4/6).
For the output y only the first 16 columns of each row and the norm are
kept.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import moe_synth as ms  # noqa: E402
import oracle  # noqa: E402

CASES = [("none", 0, 0, 0, 1), ("oea", 1, 2, 0, 1), ("xshare4", 2, 0, 4, 1),
         ("xshare6", 2, 0, 6, 1), ("xshare8", 2, 0, 8, 1), ("affinity", 3, 0, 0, 1),
         ("xshare_hier4", 4, 0, 4, 2), ("xshare_hier6", 4, 0, 6, 2)]


def _bits(a):
    return [int(v) for v in np.ascontiguousarray(a, np.float32).view(np.uint32).ravel()]


def main():
    S = ms.SHAPES["tiny"]
    out = {"shape": "tiny", "B": 4, "cases": []}
    for seed in range(3):
        L = ms.make_weights(S, seed)
        x = ms.make_tokens(S, 4, seed)
        for name, mode, k0, budget, group in CASES:
            r = oracle.layer(x, L, S.k, mode, k0=k0, budget=budget, group=group)
            out["cases"].append({
                "seed": seed, "rule": name, "mode": mode, "k0": k0, "budget": budget, "group": group,
                "logits_bits": _bits(r["logits"]), "probs_bits": _bits(r["probs"]),
                "sel_idx": r["sel_idx"].ravel().tolist(), "sel_w_bits": _bits(r["sel_w"]),
                "n_active": r["lists"]["n_active"],
                "y_head": [float(v) for v in r["y"][:, :16].ravel()],
                "y_norm": float(np.linalg.norm(r["y"])),
            })
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(out, f, separators=(",", ":"))


if __name__ == "__main__":
    main()
