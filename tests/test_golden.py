"""The oracle still reproduces the values recorded in tests/golden by
tests/golden/make_golden.py (which calls only the oracle): a guard against
silent drift of the oracle's arithmetic."""
import json
import os

import numpy as np

import moe_synth as ms

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_recorded_tiny_cases(oracle_lib):
    with open(os.path.join(HERE, "golden", "oracle_tiny.json")) as f:
        g = json.load(f)
    S = ms.SHAPES[g["shape"]]
    layers = {}
    for c in g["cases"]:
        seed = c["seed"]
        if seed not in layers:
            layers[seed] = (ms.make_weights(S, seed), ms.make_tokens(S, g["B"], seed))
        L, x = layers[seed]
        r = oracle_lib.layer(x, L, S.k, c["mode"], k0=c["k0"], budget=c["budget"], group=c.get("group", 1))
        assert r["logits"].view(np.uint32).ravel().tolist() == c["logits_bits"]
        assert r["probs"].view(np.uint32).ravel().tolist() == c["probs_bits"]
        assert r["sel_idx"].ravel().tolist() == c["sel_idx"]
        assert r["sel_w"].view(np.uint32).ravel().tolist() == c["sel_w_bits"]
        assert r["lists"]["n_active"] == c["n_active"]
        assert np.allclose(r["y"][:, :16].ravel(), np.array(c["y_head"]), rtol=1e-12, atol=1e-15)
        assert abs(np.linalg.norm(r["y"]) - c["y_norm"]) <= 1e-12 * c["y_norm"]
