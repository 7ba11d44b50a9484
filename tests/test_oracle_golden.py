"""The oracle still reproduces its committed regression fixture (tests/golden)."""
import json
import os

import numpy as np

import favor_inputs as fi
from oracle import favor_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_regression_fixture():
    with open(os.path.join(HERE, "golden", "config1_rows.json")) as f:
        g = json.load(f)
    q, k, v = fi.qkv(1, 1, 256, 16, seed=g["seed"])
    G, R = fi.orf_gaussians(1, g["M"], 16, seed=g["seed"])
    om = O.orf_matrices(G, R, g["M"]).astype(np.float32).astype(np.float64)
    Q, K, V = (x.astype(np.float64) for x in (q, k, v))
    for name, rows in g["cases"].items():
        kind = O.TRIG if name.startswith("trig") else O.RELU
        o = O.favor_attention(Q, K, V, om, kind, name.endswith("causal"))[0, 0]
        np.testing.assert_allclose(o[g["rows"]], np.array(rows), rtol=1e-12, atol=1e-14)
