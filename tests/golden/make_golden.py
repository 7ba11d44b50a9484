"""Write config1_rows.json from the oracle alone (no CUDA path involved)."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import favor_inputs as fi  # noqa: E402
from oracle import favor_oracle as O  # noqa: E402

ROWS = [0, 1, 2, 17, 100, 128, 200, 254, 255]


def build():
    q, k, v = fi.qkv(1, 1, 256, 16, seed=0)
    G, R = fi.orf_gaussians(1, 32, 16, seed=0)
    om32 = O.orf_matrices(G, R, 32).astype(np.float32).astype(np.float64)
    Q, K, V = (x.astype(np.float64) for x in (q, k, v))
    out = {"shape": [1, 1, 256, 16], "M": 32, "seed": 0, "rows": ROWS, "cases": {}}
    for kind, kname in ((O.TRIG, "trig"), (O.RELU, "relu")):
        for causal in (False, True):
            o = O.favor_attention(Q, K, V, om32, kind, causal)[0, 0]
            out["cases"][f"{kname}_{'causal' if causal else 'bidir'}"] = o[ROWS].tolist()
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "config1_rows.json"), "w") as f:
        json.dump(build(), f, indent=1)
