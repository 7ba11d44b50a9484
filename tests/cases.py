"""Seeded parity cases: the same rounded inputs for the CUDA path (device tensors) and the
oracle (fp64 arrays). Omega comes from the oracle's ORF builder, rounded to the run dtype.
Nothing here reads a value produced by the CUDA path."""
import numpy as np

import favor_inputs as fi
from oracle import favor_oracle as O
from parity_util import RowCond


class Case:
    def __init__(self, B, H, L, d, M, dtype="bf16", seed=0, heavy=0.0):
        import torch
        self.B, self.H, self.L, self.d, self.M, self.dtype = B, H, L, d, M, dtype
        q, k, v = fi.qkv(B, H, L, d, seed=seed, heavy_frac=heavy)
        G, R = fi.orf_gaussians(H, M, d, seed=seed)
        om = O.orf_matrices(G, R, M).astype(np.float32)
        self.t = [fi.round_to(x, dtype) for x in (q, k, v, om)]   # CPU torch tensors
        self.q, self.k, self.v, self.om = (fi.as_f64(t) for t in self.t)
        self._dev = None

    def device(self):
        if self._dev is None:
            self._dev = [t.to("cuda") for t in self.t]
        return self._dev

    def oracle(self, kind, causal, heads=None, rows=None):
        """Oracle rows [n_heads, n_rows, d] and a RowCond of their condition numbers [n_heads, n_rows]."""
        heads = [(b, h) for b in range(self.B) for h in range(self.H)] if heads is None else heads
        outs, conds, terms = [], [], []
        for b, h in heads:
            a = (self.q[b, h], self.k[b, h], self.v[b, h], self.om[h])
            r = np.arange(self.L) if rows is None else np.asarray(rows)
            if rows is None and not causal:
                o = O.favor_bidirectional_head(*a, kind)
            elif rows is None:
                o = O.favor_causal_head(*a, kind)
            else:
                o = O.favor_rows_head(*a, kind, causal, r)
            outs.append(o)
            conds.append(O.row_condition_head(*a, kind, causal, r, with_den=True))
            if kind == O.TRIG:
                terms.append(O.row_rounding_terms_head(*a, kind, causal, r))
        tm = {key: np.stack([t[key] for t in terms]) for key in terms[0]} if terms else None
        return (np.stack(outs), RowCond(np.stack([c for c, _ in conds]), np.stack([k for _, k in conds]), tm),
                heads)
