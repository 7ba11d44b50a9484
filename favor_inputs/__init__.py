"""Seeded synthetic inputs for FAVOR attention.

Both the CUDA path and the CPU oracle take their inputs from this module. It only draws
random numbers and rounds them to the run dtype. It computes none of the method: no
orthogonalisation, no norms, no features, no attention. The Gaussian arrays an ORF
random matrix is built from are drawn here, and each side builds the matrix itself.

Recipe:
  * Q, K, V ~ N(0, 1) * d**-0.25, drawn as float32 from numpy's PCG64
    (``default_rng``), then rounded to the run dtype with round-to-nearest-even.
    The d**-0.25 pre-scale of both Q and K carries the 1/sqrt(d) temperature of
    exp(QK^T/sqrt(d)).
  * Optional heavy-norm stress: for each (b, h), Q and K independently get
    floor(frac * L) rows, chosen by seeded sampling without replacement, scaled by
    ``heavy_scale``. V is left alone.
  * ORF Gaussians for head h: one generator seeded ``seed*1000003 + 7919*h + 1``
    draws ceil(M/d) blocks G[h, i] of d x d i.i.d. N(0, 1), then R[h] of M x d
    i.i.d. N(0, 1). The norm of R[h, r] is the chi_d length of row r.
  * i.i.d. (unstructured) Omega: M x d i.i.d. N(0, 1) rows per head.
The workloads take protein-MLM shapes (L = 1024 ... 65536, d = 64, M = 128/256) and
stand in for the UniRef/Pfam data that FAVOR was evaluated on.
"""
from __future__ import annotations

import math

import numpy as np

_SALT = 1000003


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(seed * _SALT + stream)


def qkv(B: int, H: int, L: int, d: int, seed: int = 0,
        heavy_frac: float = 0.0, heavy_scale: float = 4.0):
    """Return float32 arrays Q, K, V of shape [B, H, L, d] (not yet rounded)."""
    scale = np.float32(d ** -0.25)
    out = []
    for stream in (11, 13, 17):
        x = _rng(seed, stream).standard_normal((B, H, L, d), dtype=np.float32)
        x *= scale
        out.append(x)
    q, k, v = out
    n_heavy = int(math.floor(heavy_frac * L))
    if n_heavy > 0:
        for x, stream in ((q, 19), (k, 23)):
            g = _rng(seed, stream)
            for b in range(B):
                for h in range(H):
                    rows = g.choice(L, size=n_heavy, replace=False)
                    x[b, h, rows, :] *= np.float32(heavy_scale)
    return q, k, v


def orf_gaussians(H: int, M: int, d: int, seed: int = 0):
    """Gaussian draws for ORF matrices.

    Returns (G, R): G float64 [H, ceil(M/d), d, d], R float64 [H, M, d].
    """
    nb = -(-M // d)
    G = np.empty((H, nb, d, d), dtype=np.float64)
    R = np.empty((H, M, d), dtype=np.float64)
    for h in range(H):
        g = np.random.default_rng(seed * _SALT + 7919 * h + 1)
        G[h] = g.standard_normal((nb, d, d))
        R[h] = g.standard_normal((M, d))
    return G, R


def iid_gaussians(H: int, M: int, d: int, seed: int = 0):
    """Unstructured Omega draws: float64 [H, M, d] of i.i.d. N(0, 1)."""
    W = np.empty((H, M, d), dtype=np.float64)
    for h in range(H):
        W[h] = np.random.default_rng(seed * _SALT + 7919 * h + 2).standard_normal((M, d))
    return W


def sample_rows(L: int, n: int, seed: int = 0):
    """Sorted row indices: 0, 1, L-1 plus seeded uniform picks, n in total (at most L)."""
    n = min(n, L)
    fixed = sorted({0, min(1, L - 1), L - 1})
    rest = np.setdiff1d(np.arange(L), fixed)
    k = max(0, n - len(fixed))
    picks = _rng(seed, 29).choice(rest, size=min(k, rest.size), replace=False) if k else []
    return np.sort(np.concatenate([np.array(fixed, dtype=np.int64),
                                   np.asarray(picks, dtype=np.int64)]))


def round_to(x: np.ndarray, dtype: str):
    """Round an array to the run dtype ('bf16' or 'f32'). Returns a CPU torch tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t.clone()
    raise ValueError(dtype)


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a (CPU or device) torch tensor, for the oracle."""
    return t.detach().to("cpu").to(dtype=__import__("torch").float64).numpy()
