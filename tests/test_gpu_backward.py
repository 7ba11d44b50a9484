"""fp32 backward (dq, dk, dv) vs the oracle's analytic gradients on the same fp32 inputs.

Metric (parity_util.check_grads), row by row:
    err <= tol |o| + u (mag + c |o|),   with tol = 1e-4 and u = 16 * 2^-24 (the fp32 path's unit)
- mag is the oracle's rounding scale of the row: its sum of absolute products
  (backward_magnitudes_head).
- c is the forward row condition number for dq, and the head's worst one for dk and dv.
- Gradients cancel even where outputs do not. dq_i sums a_ij (v_j - o_i) over keys, and row 0
  of a causal head is exactly zero. The magnitude term is the standard bound for that.
- A float32 run of the same chunked algorithm on the host stays below 5% of this allowance on
  every case here.
"""
import numpy as np
import pytest

import favor_inputs as fi
from cases import Case
from oracle import favor_oracle as O
from parity_util import check_grads

pytestmark = pytest.mark.gpu

TOL, U = 1e-4, 16 * 2.0 ** -24


def _dout(shape, seed):
    return fi.round_to(np.random.default_rng(seed).standard_normal(shape).astype(np.float32), "f32")


def _check(kind, causal, B, H, L, d, M, seed):
    import linear_kernelized_attention_b200 as F
    c = Case(B, H, L, d, M, dtype="f32", seed=seed)
    dO = _dout((B, H, L, d), seed + 1)
    q, k, v, om = c.device()
    got = F.favor_attention_backward_f32(q, k, v, om, dO.cuda(), feature_kind=kind, causal=causal)
    assert F.favor_sync_status() == 0
    dO = fi.as_f64(dO)
    got = [fi.as_f64(g) for g in got]
    worst = None
    for b in range(B):
        for h in range(H):
            a = (c.q[b, h], c.k[b, h], c.v[b, h], c.om[h])
            ref = O.favor_backward_head(*a, kind, causal, dO[b, h])
            cond = O.row_condition_head(*a, kind, causal)
            mags = O.backward_magnitudes_head(*a, kind, causal, dO[b, h])
            st = check_grads([g[b, h] for g in got], ref, mags, cond, TOL, U,
                             f"kind={kind} causal={causal} {B}x{H}x{L} d={d} M={M} head=({b},{h})")
            if worst is None or st["dq"]["max_over_allowed"] > worst["dq"]["max_over_allowed"]:
                worst = st
    print(kind, causal, worst)


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,L,d,M", [
    (1, 1, 1, 16, 32),      # one token
    (1, 1, 64, 16, 32),     # one full chunk
    (1, 2, 300, 64, 128),   # 5 chunks, ragged tail, 8 feature tiles
    (2, 2, 200, 32, 40),    # ragged feature tile (F = 80 trig / 40 ReLU)
])
def test_backward_matches_oracle(kind, causal, B, H, L, d, M):
    _check(kind, causal, B, H, L, d, M, seed=L + M + d)


def test_backward_bench_shape_sampled_heads():
    # B=1, H=4, L=1024, d=64, M=256: the bench's per-head shape, 16 chunks
    for kind in (0, 1):
        _check(kind, True, 1, 4, 1024, 64, 256, seed=5)


def test_backward_rejects_wide_heads():
    import torch
    import linear_kernelized_attention_b200 as F
    x = torch.zeros(1, 1, 8, 128, device="cuda")
    om = torch.zeros(1, 32, 128, device="cuda")
    with pytest.raises(F.FavorError) as e:
        F.favor_attention_backward_f32(x, x, x, om, x)
    assert e.value.code == -5
