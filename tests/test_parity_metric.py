"""Power of the parity metric: kernel-shaped mistakes planted in oracle output must be rejected.

One head of the bench workload (L = 4096, d = 64, M = 256, bf16 inputs, seed 0). The oracle's
exact output, rounded to bf16 like a kernel's output, must pass tests/parity_util.check_rows; each
planted mistake, computed on the CPU from the oracle's own feature maps and rounded the same way,
must fail it. The mistakes are the ones a tensor-core kernel can plausibly make:
  * a strict causal mask (keys j < i instead of j <= i);
  * one 128-key chunk over-weighted by e^0.5 (a stabiliser reference applied to the wrong chunk);
  * the ragged tail tile dropped (L = 4000: the last 32 keys never reach the state);
  * V shifted by one row;
  * cos and sin exchanged for one group of 16 angles (trig).
"""
import numpy as np
import pytest
import torch

import favor_inputs as fi
from oracle import favor_oracle as O
from parity_util import TOL_BF16, U_BF16, U_BIDIR16, U_CAUSAL16, RowCond, check_rows


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _head(L, d=64, M=256, seed=0):
    q, k, v = fi.qkv(1, 1, L, d, seed=seed)
    G, R = fi.orf_gaussians(1, M, d, seed=seed)
    om = O.orf_matrices(G, R, M).astype(np.float32)
    q, k, v = (fi.as_f64(fi.round_to(x, "bf16"))[0, 0] for x in (q, k, v))
    return q, k, v, fi.as_f64(fi.round_to(om, "bf16"))[0]


def _cond(q, k, v, om, kind, causal):
    """The RowCond the GPU tests pass, for one head, with a leading head axis."""
    c, kd = O.row_condition_head(q, k, v, om, kind, causal, with_den=True)
    t = O.row_rounding_terms_head(q, k, v, om, kind, causal)
    return RowCond(c[None], kd[None], {key: val[None] for key, val in t.items()})


def _u(causal):
    return U_CAUSAL16 if causal else U_BIDIR16


def _quadratic(fq, fk, v, causal, strict=False):
    A = fq @ fk.T
    if causal:
        A = np.tril(A, -1 if strict else 0)
    return O._normalise(A @ v, A.sum(axis=1))


def _planted(kind, causal):
    """(name, bf16 output) for every planted mistake that applies, plus the oracle row
    reference, its condition numbers and the exact output."""
    L, M = 4096, 256
    q, k, v, om = _head(L)
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    ref = O.favor_causal_head(q, k, v, om, kind) if causal else O.favor_bidirectional_head(q, k, v, om, kind)
    cond = _cond(q, k, v, om, kind, causal)
    bad = []
    if causal:
        bad.append(("strict mask", _quadratic(fq, fk, v, True, strict=True)))
    fk2 = fk.copy()
    fk2[1024:1152] *= np.exp(0.5)
    bad.append(("chunk over-weighted", _quadratic(fq, fk2, v, causal)))
    bad.append(("value rows shifted", _quadratic(fq, fk, np.concatenate([v[1:], v[-1:]]), causal)))
    if kind == O.TRIG:
        fk3 = fk.copy()
        fk3[:, 16:32], fk3[:, M + 16:M + 32] = fk[:, M + 16:M + 32], fk[:, 16:32]
        bad.append(("cos/sin exchanged", _quadratic(fq, fk3, v, causal)))
    return ref, cond, [(n, _bf16(o)) for n, o in bad]


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_planted_kernel_mistakes_are_rejected(kind, causal):
    ref, cond, bad = _planted(kind, causal)
    trig = kind == O.TRIG
    check_rows(_bf16(ref)[None], ref[None], cond, TOL_BF16, _u(causal), "exact, rounded", trig=trig)
    for name, got in bad:
        with pytest.raises(AssertionError):
            check_rows(got[None], ref[None], cond, TOL_BF16, _u(causal), name, trig=trig)


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
def test_dropped_tail_tile_is_rejected(kind):
    # L = 4000: 31 full 128-token tiles and a ragged tail of 32 tokens. A kernel that drops the
    # tail tile leaves those keys out of the state. Bidirectional rows all move; causal rows
    # move from the tail on, and the ReLU map's plain tolerance catches them.
    L = 4000
    q, k, v, om = _head(L)
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    fk_drop = fk.copy()
    fk_drop[31 * 128:] = 0.0
    for causal in ((False, True) if kind == O.RELU else (False,)):
        ref = _quadratic(fq, fk, v, causal)
        cond = _cond(q, k, v, om, kind, causal)
        with pytest.raises(AssertionError):
            check_rows(_bf16(_quadratic(fq, fk_drop, v, causal))[None], ref[None], cond, TOL_BF16, _u(causal),
                       "tail dropped", trig=kind == O.TRIG)


def test_nonfinite_condition_takes_the_plain_tolerance():
    # a zero denominator (q = 0 under the ReLU map) has no finite condition number: the row is
    # held to the plain tolerance, not waved through
    ref = np.zeros((1, 3, 4))
    cond = np.array([[np.nan, np.inf, 5.0]])
    got = ref.copy()
    check_rows(got, ref, cond, TOL_BF16, U_BF16, "zeros", trig=True)
    got[0, 0, 0] = 1.0
    with pytest.raises(AssertionError):
        check_rows(got, ref, cond, TOL_BF16, U_BF16, "nan cond", trig=True)


def test_undetermined_rows_are_exempt_but_counted():
    # u kappa = 0.5 and 0.99 take u cond / (headroom (1 - u kappa)); u kappa >= 1 is exempt from
    # the per-row bound (counted) but not from the finiteness and median checks
    u, cond = U_BF16, 1000.0
    kden = np.array([[0.5, 0.99, 1.0, 3.0] + [1.0] * 5 + [0.0] * 90]) / u
    rc = RowCond(np.full(kden.shape, cond), kden)
    ref = np.ones((1, 99, 4))
    got = ref.copy()
    got[0, 0] += u * cond / 2 / 0.5 * 0.99       # just inside row 0's allowance
    got[0, 3] += 1e6                               # undetermined: exempt
    st = check_rows(got, ref, rc, TOL_BF16, u, "exempt", trig=True)
    assert st["rows_undetermined"] == 7
    bad = got.copy()
    bad[0, 0] = ref[0, 0] + u * cond / 2 / 0.5 * 1.01
    with pytest.raises(AssertionError):
        check_rows(bad, ref, rc, TOL_BF16, u, "row 0 over", trig=True)
    bad = got.copy()
    bad[0, 5:] += 1.0                               # most rows off: the median check fails
    with pytest.raises(AssertionError):
        check_rows(bad, ref, rc, TOL_BF16, u, "median", trig=True)
    # more than the allowed share of exempt rows fails on its own
    many = RowCond(rc.cond, np.where(np.arange(99) < 20, 2.0 / u, 0.0)[None])
    with pytest.raises(AssertionError):
        check_rows(got, ref, many, TOL_BF16, u, "share", trig=True)
    bad = got.copy()
    bad[0, 5:] += 1.0
    with pytest.raises(AssertionError):
        check_rows(bad, ref, rc, TOL_BF16, u, "median", trig=True)
    bad = got.copy()
    bad[0, 4, 0] = np.nan
    with pytest.raises(AssertionError):
        check_rows(bad, ref, rc, TOL_BF16, u, "nan", trig=True)
