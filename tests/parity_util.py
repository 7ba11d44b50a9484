"""Row-wise parity metric shared by the GPU tests.

e_i = max_n |g_in - o_in| / max_n |o_in|, where g is the GPU row and o the oracle row (fp64).

A row passes when e_i is within its allowance:
  * ReLU rows, and any row whose condition number is not finite (a zero denominator), are held
    to the plain tolerance: tol = 2e-2 for bf16 inputs, 1e-4 for fp32 inputs.
  * Trig rows are held to max(tol, u * cond_i / HEADROOM). cond_i is the row's first-order
    relative condition number under relative perturbation of every feature product
    (oracle.row_condition), u the unit roundoff of the 16-bit operands (2^-8 for bf16, counting
    the rounding of both factors of a product) or of fp32 (2^-24 times 16 for the angle and
    accumulation roundings). u * cond_i bounds what any evaluation of the formula in that
    precision can reach to first order; the kernels are required to stay within 1/HEADROOM of
    it. The trig estimator cancels across features and keys, so at L = 4096 almost every trig row
    has u * cond_i above tol: those rows are counted as "cond branch" rows and reported.
On top of the per-row test, the median of e_i over the checked rows must stay below tol / 2. A
kernel whose rounding behaves like the arithmetic it claims leaves the median near the output
rounding (about 2e-3 for bf16); systematic mistakes (a wrong weight on a block of keys, a shifted
value row, a swapped cos/sin group) move most rows at once and fail it even where the condition
numbers are large. tests/test_parity_metric.py plants such mistakes in oracle output and checks
that this function rejects every one of them.
"""
import numpy as np

TOL_BF16, U_BF16 = 2e-2, 2.0 ** -8
TOL_F32, U_F32 = 1e-4, 16 * 2.0 ** -24
HEADROOM = 2.0            # trig rows: the kernels stay within half of the first-order bound
MEDIAN_FRACTION = 0.5     # the median row error stays below tol * MEDIAN_FRACTION


def row_errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref).max(axis=-1)
    nrm = np.abs(ref).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(nrm > 0, err / nrm, err)


def allowances(cond, tol, u, trig, headroom=HEADROOM):
    """Per-row allowance: plain tol for ReLU rows and rows with a non-finite condition number,
    max(tol, u * cond / headroom) for trig rows."""
    cond = np.asarray(cond, dtype=np.float64)
    if not trig:
        return np.full(cond.shape, tol)
    finite = np.isfinite(cond)
    return np.where(finite, np.maximum(tol, u * np.where(finite, cond, 0.0) / headroom), tol)


def check_rows(got, ref, cond, tol, u, label="", trig=True, headroom=HEADROOM):
    """Assert the per-row and median parity conditions; return the statistics.

    got, ref: [..., rows, d]; cond: [..., rows] (oracle.row_condition of the same rows).
    trig: whether the rows come from the trig map (ReLU rows take the plain tolerance).
    """
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{label}: non-finite GPU output"
    rel = row_errors(got, ref)
    cond = np.asarray(cond, dtype=np.float64)
    allowed = allowances(cond, tol, u, trig, headroom)
    bad = rel > allowed
    finite = np.isfinite(cond)
    stats = {
        "rows": int(rel.size),
        "max_rel": float(rel.max()),
        "p99_rel": float(np.percentile(rel, 99)),
        "median_rel": float(np.median(rel)),
        "rows_cond_branch": int(np.sum(allowed > tol)),
        "rows_nonfinite_cond": int(np.sum(~finite)),
        "max_rel_plain_rows": float(rel[allowed <= tol].max()) if np.any(allowed <= tol) else 0.0,
        "max_cond": float(np.max(cond[finite])) if np.any(finite) else float("inf"),
        "max_rel_over_allowed": float(np.max(rel / allowed)),
        "bad": int(bad.sum()),
    }
    assert stats["bad"] == 0, f"{label}: {stats}"
    assert stats["median_rel"] <= tol * MEDIAN_FRACTION, f"{label}: median row error too large {stats}"
    return stats


def check_grads(got, ref, mags, cond, tol, u, label=""):
    """Backward metric for one head.

    got and ref are (dq, dk, dv) [L, d]. mags are the oracle's rounding scales
    (backward_magnitudes_head): each element's sum of absolute products. cond [L] holds the
    forward row condition numbers. Row r of each gradient passes if
        max_t |g - o|  <=  tol max_t |o_r|  +  u (max_t mag_r + c_r max_t |o_r|)
    - c_r = cond_r for dq, and the head's worst cond for dk and dv, since every query row feeds
      them.
    - The magnitude term bounds the rounding of the gradient's own sums. A row that cancels to
      zero (row 0 of a causal head) keeps that allowance and nothing more.
    - The cond term carries the rounding of the denominator the gradient divides by.
    """
    cond = np.nan_to_num(np.asarray(cond, dtype=np.float64), nan=np.inf, posinf=np.inf)
    worst = float(np.max(cond[np.isfinite(cond)])) if np.any(np.isfinite(cond)) else np.inf
    stats = {}
    for name, g, o, m, c in (("dq", got[0], ref[0], mags[0], cond), ("dk", got[1], ref[1], mags[1], worst),
                             ("dv", got[2], ref[2], mags[2], worst)):
        g, o, m = (np.asarray(x, dtype=np.float64) for x in (g, o, m))
        assert np.all(np.isfinite(g)), f"{label}: non-finite {name}"
        err = np.abs(g - o).max(axis=1)
        on = np.abs(o).max(axis=1)
        allowed = tol * on + u * (m.max(axis=1) + c * on)
        ratio = np.where(allowed > 0, err / np.where(allowed > 0, allowed, 1.0), np.where(err > 0, np.inf, 0.0))
        r = int(np.argmax(ratio))
        stats[name] = {"max_over_allowed": float(ratio[r]), "row": r,
                       "rel_at_row": float(err[r] / on[r]) if on[r] > 0 else float(err[r])}
        assert np.all(ratio <= 1.0), f"{label}: {name} {stats}"
    return stats
