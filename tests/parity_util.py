"""Row-wise parity metric shared by the GPU tests.

e_i = max_n |g_in - o_in| / max_n |o_in|, where g is the GPU row and o the oracle row (fp64).
A row passes if e_i <= max(tol, u * cond_i). tol is the stated tolerance (2e-2 for bf16 inputs,
1e-4 for fp32 inputs). u is the unit roundoff of the arithmetic's 16-bit operands (2^-8 for
bf16) or of fp32 (2^-24, times 16 for the angle and accumulation roundings). cond_i is the
row's relative condition number under relative perturbation of the feature products
(oracle.row_condition). For well-conditioned rows (every ReLU row, most trig rows at small
norms) u * cond_i < tol and the bound is the plain tolerance. Rows where u * cond_i > tol
are trig rows whose sums over features cancel heavily. No finite-precision evaluation of the
same formula can hold them to tol. They are counted and reported, never skipped.
"""
import numpy as np

TOL_BF16, U_BF16 = 2e-2, 2.0 ** -8
TOL_F32, U_F32 = 1e-4, 16 * 2.0 ** -24


def row_errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref).max(axis=-1)
    nrm = np.abs(ref).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(nrm > 0, err / nrm, err)


def check_rows(got, ref, cond, tol, u, label=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{label}: non-finite GPU output"
    rel = row_errors(got, ref)
    cond = np.nan_to_num(np.asarray(cond, dtype=np.float64), nan=np.inf)
    allowed = np.maximum(tol, u * cond)
    bad = rel > allowed
    stats = {
        "rows": int(rel.size),
        "max_rel": float(rel.max()),
        "p99_rel": float(np.percentile(rel, 99)),
        "rows_cond_branch": int(np.sum(u * cond > tol)),
        "max_cond": float(np.max(cond[np.isfinite(cond)])) if np.any(np.isfinite(cond)) else float("inf"),
        "max_rel_over_allowed": float(np.max(rel / allowed)),
        "bad": int(bad.sum()),
    }
    assert stats["bad"] == 0, f"{label}: {stats}"
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
