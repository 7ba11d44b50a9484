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
Given the condition of the denominator alone as well (kappa_i = D_i/|den_i|, oracle
row_condition_head(..., with_den=True)), trig rows use the bound that holds to every order,
u * cond_i / (1 - u kappa_i), and rows with u * kappa_i >= 1 are "undetermined": rounding of the
16-bit operands can cancel their denominator, so no evaluation in that precision fixes even the
sign of the row (the trig mode's occasional numerical instability, which the explainer sets
against the stable non-negative mode). They are exempt from the per-row bound, counted, must be
finite, and stay in the median.
On top of the per-row test, the median of e_i over the checked rows must stay below tol / 2. A
kernel whose rounding behaves like the arithmetic it claims leaves the median near the output
rounding (about 2e-3 for bf16); systematic mistakes (a wrong weight on a block of keys, a shifted
value row, a swapped cos/sin group) move most rows at once and fail it even where the condition
numbers are large. tests/test_parity_metric.py plants such mistakes in oracle output and checks
that this function rejects every one of them.
"""
from collections import namedtuple

import numpy as np

# cond: oracle.row_condition_head of the rows; kden: the denominator's condition D_i/|den_i|;
# terms: oracle.row_rounding_terms_head of the rows (trig rows only; None otherwise)
class RowCond(namedtuple("RowCond", "cond kden terms", defaults=(None,))):
    def reshape(self, *shape):
        """The same rows under a new leading shape (row arrays take `shape`, row x column
        arrays `shape` plus their last axis)."""
        rs = lambda a: np.asarray(a).reshape(*shape) if np.ndim(a) == np.ndim(self.cond) else \
            np.asarray(a).reshape(*shape, np.shape(a)[-1])
        tm = None if self.terms is None else {key: rs(x) for key, x in self.terms.items()}
        return RowCond(rs(self.cond), rs(self.kden), tm)

# Unit roundoffs of a path's operand types at the three rounding levels of
# oracle.row_rounding_terms_head, and the number of standard deviations a row may reach.
#   bf16 bidirectional trig: key features and w o V in bf16 (level 1, level 2); the state image
#     and the query features in fp16 (two roundings at level 3).
#   bf16 causal trig: key features in bf16 (level 1); masked intra products and weighted values
#     in bf16 (level 2); query features, the state image and the deposited partial numerators in
#     bf16 (three roundings at level 3).
Levels = namedtuple("Levels", "u1 u2 u3 z")
Z_SIGMA = 6.0
U_BIDIR16 = Levels(2.0 ** -8, 2.0 ** -8, np.sqrt(2.0) * 2.0 ** -11, Z_SIGMA)
U_CAUSAL16 = Levels(2.0 ** -8, 2.0 ** -8, np.sqrt(3.0) * 2.0 ** -8, Z_SIGMA)
U_OUT16 = 2.0 ** -8       # rounding of the output itself to bf16

TOL_BF16, U_BF16 = 2e-2, 2.0 ** -8
TOL_F32, U_F32 = 1e-4, 16 * 2.0 ** -24
HEADROOM = 2.0            # trig rows: the kernels stay within half of the first-order bound
MEDIAN_FRACTION = 0.5     # the median row error stays below tol * MEDIAN_FRACTION
UNDETERMINED_SHARE = 0.10  # at most this share of the checked rows may be exempt as undetermined


def row_errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref).max(axis=-1)
    nrm = np.abs(ref).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(nrm > 0, err / nrm, err)


def allowances(cond, tol, u, trig, headroom=HEADROOM):
    """Per-row allowance: plain tol for ReLU rows and rows with a non-finite condition number,
    max(tol, u * cond / headroom) for trig rows. With cond a RowCond, trig rows take
    max(tol, u * cond / ((1 - u kappa) headroom)) and undetermined rows (u kappa >= 1) +inf."""
    kden = None
    if isinstance(cond, RowCond):
        cond, kden = cond.cond, cond.kden
    cond = np.asarray(cond, dtype=np.float64)
    if not trig:
        return np.full(cond.shape, tol)
    finite = np.isfinite(cond)
    c = np.where(finite, cond, 0.0)
    if kden is not None:
        r = np.asarray(kden, dtype=np.float64) * u
        with np.errstate(divide="ignore", invalid="ignore"):
            c = np.where(r < 1.0, c / (1.0 - r), np.inf)
        c = np.where(finite, c, 0.0)
    return np.where(finite, np.maximum(tol, u * c / headroom), tol)


def stat_allowances(terms, tol, lv, u_out=U_OUT16):
    """Per-row allowance from the rounding-level sums of squares: a relative error with
    variance u^2/3 per operand (uniform rounding) gives sd_num_n and sd_den; a row may reach
    z (sd_num_n + |out_n| sd_den) / |den| / max|out|, widened by 1/(1 - z sd_den/|den|), plus
    the output's own rounding. Rows with z sd_den >= |den|/2 are undetermined (+inf)."""
    def sd(a, b, c):
        return np.sqrt((lv.u1 ** 2 * a + lv.u2 ** 2 * b + lv.u3 ** 2 * c) / 3.0)
    sn = sd(terms["N1"], terms["N2"], terms["N3"])
    sdd = sd(terms["D1"], terms["D2"], terms["D3"])
    out, den = np.asarray(terms["out"]), np.abs(np.asarray(terms["den"]))
    on = np.abs(out).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = (sn + np.abs(out) * sdd[..., None]).max(axis=-1) / (den * on)
        rd = lv.z * sdd / den
        a = np.maximum(tol, lv.z * rel / (1.0 - rd) + u_out)
    a = np.where(np.isfinite(a), a, tol)          # zero rows: plain tolerance
    return np.where((rd < 0.5) | (den == 0), a, np.inf)


def check_rows(got, ref, cond, tol, u, label="", trig=True, headroom=HEADROOM):
    """Assert the per-row and median parity conditions; return the statistics.

    got, ref: [..., rows, d]; cond: [..., rows] (oracle.row_condition of the same rows), or a
    RowCond that adds the denominator's condition.
    trig: whether the rows come from the trig map (ReLU rows take the plain tolerance).
    """
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{label}: non-finite GPU output"
    rel = row_errors(got, ref)
    if isinstance(u, Levels) and trig:
        assert isinstance(cond, RowCond) and cond.terms is not None, f"{label}: no rounding terms"
        allowed = stat_allowances(cond.terms, tol, u)
    else:
        allowed = allowances(cond, tol, u.u1 if isinstance(u, Levels) else u, trig, headroom)
    if isinstance(cond, RowCond):
        cond = cond.cond
    cond = np.asarray(cond, dtype=np.float64)
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
        "rows_undetermined": int(np.sum(np.isinf(allowed))),
        "max_rel_over_allowed": float(np.max(rel / allowed)),
        "bad": int(bad.sum()),
    }
    assert stats["bad"] == 0, f"{label}: {stats}"
    assert stats["median_rel"] <= tol * MEDIAN_FRACTION, f"{label}: median row error too large {stats}"
    # the exempt rows stay a small share (2-6% of the trig rows of every configuration tested);
    # a larger share would mean the metric itself had drifted
    assert stats["rows_undetermined"] <= max(2, UNDETERMINED_SHARE * stats["rows"]), \
        f"{label}: too many undetermined rows {stats}"
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
