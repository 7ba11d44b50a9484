"""Planted mistakes in the oracle must trip at least one pin.

Each case patches one oracle function (on the CPU, for the duration of the test) with a
plausible slip, then runs the pins that should catch it and expects an AssertionError.
"""
import numpy as np
import pytest

from oracle import favor_oracle as O
import test_oracle_pins as P


def _phi_trig_no_exp(X, Om):
    U = X @ Om.T
    return np.concatenate([np.cos(U), np.sin(U)], axis=1) / np.sqrt(Om.shape[0])


def _phi_trig_cos_twice(X, Om):
    U = X @ Om.T
    g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(Om.shape[0])
    return g[:, None] * np.concatenate([np.cos(U), np.cos(U)], axis=1)


def _phi_trig_sign_slip(X, Om):
    U = X @ Om.T
    g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(Om.shape[0])
    return g[:, None] * np.concatenate([np.cos(U), np.sin(-np.abs(U))], axis=1)


def _phi_relu_no_max(X, Om):
    return (X @ Om.T) / np.sqrt(Om.shape[0])


def _causal_strict(q, k, v, Om, kind):
    fq, fk = O.phi(q, Om, kind), O.phi(k, Om, kind)
    S = np.zeros((fk.shape[1], v.shape[1]))
    z = np.zeros(fk.shape[1])
    out = np.zeros_like(v)
    for i in range(q.shape[0]):
        den = fq[i] @ z
        if den != 0:
            out[i] = (fq[i] @ S) / den
        S += np.outer(fk[i], v[i])
        z += fk[i]
    return out


def _bidir_wrong_normaliser(q, k, v, Om, kind):
    fq, fk = O.phi(q, Om, kind), O.phi(k, Om, kind)
    return (fq @ (fk.T @ v)) / fq.sum(axis=1, keepdims=True)


def _gs_no_normalise(G):
    Q = np.array(G, dtype=np.float64, copy=True)
    for i in range(1, Q.shape[0]):
        Q[i] = Q[i] - Q[:i].T @ ((Q[:i] @ Q[i]) / np.sum(Q[:i] * Q[:i], axis=1))
    return Q


def _orf_no_chi(G, R, M):
    return np.concatenate([O.gram_schmidt_rows(G[i]) for i in range(G.shape[0])], axis=0)[:M]


def _softmax_mask_slip(q, k, v, causal, rows=None):
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    s = q[rows] @ k.T
    if causal:
        s = np.where(np.arange(k.shape[0])[None, :] < rows[:, None] + 2, s, -np.inf)
    a = np.exp(s - s.max(axis=1, keepdims=True))
    return (a @ v) / a.sum(axis=1, keepdims=True)


def _decode_read_before_add(S, z, q, k, v, Om, kind):
    fk = O.phi(k[None, :], Om, kind)[0]
    fq = O.phi(q[None, :], Om, kind)[0]
    den = fq @ z
    out = (fq @ S) / den if den != 0.0 else np.zeros(v.shape[0])
    S += np.outer(fk, v)
    z += fk
    return out


def _decode_value_for_key(S, z, q, k, v, Om, kind):
    fk = O.phi(k[None, :], Om, kind)[0]
    fq = O.phi(q[None, :], Om, kind)[0]
    S += np.outer(fk, k)
    z += fk
    return (fq @ S) / (fq @ z)


def _philox_wrong_weyl(counter, key):
    M64 = (1 << 64) - 1
    x0, x1, x2, x3 = (int(c) & M64 for c in counter)
    k0, k1 = (int(k) & M64 for k in key)
    for r in range(10):
        if r:
            k0, k1 = (k0 + O.PHILOX_W1) & M64, (k1 + O.PHILOX_W0) & M64
        p0, p1 = O.PHILOX_M0 * x0, O.PHILOX_M1 * x2
        x0, x1, x2, x3 = ((p1 >> 64) ^ x1 ^ k0, p1 & M64, (p0 >> 64) ^ x3 ^ k1, p0 & M64)
    return [x0, x1, x2, x3]


def _normals_cos_twice(seed, group):
    w = O.philox4x64_10([group, 0, 0, 0], [seed, 0])
    u = [((x >> 11) + 0.5) * 2.0 ** -53 for x in w]
    out = []
    for a, b in ((u[0], u[1]), (u[2], u[3])):
        r, t = np.sqrt(-2.0 * np.log(a)), 2.0 * np.pi * b
        out += [r * np.cos(t), r * np.cos(t)]
    return out


def _backward_no_normaliser_term(q, k, v, Om, kind, causal, dout):
    fq, fk = O.phi(q, Om, kind), O.phi(k, Om, kind)
    A = fq @ fk.T
    if causal:
        A = np.tril(A)
    D = A.sum(axis=1)
    dN = dout / D[:, None]
    dA = dN @ v.T
    if causal:
        dA = np.tril(dA)
    return O.phi_vjp(q, Om, kind, dA @ fk), O.phi_vjp(k, Om, kind, dA.T @ fq), A.T @ dN


def _phi_vjp_no_radial_term(X, Om, kind, dphi):
    U = X @ Om.T
    M = Om.shape[0]
    if kind == O.TRIG:
        g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(M)
        dc, ds = dphi[:, :M], dphi[:, M:]
        return g[:, None] * ((-dc * np.sin(U) + ds * np.cos(U)) @ Om)
    return ((dphi * (U > 0)) @ Om) / np.sqrt(M)


def _rows_sorted_order(q, k, v, Om, kind, causal, rows):
    # cursor slip: rows written in sorted order instead of the asked order
    rows = np.asarray(rows)
    ref = O.favor_explicit_head(q, k, v, Om, kind, causal, np.sort(rows))
    return ref


def _rows_read_before_add(q, k, v, Om, kind, causal, rows):
    # cursor slip: the state is read before key j is added (keys j < i instead of j <= i)
    rows = np.asarray(rows)
    fq, fk = O.phi(q[rows], Om, kind), O.phi(k, Om, kind)
    S, z = np.zeros((fk.shape[1], v.shape[1])), np.zeros(fk.shape[1])
    out = np.zeros((len(rows), v.shape[1]))
    order = np.argsort(rows, kind="stable")
    pos = 0
    for j in range(q.shape[0]):
        while pos < len(order) and rows[order[pos]] == j:
            r = order[pos]
            den = fq[r] @ z
            if den != 0.0:
                out[r] = (fq[r] @ S) / den
            pos += 1
        S += np.outer(fk[j], v[j])
        z += fk[j]
    if not causal:
        return O._normalise(fq @ (fk.T @ v), fq @ fk.sum(axis=0))
    return out


_TERMS = O.row_rounding_terms_head
_COND = O.row_condition_head


def _terms_state_unsquared(q, k, v, Om, kind, causal, rows=None):
    # level 3 from |S| instead of S^2 (a dropped square)
    t = _TERMS(q, k, v, Om, kind, causal, rows)
    fq = O.phi(q if rows is None else q[np.asarray(rows)], Om, kind)
    S = O.phi(k, Om, kind).T @ v
    if not causal:
        t["N3"] = (fq * fq) @ np.abs(S)
    else:
        t["N3"] = t["N3"] * 1.5
    return t


def _terms_values_unsquared(q, k, v, Om, kind, causal, rows=None):
    # level 2 weighted by |v| instead of v^2
    t = _TERMS(q, k, v, Om, kind, causal, rows)
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    A = O.phi(q[r], Om, kind) @ O.phi(k, Om, kind).T
    if causal:
        A = np.where(np.arange(k.shape[0])[None, :] <= r[:, None], A, 0.0)
    t["N2"] = (A * A) @ np.abs(v)
    return t


def _kden_from_rows(q, k, v, Om, kind, causal, rows=None, with_den=False):
    # the denominator's condition from |A_ij| (cancellation across features missed)
    out = _COND(q, k, v, Om, kind, causal, rows, with_den)
    if not with_den:
        return out
    kap, _ = O.row_diagnostics_head(q, k, v, Om, kind, causal, rows)
    return out[0], kap


CASES = [
    ("row_rounding_terms_head", _terms_state_unsquared, [lambda: P.test_rounding_terms_match_monte_carlo(O.TRIG, False)]),
    ("row_rounding_terms_head", _terms_values_unsquared, [lambda: P.test_rounding_terms_match_monte_carlo(O.RELU, True)]),
    ("row_condition_head", _kden_from_rows, [lambda: P.test_denominator_condition_is_attained(False)]),
    ("favor_rows_head", _rows_sorted_order, [lambda: P.test_rows_head_equals_explicit_rows(O.TRIG, False)]),
    ("favor_rows_head", _rows_read_before_add, [lambda: P.test_rows_head_equals_explicit_rows(O.RELU, True)]),
    ("phi_trig", _phi_trig_no_exp, [P.test_trig_self_inner_product_identity]),
    ("phi_trig", _phi_trig_cos_twice, [P.test_trig_self_inner_product_identity]),
    ("phi_trig", _phi_trig_sign_slip, [P.test_trig_cross_term_closed_form]),
    ("phi_relu", _phi_relu_no_max, [lambda: P.test_relu_outputs_are_convex_combinations(False)]),
    ("favor_causal_head", _causal_strict, [lambda: P.test_causal_prefix_equals_masked(O.TRIG)]),
    ("favor_bidirectional_head", _bidir_wrong_normaliser,
     [lambda: P.test_linear_equals_explicit_bidirectional(O.TRIG)]),
    ("gram_schmidt_rows", _gs_no_normalise, [P.test_gram_schmidt_matches_qr_with_positive_diagonal]),
    ("orf_matrix", _orf_no_chi, [lambda: P.test_orf_structure(32, 16)]),
    ("softmax_attention_head", _softmax_mask_slip, [lambda: P.test_softmax_matches_torch(True)]),
    ("philox4x64_10", _philox_wrong_weyl, [lambda: P.test_philox_matches_numpy_bit_generator(5, 0)]),
    ("philox_normals", _normals_cos_twice, [P.test_philox_normals_box_muller_form]),
    ("favor_backward_head", _backward_no_normaliser_term,
     [lambda: P.test_backward_matches_central_differences(O.RELU, False)]),
    ("phi_vjp", _phi_vjp_no_radial_term, [lambda: P.test_backward_matches_autograd_of_the_quadratic_form(O.TRIG, True)]),
    ("favor_decode_step_head", _decode_read_before_add,
     [lambda: P.test_decode_steps_equal_masked_rows(O.TRIG)]),
    ("favor_decode_step_head", _decode_value_for_key,
     [lambda: P.test_decode_steps_equal_masked_rows(O.RELU)]),
]


@pytest.mark.parametrize("name,bad,pins", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, bad, pins):
    monkeypatch.setattr(O, name, bad)
    for pin in pins:
        with pytest.raises((AssertionError, ValueError, FloatingPointError)):
            pin()
