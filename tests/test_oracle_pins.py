"""Pins for the fp64 oracle, each against something other than the oracle itself.

What pins what:
  * exact softmax attention          -> torch.softmax (library special case), brute force
  * trig features                    -> the identity cos^2 + sin^2 = 1, the cosine-difference
                                        identity, a scalar closed form
  * bidirectional linear form        -> the explicit quadratic form D_hat^-1 A_hat V
  * causal prefix loop               -> the masked quadratic form, row 0 = v_0,
                                        last row = bidirectional last row
  * invariants                       -> constant V, linearity in V, joint (k, v)
                                        permutation, permutation of Omega rows, ReLU convexity
  * ORF                              -> QR with a positive R diagonal (numpy.linalg.qr),
                                        orthogonality, chi norms, N(0, I) marginal
  * unbiasedness / variance / M      -> Gaussian characteristic function,
                                        arc-cosine kernel, closed-form i.i.d. variance
The pages print no worked example, so no stored page value pins the oracle.
"""
import math

import numpy as np
import pytest
import torch

import favor_inputs as fi
from oracle import favor_oracle as O


def _qkv(L, d, seed=0, B=1, H=1):
    q, k, v = fi.qkv(B, H, L, d, seed=seed)
    return q.astype(np.float64)[0, 0], k.astype(np.float64)[0, 0], v.astype(np.float64)[0, 0]


def _orf(M, d, seed=0, H=1):
    G, R = fi.orf_gaussians(H, M, d, seed=seed)
    return O.orf_matrices(G, R, M)


# ------------------------------------------------------------------ exact softmax
@pytest.mark.parametrize("causal", [False, True])
def test_softmax_matches_torch(causal):
    q, k, v = _qkv(37, 8, seed=3)
    got = O.softmax_attention_head(q, k, v, causal)
    s = torch.from_numpy(q) @ torch.from_numpy(k).T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(37, 37, dtype=torch.bool), 1), float("-inf"))
    ref = torch.softmax(s, dim=-1) @ torch.from_numpy(v)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_softmax_bruteforce_tiny():
    q = np.array([[0.3, -1.0], [2.0, 0.5], [-0.7, 0.1]])
    k = np.array([[1.0, 0.0], [0.2, -0.4], [0.0, 1.5]])
    v = np.array([[1.0, 2.0, 3.0], [-1.0, 0.0, 4.0], [0.5, 0.5, -2.0]])
    for causal in (False, True):
        exp_out = np.zeros((3, 3))
        for i in range(3):
            w = [math.exp(sum(q[i, t] * k[j, t] for t in range(2))) if (not causal or j <= i) else 0.0
                 for j in range(3)]
            for c in range(3):
                exp_out[i, c] = sum(w[j] * v[j, c] for j in range(3)) / sum(w)
        np.testing.assert_allclose(O.softmax_attention_head(q, k, v, causal), exp_out, rtol=1e-13)
    # rows of D^-1 A sum to one: V = ones gives ones
    np.testing.assert_allclose(O.softmax_attention_head(q, k, np.ones((3, 2)), False), 1.0, rtol=1e-14)


# ------------------------------------------------------------------ feature maps
def test_trig_self_inner_product_identity():
    x, _, _ = _qkv(50, 16, seed=1)
    x = x * 2.5
    om = np.random.default_rng(5).standard_normal((24, 16)) * 3.0  # any Omega works
    f = O.phi_trig(x, om)
    np.testing.assert_allclose(np.sum(f * f, axis=1), np.exp(np.sum(x * x, axis=1)), rtol=1e-12)


def test_trig_cross_term_closed_form():
    q, k, _ = _qkv(20, 16, seed=2)
    om = _orf(32, 16, seed=4)[0]
    got = O.phi_trig(q, om) @ O.phi_trig(k, om).T
    nq = np.sum(q * q, axis=1)[:, None]
    nk = np.sum(k * k, axis=1)[None, :]
    diff = q[:, None, :] - k[None, :, :]                       # [20, 20, d]
    mean_cos = np.cos(np.einsum("ijd,md->ijm", diff, om)).mean(axis=2)
    np.testing.assert_allclose(got, np.exp(0.5 * (nq + nk)) * mean_cos, rtol=1e-11, atol=1e-300)


def test_scalar_closed_form_trig():
    # d = 1, M = 1: a_ij = exp((q_i^2 + k_j^2)/2) cos(w (q_i - k_j)), worked by hand
    w = 0.8
    q = np.array([[0.4], [-1.1], [0.25]])
    k = np.array([[0.9], [-0.3], [0.0]])
    v = np.array([[1.0, -2.0], [0.5, 3.0], [-1.5, 0.25]])
    a = np.array([[math.exp((qi * qi + kj * kj) / 2) * math.cos(w * (qi - kj)) for kj in k[:, 0]]
                  for qi in q[:, 0]])
    bid = (a @ v) / a.sum(axis=1, keepdims=True)
    al = np.tril(a)
    cau = (al @ v) / al.sum(axis=1, keepdims=True)
    om = np.array([[w]])
    np.testing.assert_allclose(O.favor_bidirectional_head(q, k, v, om, O.TRIG), bid, rtol=1e-12)
    np.testing.assert_allclose(O.favor_causal_head(q, k, v, om, O.TRIG), cau, rtol=1e-12)


def test_small_closed_form_relu():
    # Omega = I_2 plus the row (1, -1): phi(x) = (max(x1,0), max(x2,0), max(x1-x2,0))/sqrt(3)
    om = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, -1.0]])
    q = np.array([[1.0, 2.0], [-1.0, 0.5]])
    k = np.array([[2.0, 1.0], [0.5, -1.0], [-3.0, 4.0]])
    v = np.array([[1.0], [2.0], [4.0]])
    f = lambda x: np.array([max(x[0], 0), max(x[1], 0), max(x[0] - x[1], 0)]) / math.sqrt(3)
    a = np.array([[f(qi) @ f(kj) for kj in k] for qi in q])
    # q0 = (1,2): f = (1,2,0)/sqrt3. k0: (2,1,1)/sqrt3 -> 4/3, k1: (.5,0,1.5)/sqrt3 -> .5/3, k2: (0,4,0)/sqrt3 -> 8/3
    np.testing.assert_allclose(a[0], [4 / 3, 0.5 / 3, 8 / 3], rtol=1e-14)
    bid = (a @ v)[:, 0] / a.sum(axis=1)
    np.testing.assert_allclose(O.favor_bidirectional_head(q, k, v, om, O.RELU)[:, 0], bid, rtol=1e-13)


# ------------------------------------------------------------------ reassociation and causal prefix
@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
def test_linear_equals_explicit_bidirectional(kind):
    q, k, v = _qkv(256, 16, seed=0)
    om = _orf(32, 16, seed=0)[0]
    lin = O.favor_bidirectional_head(q, k, v, om, kind)
    exp_ = O.favor_explicit_head(q, k, v, om, kind, causal=False)
    np.testing.assert_allclose(lin, exp_, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
def test_causal_prefix_equals_masked(kind):
    q, k, v = _qkv(200, 16, seed=1)
    om = _orf(32, 16, seed=1)[0]
    cau = O.favor_causal_head(q, k, v, om, kind)
    np.testing.assert_allclose(cau, O.favor_explicit_head(q, k, v, om, kind, causal=True),
                               rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(cau[0], v[0], rtol=1e-12)
    np.testing.assert_allclose(cau[-1], O.favor_bidirectional_head(q, k, v, om, kind)[-1], rtol=1e-10)


# ------------------------------------------------------------------ sampled rows (the GPU tests' reference)
def _sample_rows(L, seed):
    # unsorted, with duplicates, and both ends of the sequence
    rng = np.random.default_rng(seed)
    return np.concatenate([[L - 1, 0], rng.integers(0, L, 40), [7, 7, L - 1, 0, 1]])


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_rows_head_equals_explicit_rows(kind, causal):
    # favor_rows_head walks the keys once with a cursor over the sorted rows; the explicit
    # quadratic form D^-1 A V computes each asked row on its own, in the asked order
    L = 97
    q, k, v = _qkv(L, 16, seed=61)
    om = _orf(32, 16, seed=61)[0]
    rows = _sample_rows(L, 61)
    got = O.favor_rows_head(q, k, v, om, kind, causal, rows)
    ref = O.favor_explicit_head(q, k, v, om, kind, causal, rows)
    assert got.shape == (len(rows), v.shape[1])
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    if causal:
        np.testing.assert_allclose(got[1], v[0], rtol=1e-12)  # row 0 reads key 0 alone
    np.testing.assert_allclose(got[0], got[-3], rtol=1e-13)  # duplicated row L-1


@pytest.mark.parametrize("causal", [False, True])
def test_row_condition_follows_the_asked_rows(causal):
    # the cursor of row_condition_head: asked rows in any order (duplicates included) give the
    # same numbers as the full sequence taken at those rows
    L = 97
    q, k, v = _qkv(L, 16, seed=62)
    om = _orf(32, 16, seed=62)[0]
    rows = _sample_rows(L, 62)
    full = O.row_condition_head(q, k, v, om, O.TRIG, causal)
    np.testing.assert_allclose(O.row_condition_head(q, k, v, om, O.TRIG, causal, rows), full[rows], rtol=1e-12)


# ------------------------------------------------------------------ decode step (carried state)
@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
def test_decode_steps_equal_masked_rows(kind):
    # calls from an empty state reproduce the quadratic masked form row by row
    L, d, M = 150, 16, 32
    q, k, v = _qkv(L, d, seed=2)
    om = _orf(M, d, seed=2)[0]
    S, z = O.favor_decode_state(M, d, kind)
    rows = np.stack([O.favor_decode_step_head(S, z, q[i], k[i], v[i], om, kind) for i in range(L)])
    np.testing.assert_allclose(rows, O.favor_explicit_head(q, k, v, om, kind, causal=True),
                               rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(rows[0], v[0], rtol=1e-12)
    # the final state, read by fresh queries, is bidirectional attention over all L keys
    qn = np.random.default_rng(5).standard_normal((7, d)) * 0.3
    fq = O.phi(qn, om, kind)
    np.testing.assert_allclose((fq @ S) / (fq @ z)[:, None],
                               O.favor_explicit_head(qn, k, v, om, kind, causal=False),
                               rtol=1e-9, atol=1e-12)


def test_decode_state_is_order_free():
    # the state is a sum over tokens: feeding them in another order gives the same state
    L, d, M = 40, 8, 16
    q, k, v = _qkv(L, d, seed=3)
    om = _orf(M, d, seed=3)[0]
    S1, z1 = O.favor_decode_state(M, d, O.TRIG)
    S2, z2 = O.favor_decode_state(M, d, O.TRIG)
    for i in range(L):
        O.favor_decode_step_head(S1, z1, q[i], k[i], v[i], om, O.TRIG)
    for i in np.random.default_rng(0).permutation(L):
        O.favor_decode_step_head(S2, z2, q[i], k[i], v[i], om, O.TRIG)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z1, z2, rtol=1e-12, atol=1e-12)
    assert S1.shape == (2 * M, d) and z1.shape == (2 * M,)


# ------------------------------------------------------------------ counter-based ORF draws
def _words(x, n):
    return [(x >> (64 * i)) & ((1 << 64) - 1) for i in range(n)]


@pytest.mark.parametrize("key,counter", [(0, 0), (5, 0), (2**64 + 3, 2**64 - 3), (2**128 - 1, 2**200 + 2**64 - 2),
                                         (0x243F6A8885A308D3, 0x13198A2E03707344)])
def test_philox_matches_numpy_bit_generator(key, counter):
    # numpy's Philox bit generator (its own C implementation) advances the counter before each
    # block: its outputs 4i .. 4i+3 are the block of counter + 1 + i
    raw = np.random.Philox(key=key, counter=counter).random_raw(24)
    mine = []
    for i in range(6):
        mine += O.philox4x64_10(_words((counter + 1 + i) % 2**256, 4), _words(key, 2))
    assert [int(x) for x in raw] == mine


def test_philox_normals_are_standard_normal():
    from scipy import stats
    z = np.array([x for g in range(5000) for x in O.philox_normals(11, g)])
    assert abs(z.mean()) < 4 / np.sqrt(z.size) and abs(z.var() - 1) < 6 * np.sqrt(2 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # the two members of a Box-Muller pair are uncorrelated, and so are neighbouring groups
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 4 / np.sqrt(z.size / 2)
    assert abs(np.corrcoef(z[:-4], z[4:])[0, 1]) < 4 / np.sqrt(z.size)


def test_philox_normals_box_muller_form():
    # the words map to u in (0, 1) and a pair (u_a, u_b) to sqrt(-2 ln u_a) (cos, sin)(2 pi u_b):
    # the squared norm of each pair is -2 ln u_a, whatever u_b
    for g in (0, 7, 123456789):
        w = O.philox4x64_10([g, 0, 0, 0], [3, 0])
        z = O.philox_normals(3, g)
        for p in range(2):
            ua = ((w[2 * p] >> 11) + 0.5) * 2.0 ** -53
            assert 0.0 < ua < 1.0
            assert z[2 * p] ** 2 + z[2 * p + 1] ** 2 == pytest.approx(-2.0 * math.log(ua), rel=1e-13)


def test_seeded_orf_gaussians_layout():
    H, M, d, seed = 2, 40, 8, 9
    G, R = O.seeded_orf_gaussians(seed, H, M, d)
    nb = 5
    assert G.shape == (H, nb, d, d) and R.shape == (H, M, d)
    NG = -(-H * nb * d * d // 4) * 4
    for (h, b, i, j) in [(0, 0, 0, 0), (1, 4, 7, 7), (1, 2, 3, 5)]:
        n = ((h * nb + b) * d + i) * d + j
        assert G[h, b, i, j] == O.philox_normals(seed, n // 4)[n % 4]
    for (h, r, j) in [(0, 0, 0), (1, 39, 7), (0, 17, 2)]:
        n = NG + (h * M + r) * d + j
        assert R[h, r, j] == O.philox_normals(seed, n // 4)[n % 4]
    # a different seed gives different draws; the same seed the same draws
    G2, _ = O.seeded_orf_gaussians(seed + 1, H, M, d)
    assert not np.allclose(G, G2)
    assert np.array_equal(G, O.seeded_orf_gaussians(seed, H, M, d)[0])


# ------------------------------------------------------------------ backward
def _loss(q, k, v, om, kind, causal, dout):
    return float(np.sum(dout * O.favor_explicit_head(q, k, v, om, kind, causal)))


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_differences(kind, causal):
    # every coordinate of q, k and v, central differences of sum(dout * out) in fp64
    L, d, M = 10, 4, 8
    q, k, v = _qkv(L, d, seed=4)
    om = _orf(M, d, seed=4)[0]
    dout = np.random.default_rng(8).standard_normal((L, d))
    g = O.favor_backward_head(q, k, v, om, kind, causal, dout)
    h = 1e-6
    for which, x in enumerate((q, k, v)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd[idx] = (_loss(*args_p, om, kind, causal, dout) - _loss(*args_m, om, kind, causal, dout)) / (2 * h)
        np.testing.assert_allclose(g[which], fd, rtol=1e-5, atol=1e-6 * np.abs(fd).max())


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_autograd_of_the_quadratic_form(kind, causal):
    # torch autograd (fp64) through the quadratic form written with torch ops
    L, d, M = 40, 8, 16
    q, k, v = _qkv(L, d, seed=6)
    om = _orf(M, d, seed=6)[0]
    dout = np.random.default_rng(9).standard_normal((L, d))
    T = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
    W = torch.tensor(om, dtype=torch.float64)

    def feats(X):
        U = X @ W.T
        if kind == O.TRIG:
            g = torch.exp(0.5 * (X * X).sum(dim=1, keepdim=True)) / math.sqrt(M)
            return g * torch.cat([torch.cos(U), torch.sin(U)], dim=1)
        return torch.relu(U) / math.sqrt(M)

    A = feats(T[0]) @ feats(T[1]).T
    if causal:
        A = torch.tril(A)
    out = (A @ T[2]) / A.sum(dim=1, keepdim=True)
    (out * torch.tensor(dout)).sum().backward()
    for mine, t in zip(O.favor_backward_head(q, k, v, om, kind, causal, dout), T):
        np.testing.assert_allclose(mine, t.grad.numpy(), rtol=1e-9, atol=1e-12 * np.abs(t.grad.numpy()).max())


def test_backward_of_constant_v_has_no_q_or_k_gradient():
    # out_i = c for every row whatever the weights, so dq = dk = 0 and dv sums dout
    L, d, M = 30, 8, 16
    q, k, _ = _qkv(L, d, seed=2)
    v = np.tile(np.linspace(-1, 1, d), (L, 1))
    om = _orf(M, d, seed=2)[0]
    dout = np.random.default_rng(1).standard_normal((L, d))
    for kind in (O.TRIG, O.RELU):
        dq, dk, dv = O.favor_backward_head(q, k, v, om, kind, False, dout)
        assert np.abs(dq).max() < 1e-9 * np.abs(dout).max() and np.abs(dk).max() < 1e-9 * np.abs(dout).max()
        # rows of A / D sum to one, so sum_j dv_j = sum_i dout_i
        np.testing.assert_allclose(dv.sum(axis=0), dout.sum(axis=0), rtol=1e-9)


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_magnitudes_bound_perturbed_gradients(kind, causal):
    # the magnitudes dominate the gradients, and a relative perturbation of size eps on every
    # factor (features, V, dout) moves the gradients by at most a few eps times them
    L, d, M = 24, 8, 16
    q, k, v = _qkv(L, d, seed=12)
    om = _orf(M, d, seed=12)[0]
    dout = np.random.default_rng(13).standard_normal((L, d))
    g = O.favor_backward_head(q, k, v, om, kind, causal, dout)
    mags = O.backward_magnitudes_head(q, k, v, om, kind, causal, dout)
    cond = O.row_condition_head(q, k, v, om, kind, causal)
    for a, m in zip(g, mags):
        assert np.all(np.abs(a) <= m * (1 + 1e-12) + 1e-300)
    eps = 1e-7
    rng = np.random.default_rng(14)
    base_phi = O.phi
    orig = O.phi

    def noisy(X, Om, kd):
        f = base_phi(X, Om, kd)
        return f * (1 + eps * rng.uniform(-1, 1, f.shape))
    try:
        O.phi = noisy
        gp = O.favor_backward_head(q, k, v * (1 + eps * rng.uniform(-1, 1, v.shape)), om, kind, causal,
                                   dout * (1 + eps * rng.uniform(-1, 1, dout.shape)))
    finally:
        O.phi = orig
    # first order: the change is bounded by eps (magnitudes + cond * |gradient|), up to a small factor
    worst = max(float(cond[np.isfinite(cond)].max()), 1.0)
    for a, b, m in zip(g, gp, mags):
        assert np.all(np.abs(a - b) <= 20 * eps * (m + worst * np.abs(a).max()))


# ------------------------------------------------------------------ invariants
@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_invariants(kind, causal):
    q, k, v = _qkv(96, 16, seed=7)
    om = _orf(32, 16, seed=7)[0]
    f = O.favor_causal_head if causal else O.favor_bidirectional_head
    c = np.linspace(-1.0, 2.0, 16)
    np.testing.assert_allclose(f(q, k, np.tile(c, (96, 1)), om, kind), np.tile(c, (96, 1)), rtol=1e-9)
    v2 = np.random.default_rng(1).standard_normal(v.shape)
    np.testing.assert_allclose(f(q, k, 2.0 * v - 3.0 * v2, om, kind),
                               2.0 * f(q, k, v, om, kind) - 3.0 * f(q, k, v2, om, kind), rtol=1e-9, atol=1e-11)
    perm = np.random.default_rng(2).permutation(32)
    np.testing.assert_allclose(f(q, k, v, om[perm], kind), f(q, k, v, om, kind), rtol=1e-9, atol=1e-12)
    if not causal:
        p = np.random.default_rng(3).permutation(96)
        np.testing.assert_allclose(f(q, k[p], v[p], om, kind), f(q, k, v, om, kind), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_relu_outputs_are_convex_combinations(causal):
    q, k, v = _qkv(128, 16, seed=9)
    om = _orf(32, 16, seed=9)[0]
    out = (O.favor_causal_head if causal else O.favor_bidirectional_head)(q, k, v, om, O.RELU)
    for i in range(128):
        vv = v[: i + 1] if causal else v
        assert np.all(out[i] >= vv.min(axis=0) - 1e-12) and np.all(out[i] <= vv.max(axis=0) + 1e-12)
    kap, _ = O.row_diagnostics_head(q, k, v, om, O.RELU, causal)
    np.testing.assert_allclose(kap, 1.0, rtol=1e-12)


def test_zero_denominator_gives_zero_row():
    om = np.array([[1.0, 0.0], [0.0, 1.0]])
    q = np.array([[-1.0, -1.0], [1.0, 1.0]])        # phi_relu(q0) = 0
    k = np.array([[1.0, 2.0], [3.0, 0.5]])
    v = np.array([[1.0, 1.0], [2.0, -1.0]])
    out = O.favor_bidirectional_head(q, k, v, om, O.RELU)
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out))


# ------------------------------------------------------------------ ORF
def test_gram_schmidt_matches_qr_with_positive_diagonal():
    G = np.random.default_rng(11).standard_normal((64, 64))
    Qr, Rr = np.linalg.qr(G.T)          # G^T = Qr Rr, columns of Qr = rows orthonormalised in order
    Qr = Qr * np.sign(np.diag(Rr))[None, :]
    np.testing.assert_allclose(O.gram_schmidt_rows(G), Qr.T, atol=1e-11)


@pytest.mark.parametrize("M,d", [(32, 16), (256, 64), (40, 16)])
def test_orf_structure(M, d):
    G, R = fi.orf_gaussians(1, M, d, seed=5)
    om = O.orf_matrix(G[0], R[0], M)
    assert om.shape == (M, d)
    norms = np.linalg.norm(om, axis=1)
    np.testing.assert_allclose(norms, np.linalg.norm(R[0], axis=1), rtol=1e-12)
    unit = om / norms[:, None]
    for b0 in range(0, M, d):
        blk = unit[b0:b0 + d]
        np.testing.assert_allclose(blk @ blk.T, np.eye(blk.shape[0]), atol=1e-12)
    # the rows come from the blocks in order, the last block cut when d does not divide M
    np.testing.assert_allclose(unit[:d], O.gram_schmidt_rows(G[0, 0]), atol=1e-13)


def test_orf_row_marginal_is_standard_normal():
    d, M, n = 8, 16, 3000
    rows = []
    for s in range(n):
        G, R = fi.orf_gaussians(1, M, d, seed=1000 + s)
        rows.append(O.orf_matrix(G[0], R[0], M))
    W = np.concatenate(rows)                      # n*M rows
    cov = W.T @ W / W.shape[0]
    np.testing.assert_allclose(cov, np.eye(d), atol=0.05)
    chi_mean = math.sqrt(2) * math.exp(math.lgamma((d + 1) / 2) - math.lgamma(d / 2))
    assert abs(np.linalg.norm(W, axis=1).mean() - chi_mean) < 0.02


# ------------------------------------------------------------------ Monte-Carlo: unbiasedness, variance, M
def _mc_estimates(q, k, M, n, kind, structured):
    d = q.shape[1]
    est = np.empty((n, q.shape[0], k.shape[0]))
    for s in range(n):
        if structured:
            G, R = fi.orf_gaussians(1, M, d, seed=50000 + s)
            om = O.orf_matrix(G[0], R[0], M)
        else:
            om = fi.iid_gaussians(1, M, d, seed=50000 + s)[0]
        est[s] = O.phi(q, om, kind) @ O.phi(k, om, kind).T
    return est


def _arccos_kernel(q, k):
    nq = np.linalg.norm(q, axis=1)[:, None]
    nk = np.linalg.norm(k, axis=1)[None, :]
    c = np.clip(q @ k.T / (nq * nk), -1, 1)
    t = np.arccos(c)
    return nq * nk * (np.sin(t) + (np.pi - t) * c) / (2 * np.pi)


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("structured", [True, False])
def test_kernel_estimate_is_unbiased(kind, structured):
    q, k, _ = _qkv(16, 16, seed=21)
    n = 3000
    est = _mc_estimates(q, k[:12], 32, n, kind, structured)
    exact = np.exp(q @ k[:12].T) if kind == O.TRIG else _arccos_kernel(q, k[:12])
    z = (est.mean(axis=0) - exact) / (est.std(axis=0, ddof=1) / math.sqrt(n))
    # the pairs share the same draws, so their z-scores are correlated: bound each one
    assert np.abs(z).max() < 4.5


def test_trig_variance_closed_form_and_orf_reduction():
    # small |q - k|, where orthogonal directions cut the variance most
    q, k, _ = _qkv(10, 16, seed=31)
    q, k = 0.5 * q, 0.5 * k[:10]
    n, M = 2000, 32
    iid = _mc_estimates(q, k, M, n, O.TRIG, structured=False)
    orf = _mc_estimates(q, k, M, n, O.TRIG, structured=True)
    nq = np.sum(q * q, axis=1)[:, None]
    nk = np.sum(k * k, axis=1)[None, :]
    dd = np.sum((q[:, None, :] - k[None, :, :]) ** 2, axis=2)
    closed = np.exp(nq + nk) * (1 - np.exp(-dd)) ** 2 / (2 * M)
    ratio = iid.var(axis=0, ddof=1) / closed
    assert 0.9 < ratio.mean() < 1.1
    assert np.all((ratio > 0.75) & (ratio < 1.3))
    assert (orf.var(axis=0, ddof=1) / closed).mean() < 0.5


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
def test_error_shrinks_with_feature_count(kind):
    q, k, v = _qkv(64, 16, seed=41)
    ref = (O.softmax_attention_head(q, k, v, False) if kind == O.TRIG
           else O.arccos_attention_head(q, k, v, False))
    Ms = [16, 64, 256, 1024]
    err = []
    for M in Ms:
        e = []
        for s in range(16):
            G, R = fi.orf_gaussians(1, M, 16, seed=7000 + 97 * s + M)
            om = O.orf_matrix(G[0], R[0], M)
            e.append(np.median(np.abs(O.favor_bidirectional_head(q, k, v, om, kind) - ref)))
        # medians: the trig ratio estimator has a signed denominator and heavy tails
        err.append(np.median(e))
    assert all(err[i + 1] < err[i] for i in range(len(err) - 1))
    slope = np.polyfit(np.log(Ms), np.log(err), 1)[0]
    assert -0.7 < slope < -0.35


# ------------------------------------------------------------------ condition number used by the parity metric
@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_row_condition_bounds_feature_perturbations(kind, causal):
    # perturb every feature of q and k by a relative +-u: each product moves by at most ~2u, so
    # each row may move by at most ~2u cond_i max|o_i|
    q, k, v = _qkv(80, 16, seed=51)
    om = _orf(32, 16, seed=51)[0]
    rows = np.arange(80)
    cond = O.row_condition_head(q, k, v, om, kind, causal, rows)
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    base = O.favor_explicit_head(q, k, v, om, kind, causal)
    u = 1e-6
    rng = np.random.default_rng(3)
    worst = 0.0
    for _ in range(5):
        pq = fq * (1 + u * rng.choice([-1.0, 1.0], fq.shape))
        pk = fk * (1 + u * rng.choice([-1.0, 1.0], fk.shape))
        A = pq @ pk.T
        if causal:
            A = np.tril(A)
        out = (A @ v) / A.sum(axis=1, keepdims=True)
        ratio = np.abs(out - base).max(axis=1) / (np.abs(base).max(axis=1) * 2 * u * cond)
        worst = max(worst, ratio.max())
    assert worst <= 1.01
    if kind == O.RELU:
        # all terms non-negative: D_i = den_i, so cond_i = N_i/(den_i |o_i|) + 1 is modest
        assert cond.max() < 1e3


def _terms(q, k, om, kind, causal):
    """Products t[i, f, j] = phi_f(q_i) phi_f(k_j), zero where j > i when causal."""
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    t = fq[:, :, None] * fk.T[None, :, :]
    if causal:
        t = t * (np.arange(k.shape[0])[None, None, :] <= np.arange(q.shape[0])[:, None, None])
    return t


@pytest.mark.parametrize("causal", [False, True])
def test_denominator_condition_is_attained(causal):
    # every product moved by u |t| against the sign of den_i moves den_i by exactly u D_i: at
    # u = 0.999 / kappa_i the denominator keeps its sign with |den_i| (1 - u kappa_i) left, at
    # u = 1.001 / kappa_i it changes sign. This fixes both D_i and |den_i|.
    q, k, v = _qkv(80, 16, seed=52)
    om = _orf(32, 16, seed=52)[0]
    _, kden = O.row_condition_head(q, k, v, om, O.TRIG, causal, with_den=True)
    t = _terms(q, k, om, O.TRIG, causal)
    den = t.sum(axis=(1, 2))
    sgn = np.sign(den)[:, None, None]
    for frac in (0.999, 1.001):
        u = (frac / kden)[:, None, None]
        den2 = (t - u * np.abs(t) * sgn).sum(axis=(1, 2))
        if frac < 1:
            assert np.all(np.sign(den2) == np.sign(den))
            np.testing.assert_allclose(np.abs(den2), np.abs(den) * (1 - frac), rtol=1e-6)
        else:
            assert np.all(np.sign(den2) == -np.sign(den))
    # ReLU products are non-negative: the denominator is perfectly conditioned
    _, kr = O.row_condition_head(q, k, v, om, O.RELU, causal, with_den=True)
    ok = np.isfinite(kr)
    np.testing.assert_allclose(kr[ok], 1.0, rtol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_all_orders_bound_holds_far_from_first_order(causal):
    # independent relative perturbations of size <= u of every numerator and denominator
    # product, with u so large that u kappa_i reaches 0.9 on the worst row: every row moves by
    # at most u cond_i / (1 - u kappa_i) of its max, the bound the parity metric uses
    q, k, v = _qkv(48, 16, seed=53)
    om = _orf(32, 16, seed=53)[0]
    cond, kden = O.row_condition_head(q, k, v, om, O.TRIG, causal, with_den=True)
    t = _terms(q, k, om, O.TRIG, causal)
    base = O.favor_explicit_head(q, k, v, om, O.TRIG, causal)
    u = 0.9 / kden.max()
    rng = np.random.default_rng(5)
    worst = 0.0
    for trial in range(4):
        # trial 0 pushes every product against its row's denominator; the rest are random
        if trial == 0:
            ed = -np.sign(t.sum(axis=(1, 2)))[:, None, None] * np.sign(t)
        else:
            ed = rng.uniform(-1, 1, t.shape)
        en = rng.uniform(-1, 1, t.shape + (v.shape[1],))
        num = np.einsum("ifj,ifjn,jn->in", t, 1 + u * en, v)
        den = (t * (1 + u * ed)).sum(axis=(1, 2))
        out = num / den[:, None]
        bound = u * cond / (1 - u * kden)
        ratio = np.abs(out - base).max(axis=1) / (np.abs(base).max(axis=1) * bound)
        worst = max(worst, ratio.max())
    assert worst <= 1.0 + 1e-9


@pytest.mark.parametrize("kind", [O.TRIG, O.RELU])
@pytest.mark.parametrize("causal", [False, True])
def test_rounding_terms_match_monte_carlo(kind, causal):
    # perturb one level's operands by independent N(0, s^2) relative errors and recompute
    # num and den by brute force: their sample variances over the trials must equal s^2 times
    # the level's sums of squares (4000 trials: the ratio's spread is about 2%)
    L, d, M = 24, 8, 8
    q, k, v = _qkv(L, d, seed=54)
    om = _orf(M, d, seed=54)[0]
    t = O.row_rounding_terms_head(q, k, v, om, kind, causal)
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    mask = np.tril(np.ones((L, L))) if causal else np.ones((L, L))
    # per-row states S_i, z_i over the keys each row sees
    S = np.einsum("ij,jf,jn->ifn", mask, fk, v)
    z = np.einsum("ij,jf->if", mask, fk)
    A = (fq @ fk.T) * mask
    s, T = 1e-7, 4000
    rng = np.random.default_rng(11)
    acc = {key: [] for key in ("1", "2", "3")}
    for _ in range(T):
        e1 = rng.standard_normal(fk.shape) * s
        fk_p = fk * (1 + e1)
        A1 = (fq @ fk_p.T) * mask
        e2 = rng.standard_normal((L, L)) * s
        A2 = A * (1 + e2)
        e3 = rng.standard_normal(S.shape[1:]) * s
        e3z = rng.standard_normal(z.shape[1:]) * s
        n3 = np.einsum("if,ifn->in", fq, S * (1 + e3)[None])
        d3 = np.einsum("if,if->i", fq, z * (1 + e3z)[None])
        acc["1"].append(np.concatenate([A1 @ v, A1.sum(axis=1)[:, None]], axis=1))
        acc["2"].append(np.concatenate([A2 @ v, A2.sum(axis=1)[:, None]], axis=1))
        acc["3"].append(np.concatenate([n3, d3[:, None]], axis=1))
    for lev in ("1", "2", "3"):
        var = np.var(np.stack(acc[lev]), axis=0) / s ** 2
        want = np.concatenate([t["N" + lev], t["D" + lev][:, None]], axis=1)
        live = want > 1e-12 * want.max()
        np.testing.assert_allclose(var[live], want[live], rtol=0.12)
        assert np.all(var[~live] <= 1e-6 * want.max())
    # and the values themselves
    base = O.favor_explicit_head(q, k, v, om, kind, causal)
    np.testing.assert_allclose(t["out"], base, rtol=1e-9, atol=1e-12 * np.abs(base).max())
    np.testing.assert_allclose(t["den"], A.sum(axis=1), rtol=1e-9)


@pytest.mark.parametrize("causal", [False, True])
def test_rounding_terms_follow_the_asked_rows(causal):
    q, k, v = _qkv(97, 16, seed=55)
    om = _orf(32, 16, seed=55)[0]
    rows = np.array([96, 3, 40, 3, 0, 77])
    full = O.row_rounding_terms_head(q, k, v, om, O.TRIG, causal)
    part = O.row_rounding_terms_head(q, k, v, om, O.TRIG, causal, rows)
    for key in full:
        np.testing.assert_allclose(part[key], full[key][rows], rtol=1e-12, atol=0)
