"""FAVOR attention oracle: a plain, slow fp64 CPU implementation.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs may import this module. The CUDA library never calls it and shares no
code with it. Inputs reach both sides from the ``favor_inputs`` generator alone.

Sources (page title, section):
  [EXPL] "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？" (explainer of arXiv 2009.14794),
         section "核心机制：FAVOR+". Covers:
         - Att = D^-1 A V with A = exp(QK^T/sqrt(d));
         - exp(q^T k/sqrt(d)) ~ phi(q)^T phi(k);
         - phi(K)^T V aggregated first (an m x v state), then left-multiplied by phi(Q);
         - D_hat = phi(Q)(phi(K)^T 1);
         - the trigonometric mode (cos/sin pairs, from Rahimi-Recht random Fourier features);
         - ORF directions;
         - the causal prefix sum of phi(k_j) v_j^T over j <= i.
  [MLMP-zh] "Masked Language Modeling for Proteins via Linearly Scalable Long-Context
         Transformers" (gptget.net, Chinese), sections "方法详解" and "核心创新"
         (Gaussian-kernel random features, ORF, prefix sum, generalized attention),
         and "实验设计" (orthogonal vs unstructured ablation).
  [MLMP-en] the same title (gptget.net, English), sections "Methodology" and
         "AI Executive Summary" (Gaussian kernel random features, orthogonal sampling).

Readings where the pages are silent:
  * Trig map. phi(x) = exp(|x|^2/2)/sqrt(M) * [cos(w_1.x) .. cos(w_M.x), sin(w_1.x) .. sin(w_M.x)].
    This is the random Fourier feature map of the Gaussian kernel, times exp(|x|^2/2),
    because exp(q.k) = exp(|q|^2/2) exp(-|q-k|^2/2) exp(|k|^2/2).
  * ReLU (generalized attention) map. phi(x) = max(Omega x, 0)/sqrt(M).
  * Temperature. The 1/sqrt(d) is carried by the inputs (Q and K pre-scaled by
    d^-1/4). Nothing here rescales.
  * ORF. ceil(M/d) blocks of d x d Gaussians, rows orthonormalised in order
    (Gram-Schmidt, equivalently QR with a positive R diagonal). Row r is then scaled by
    the length of an independent N(0, I_d) vector (chi_d), the blocks are stacked,
    and the result is cut to M rows.
  * A zero denominator gives a zero output row. A negative trig denominator is used
    as is.
Every factor is kept in fp64. There is no stabiliser, and exp(|x|^2/2) is finite
for |x|^2/2 < 709.
"""
from __future__ import annotations

import numpy as np

TRIG = 0
RELU = 1


# ---------------------------------------------------------------- random matrices
def gram_schmidt_rows(G: np.ndarray) -> np.ndarray:
    """Orthonormalise the rows of a square block in order.

    Classical Gram-Schmidt, applied twice per row ("twice is enough"), so the rows are
    orthonormal to fp64 rounding. [EXPL, 核心机制] constrains the directions to a random
    subsample of an orthogonal matrix, and [MLMP-zh, 方法详解] calls them orthogonal
    random features.
    """
    Q = np.array(G, dtype=np.float64, copy=True)
    for i in range(Q.shape[0]):
        v = Q[i].copy()
        for _ in range(2):
            if i:
                v = v - Q[:i].T @ (Q[:i] @ v)
        Q[i] = v / np.linalg.norm(v)
    return Q


def orf_matrix(G: np.ndarray, R: np.ndarray, M: int) -> np.ndarray:
    """ORF Omega [M, d] for one head.

    G [nb, d, d] holds the Gaussian blocks and R [M, d] the chi draws. Each block is
    orthonormalised, row r is scaled by |R[r]|, the blocks are stacked and the result
    is cut to M rows.
    """
    blocks = [gram_schmidt_rows(G[i]) for i in range(G.shape[0])]
    Q = np.concatenate(blocks, axis=0)[:M]
    return Q * np.linalg.norm(R, axis=1)[:, None]


def orf_matrices(G: np.ndarray, R: np.ndarray, M: int) -> np.ndarray:
    """Per-head ORF matrices: G [H, nb, d, d], R [H, M, d] -> Omega [H, M, d]."""
    return np.stack([orf_matrix(G[h], R[h], M) for h in range(G.shape[0])])


# ---------------------------------------------------------------- counter-based draws
# The ORF directions and lengths are Gaussian draws ([EXPL, 核心机制]; [MLMP-zh, 方法详解]).
# To redraw Omega on the device from a seed, both sides generate the draws with the same
# counter-based generator, each from its published definition: Philox4x64 with 10 rounds
# (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011).
_M64 = (1 << 64) - 1
PHILOX_M0, PHILOX_M1 = 0xD2E7470EE14C6C93, 0xCA5A826395121157   # round multipliers
PHILOX_W0, PHILOX_W1 = 0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B   # key increments (Weyl)


def philox4x64_10(counter, key):
    """One Philox4x64-10 block: counter (4 words) and key (2 words) -> 4 uint64 words.

    Python integers, so every product and xor is exact. A round maps
    (x0, x1, x2, x3) to (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0));
    the key gains (W0, W1) between rounds.
    """
    x0, x1, x2, x3 = (int(c) & _M64 for c in counter)
    k0, k1 = (int(k) & _M64 for k in key)
    for r in range(10):
        if r:
            k0, k1 = (k0 + PHILOX_W0) & _M64, (k1 + PHILOX_W1) & _M64
        p0, p1 = PHILOX_M0 * x0, PHILOX_M1 * x2
        x0, x1, x2, x3 = ((p1 >> 64) ^ x1 ^ k0, p1 & _M64, (p0 >> 64) ^ x3 ^ k1, p0 & _M64)
    return [x0, x1, x2, x3]


def philox_normals(seed, group):
    """Four N(0, 1) draws of group `group`: Philox4x64-10 of counter (group, 0, 0, 0) and key
    (seed, 0); each word w gives u = (floor(w / 2^11) + 1/2) 2^-53 in (0, 1), and the pairs
    (u0, u1), (u2, u3) go through Box-Muller: sqrt(-2 ln u_a) (cos, sin)(2 pi u_b)."""
    w = philox4x64_10([group, 0, 0, 0], [seed, 0])
    u = [((x >> 11) + 0.5) * 2.0 ** -53 for x in w]
    out = []
    for a, b in ((u[0], u[1]), (u[2], u[3])):
        r, t = np.sqrt(-2.0 * np.log(a)), 2.0 * np.pi * b
        out += [r * np.cos(t), r * np.sin(t)]
    return out


def seeded_orf_gaussians(seed, H, M, d):
    """The ORF draws of seed `seed`: G [H, ceil(M/d), d, d] and R [H, M, d].

    Draw n of the stream is normal n % 4 of group n // 4. G[h, b, i, j] is draw
    ((h nb + b) d + i) d + j; R[h, r, j] is draw NG + (h M + r) d + j, with NG the size of G
    rounded up to a multiple of 4.
    """
    nb = -(-M // d)
    ng = H * nb * d * d
    NG = -(-ng // 4) * 4
    total = NG + H * M * d
    draws = np.empty(-(-total // 4) * 4)
    for g in range(len(draws) // 4):
        draws[4 * g:4 * g + 4] = philox_normals(seed, g)
    G = draws[:ng].reshape(H, nb, d, d)
    R = draws[NG:NG + H * M * d].reshape(H, M, d)
    return G, R


# ---------------------------------------------------------------- feature maps
def phi_trig(X: np.ndarray, Om: np.ndarray) -> np.ndarray:
    """Trigonometric softmax-kernel features [L, 2M] of the rows of X [L, d].

    [EXPL, 核心机制]: cos/sin pairs from random Fourier features. [MLMP-en, AI Executive
    Summary]: random features of the Gaussian kernel. The exp(|x|^2/2) factor turns the
    Gaussian kernel into exp(q.k).
    """
    M = Om.shape[0]
    U = X @ Om.T
    g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(M)
    return g[:, None] * np.concatenate([np.cos(U), np.sin(U)], axis=1)


def phi_relu(X: np.ndarray, Om: np.ndarray) -> np.ndarray:
    """Generalized-attention ReLU features [L, M]: max(Omega x, 0)/sqrt(M).

    [MLMP-zh, 核心创新] names generalized kernel attention (GA). The ReLU map is the GA
    kernel this library implements.
    """
    return np.maximum(X @ Om.T, 0.0) / np.sqrt(Om.shape[0])


def phi(X: np.ndarray, Om: np.ndarray, kind: int) -> np.ndarray:
    if kind == TRIG:
        return phi_trig(X, Om)
    if kind == RELU:
        return phi_relu(X, Om)
    raise ValueError(f"unknown feature kind {kind}")


def _normalise(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    out = np.zeros_like(num)
    nz = den != 0.0
    out[nz] = num[nz] / den[nz, None]
    return out


# ---------------------------------------------------------------- one head
def favor_bidirectional_head(q, k, v, Om, kind):
    """Bidirectional FAVOR for one head, in linear time.

    [EXPL, 核心机制]: aggregate S = phi(K)^T V and z = phi(K)^T 1 first, then
    out = D_hat^-1 phi(Q) S with D_hat = diag(phi(Q) z). No L x L matrix is formed.
    """
    fq = phi(q, Om, kind)
    fk = phi(k, Om, kind)
    S = fk.T @ v
    z = fk.T @ np.ones(k.shape[0])
    return _normalise(fq @ S, fq @ z)


def favor_causal_head(q, k, v, Om, kind):
    """Causal FAVOR for one head, as a sequential fp64 prefix loop.

    [EXPL, 核心机制]: the state sum_{j<=i} phi(k_j) v_j^T and its normaliser
    sum_{j<=i} phi(k_j) are accumulated in order. Row i reads the state after
    token i is added.
    """
    fq = phi(q, Om, kind)
    fk = phi(k, Om, kind)
    L, dv = v.shape
    S = np.zeros((fk.shape[1], dv))
    z = np.zeros(fk.shape[1])
    out = np.zeros((L, dv))
    for i in range(L):
        S += np.outer(fk[i], v[i])
        z += fk[i]
        den = fq[i] @ z
        if den != 0.0:
            out[i] = (fq[i] @ S) / den
    return out


def favor_explicit_head(q, k, v, Om, kind, causal, rows=None):
    """The quadratic form D_hat^-1 A_hat V with A_hat = phi(Q) phi(K)^T, for chosen rows.

    [EXPL, 核心机制]: the estimate of A whose reassociation gives the linear-time form.
    Causal keeps j <= i only.
    """
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    A = phi(q[rows], Om, kind) @ phi(k, Om, kind).T
    if causal:
        A = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], A, 0.0)
    return _normalise(A @ v, A.sum(axis=1))


def softmax_attention_head(q, k, v, causal, rows=None):
    """Exact softmax attention D^-1 A V with A = exp(q_i . k_j) ([EXPL, 核心机制]).

    The inputs carry the 1/sqrt(d) temperature. Rows are shifted by their max before
    the exponential.
    """
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    s = q[rows] @ k.T
    if causal:
        s = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    a = np.exp(s)
    return (a @ v) / a.sum(axis=1, keepdims=True)


def arccos_attention_head(q, k, v, causal, rows=None):
    """The ReLU map's M -> infinity limit: attention with the degree-1 arc-cosine kernel.

    E[relu(w.q) relu(w.k)] over w ~ N(0, I) is |q||k|(sin t + (pi - t) cos t)/(2 pi), with
    t the angle between q and k (Cho & Saul 2009). ORF rows have the same N(0, I)
    marginal. Used only to check convergence in M.
    """
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    qs = q[rows]
    nq = np.linalg.norm(qs, axis=1)[:, None]
    nk = np.linalg.norm(k, axis=1)[None, :]
    c = np.clip((qs @ k.T) / (nq * nk), -1.0, 1.0)
    t = np.arccos(c)
    A = nq * nk * (np.sin(t) + (np.pi - t) * c) / (2 * np.pi)
    if causal:
        A = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], A, 0.0)
    return _normalise(A @ v, A.sum(axis=1))


def row_diagnostics_head(q, k, v, Om, kind, causal, rows=None):
    """Cancellation diagnostics for chosen rows of the FAVOR estimate.

    kappa_i = sum_j |a_ij| / |sum_j a_ij|  (1 for the ReLU map)
    s_i     = sum_j |a_ij| * max|v_j| / |sum_j a_ij|
    a_ij = phi(q_i).phi(k_j). Causal keeps j <= i.
    """
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    A = phi(q[rows], Om, kind) @ phi(k, Om, kind).T
    if causal:
        A = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], A, 0.0)
    absA = np.abs(A)
    den = np.abs(A.sum(axis=1))
    with np.errstate(divide="ignore", invalid="ignore"):
        kappa = absA.sum(axis=1) / den
        s = (absA @ np.abs(v).max(axis=1)) / den
    return kappa, s


def row_condition_head(q, k, v, Om, kind, causal, rows=None, with_den=False):
    """Relative condition number of each chosen output row under rounding of the features.

    The method computes out_i = sum_f phi_f(q_i) S_f / sum_f phi_f(q_i) z_f with
    S_f = sum_j phi_f(k_j) v_j ([EXPL, 核心机制]). If every product phi_f(q_i) phi_f(k_j)
    carries a relative error of at most u, then to first order
        |d out_i| <= u (N_i + |out_i| D_i) / |den_i|,
    with N_i = sum_f sum_j |phi_f(q_i)| |phi_f(k_j)| |v_j| and
    D_i = sum_f sum_j |phi_f(q_i) phi_f(k_j)|. This returns
        cond_i = (max|N_i| + max|out_i| D_i) / (|den_i| max|out_i|).
    The trig map cancels across features as well as keys, so cond_i can reach 1e5 where
    kappa_i is small. Causal sums run over j <= i.

    with_den=True also returns kappa_i = D_i / |den_i|, the condition of the denominator alone.
    Past first order the same perturbations give exactly
        |d out_i| <= u (N_i + |out_i| D_i) / (|den_i| (1 - u kappa_i))   while u kappa_i < 1,
    and once u kappa_i >= 1 they can cancel den_i altogether, so no bound holds: this is the
    trig mode's occasional numerical instability that the explainer's engineering notes set
    against the stable non-negative mode ([EXPL], the paragraph on the two feature modes).
    """
    L = q.shape[0]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    fq = phi(q[rows], Om, kind)
    fk = phi(k, Om, kind)
    aq, ak, av = np.abs(fq), np.abs(fk), np.abs(v)
    if not causal:
        num = fq @ (fk.T @ v)
        den = fq @ fk.sum(axis=0)
        N = aq @ (ak.T @ av)
        D = aq @ ak.sum(axis=0)
    else:
        F, dv = fk.shape[1], v.shape[1]
        num = np.zeros((len(rows), dv))
        den = np.zeros(len(rows))
        N = np.zeros((len(rows), dv))
        D = np.zeros(len(rows))
        S, z = np.zeros((F, dv)), np.zeros(F)
        SA, zA = np.zeros((F, dv)), np.zeros(F)
        order = np.argsort(rows, kind="stable")
        pos = 0
        for j in range(L):
            S += np.outer(fk[j], v[j])
            z += fk[j]
            SA += np.outer(ak[j], av[j])
            zA += ak[j]
            while pos < len(order) and rows[order[pos]] == j:
                r = order[pos]
                num[r], den[r] = fq[r] @ S, fq[r] @ z
                N[r], D[r] = aq[r] @ SA, aq[r] @ zA
                pos += 1
            if pos == len(order):
                break
    out = _normalise(num, den)
    on = np.abs(out).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        cond = (np.abs(N).max(axis=1) + on * D) / (np.abs(den) * on)
        if not with_den:
            return cond
        return cond, D / np.abs(den)


def row_rounding_terms_head(q, k, v, Om, kind, causal, rows=None):
    """Sums of squares of the terms that each rounding level of the linear-time form touches.

    [EXPL, 核心机制] evaluates num_i = phi(q_i)^T S and den_i = phi(q_i)^T z with the state
    S = sum_j phi(k_j) v_j^T, z = sum_j phi(k_j) (j <= i when causal). Rounding in a finite
    precision enters at three levels; with independent relative errors e of mean zero and
    variance s^2 at one level, the variance of num_in is s^2 times:
      level 1, one error per (feature f, key j) (the key features):
          N1_in = sum_f sum_j (phi_f(q_i) phi_f(k_j) v_jn)^2,   D1_i = sum_f sum_j (phi_f(q_i) phi_f(k_j))^2
      level 2, one error per (query i, key j) or per (key j, column n) (values, masked products):
          N2_in = sum_j (A_ij v_jn)^2,   D2_i = sum_j A_ij^2,   A_ij = phi(q_i)^T phi(k_j)
      level 3, one error per (feature f, column n) (query features, the state):
          N3_in = sum_f (phi_f(q_i) S_fn)^2,   D3_i = sum_f (phi_f(q_i) z_f)^2
    Returns a dict of out [rows, dv], den [rows] and N1, N2, N3 [rows, dv], D1, D2, D3 [rows].
    Nothing here depends on how a kernel blocks the sums; the tests combine the levels with
    the unit roundoffs of a path's operand types (probabilistic rounding error analysis in the
    sense of Higham and Mary, SIAM J. Sci. Comput. 41(5), 2019).
    """
    L = q.shape[0]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    fq = phi(q[rows], Om, kind)
    fk = phi(k, Om, kind)
    A = fq @ fk.T
    if causal:
        A = np.where(np.arange(L)[None, :] <= rows[:, None], A, 0.0)
    t = {"N2": (A * A) @ (v * v), "D2": (A * A).sum(axis=1)}
    fq2, fk2, v2 = fq * fq, fk * fk, v * v
    if not causal:
        S, z = fk.T @ v, fk.sum(axis=0)
        num, den = fq @ S, fq @ z
        t["N1"], t["D1"] = fq2 @ (fk2.T @ v2), fq2 @ fk2.sum(axis=0)
        t["N3"], t["D3"] = fq2 @ (S * S), fq2 @ (z * z)
    else:
        F, dv = fk.shape[1], v.shape[1]
        n = len(rows)
        num, den = np.zeros((n, dv)), np.zeros(n)
        for key in ("N1", "N3"):
            t[key] = np.zeros((n, dv))
        for key in ("D1", "D3"):
            t[key] = np.zeros(n)
        S, z = np.zeros((F, dv)), np.zeros(F)
        SS, zz = np.zeros((F, dv)), np.zeros(F)
        j0 = 0                       # keys [0, j0) are in the prefix sums
        for r in np.argsort(rows, kind="stable"):
            j1 = rows[r] + 1
            if j1 > j0:
                S += fk[j0:j1].T @ v[j0:j1]
                z += fk[j0:j1].sum(axis=0)
                SS += fk2[j0:j1].T @ v2[j0:j1]
                zz += fk2[j0:j1].sum(axis=0)
                j0 = j1
            num[r], den[r] = fq[r] @ S, fq[r] @ z
            t["N1"][r], t["D1"][r] = fq2[r] @ SS, fq2[r] @ zz
            t["N3"][r], t["D3"][r] = fq2[r] @ (S * S), fq2[r] @ (z * z)
    t["out"], t["den"] = _normalise(num, den), den
    return t


def favor_rows_head(q, k, v, Om, kind, causal, rows):
    """FAVOR output rows `rows` of one head, by the linear-time form (prefix loop if causal)."""
    rows = np.asarray(rows)
    if not causal:
        fq = phi(q[rows], Om, kind)
        fk = phi(k, Om, kind)
        return _normalise(fq @ (fk.T @ v), fq @ fk.sum(axis=0))
    fq = phi(q[rows], Om, kind)
    fk = phi(k, Om, kind)
    S, z = np.zeros((fk.shape[1], v.shape[1])), np.zeros(fk.shape[1])
    out = np.zeros((len(rows), v.shape[1]))
    order = np.argsort(rows, kind="stable")
    pos = 0
    for j in range(q.shape[0]):
        S += np.outer(fk[j], v[j])
        z += fk[j]
        while pos < len(order) and rows[order[pos]] == j:
            r = order[pos]
            den = fq[r] @ z
            if den != 0.0:
                out[r] = (fq[r] @ S) / den
            pos += 1
        if pos == len(order):
            break
    return out


# ---------------------------------------------------------------- backward (gradients)
def phi_vjp(X, Om, kind, dphi):
    """Gradient with respect to X [L, d] of sum(dphi * phi(X, Om)): the feature map's
    vector-Jacobian product, row by row.

    Trig, phi = g(x) [cos u, sin u] with u = Omega x and g = exp(|x|^2/2)/sqrt(M):
        dx = x (dphi . phi) + g Omega^T (-dphi_cos * sin u + dphi_sin * cos u).
    ReLU, phi = max(u, 0)/sqrt(M):  dx = Omega^T (dphi * [u > 0]) / sqrt(M).
    """
    U = X @ Om.T
    M = Om.shape[0]
    if kind == TRIG:
        g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(M)
        dc, ds = dphi[:, :M], dphi[:, M:]
        return X * np.sum(dphi * phi_trig(X, Om), axis=1)[:, None] + g[:, None] * ((-dc * np.sin(U) + ds * np.cos(U)) @ Om)
    if kind == RELU:
        return ((dphi * (U > 0)) @ Om) / np.sqrt(M)
    raise ValueError(f"unknown feature kind {kind}")


def favor_backward_head(q, k, v, Om, kind, causal, dout):
    """Gradients (dq, dk, dv) of sum(dout * out) for one head, out = FAVOR(q, k, v).

    The definition differentiated is the quadratic form D^-1 A V with A = phi(Q) phi(K)^T
    (masked to j <= i when causal) ([EXPL, 核心机制]). The linear-time form computes the same out.
    Reverse mode:
        dN = dout / D,  dD = -(dout . out) / D            (rows with D = 0 give out = 0: no gradient)
        dA = dN V^T + dD 1^T  (masked)
        dphi(Q) = dA phi(K),  dphi(K) = dA^T phi(Q),  dV = A^T dN
    then each phi through phi_vjp. Omega is a fixed random draw and gets no gradient.
    """
    fq, fk = phi(q, Om, kind), phi(k, Om, kind)
    A = fq @ fk.T
    if causal:
        A = np.where(np.arange(k.shape[0])[None, :] <= np.arange(q.shape[0])[:, None], A, 0.0)
    N, D = A @ v, A.sum(axis=1)
    out = _normalise(N, D)
    nz = D != 0.0
    dN = np.zeros_like(N)
    dD = np.zeros_like(D)
    dN[nz] = dout[nz] / D[nz, None]
    dD[nz] = -np.sum(dout[nz] * out[nz], axis=1) / D[nz]
    dA = dN @ v.T + dD[:, None]
    if causal:
        dA = np.where(np.arange(k.shape[0])[None, :] <= np.arange(q.shape[0])[:, None], dA, 0.0)
    dq = phi_vjp(q, Om, kind, dA @ fk)
    dk = phi_vjp(k, Om, kind, dA.T @ fq)
    return dq, dk, A.T @ dN


def backward_magnitudes_head(q, k, v, Om, kind, causal, dout):
    """Rounding scales of the gradients: the reverse pass of favor_backward_head with every
    factor replaced by its absolute value (|phi|, |V|, |dout|, |out|, |1/D|, |sin|, |cos|, |x|).

    Each gradient element is a sum of products; a finite-precision evaluation of it errs by at
    most a small multiple of the unit roundoff times the sum of the products' absolute values,
    which is what this returns (dq_abs, dk_abs, dv_abs). A gradient that cancels (row 0 of a
    causal head has dq = 0 exactly, its output being v_0 whatever q_0 is) keeps a non-zero
    scale here.
    """
    fq, fk = np.abs(phi(q, Om, kind)), np.abs(phi(k, Om, kind))
    A = fq @ fk.T
    Aphi = phi(q, Om, kind) @ phi(k, Om, kind).T
    if causal:
        mask = np.arange(k.shape[0])[None, :] <= np.arange(q.shape[0])[:, None]
        A, Aphi = np.where(mask, A, 0.0), np.where(mask, Aphi, 0.0)
    D = Aphi.sum(axis=1)
    out = _normalise(Aphi @ v, D)
    nz = D != 0.0
    dN = np.zeros((q.shape[0], v.shape[1]))
    dD = np.zeros(q.shape[0])
    dN[nz] = np.abs(dout[nz]) / np.abs(D[nz, None])
    dD[nz] = np.sum(np.abs(dout[nz] * out[nz]), axis=1) / np.abs(D[nz])
    dA = dN @ np.abs(v).T + dD[:, None]
    if causal:
        dA = np.where(mask, dA, 0.0)

    def jac_abs(X, dphi):
        U = X @ Om.T
        M = Om.shape[0]
        aO = np.abs(Om)
        if kind == TRIG:
            g = np.exp(0.5 * np.sum(X * X, axis=1)) / np.sqrt(M)
            dc, ds = dphi[:, :M], dphi[:, M:]
            radial = np.abs(X) * np.sum(dphi * np.abs(phi_trig(X, Om)), axis=1)[:, None]
            return radial + g[:, None] * ((dc * np.abs(np.sin(U)) + ds * np.abs(np.cos(U))) @ aO)
        return ((dphi * (U > 0)) @ aO) / np.sqrt(M)

    return jac_abs(q, dA @ fk), jac_abs(k, dA.T @ fq), A.T @ dN


def favor_backward(Q, K, V, Om, kind, causal, dO):
    """favor_backward_head over [B, H, L, d]: returns (dQ, dK, dV)."""
    B, H = Q.shape[:2]
    res = [np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)]
    for b in range(B):
        for h in range(H):
            g = favor_backward_head(Q[b, h], K[b, h], V[b, h], Om[h], kind, causal, dO[b, h])
            for r, x in zip(res, g):
                r[b, h] = x
    return tuple(res)


# ---------------------------------------------------------------- decode: one token per call
def favor_decode_state(M, dv, kind):
    """An empty carried state (S [F, dv], z [F]) for one head; F = 2M (trig) or M (ReLU)."""
    F = 2 * M if kind == TRIG else M
    return np.zeros((F, dv)), np.zeros(F)


def favor_decode_step_head(S, z, q, k, v, Om, kind):
    """One causal step for one head with a carried state. S and z are updated in place.

    [EXPL, 核心机制]: the causal prefix sum of phi(k_j) v_j^T (and of phi(k_j) for the
    normaliser) over j <= i, read by phi(q_i). Token i's key and value enter the state
    before its query reads it, so starting from an empty state the i-th call returns
    causal row i.
    """
    fk = phi(k[None, :], Om, kind)[0]
    fq = phi(q[None, :], Om, kind)[0]
    S += np.outer(fk, v)
    z += fk
    den = fq @ z
    return (fq @ S) / den if den != 0.0 else np.zeros(v.shape[0])


# ---------------------------------------------------------------- [B, H, L, d] wrappers
def _per_head(fn, Q, K, V, Om, *args, **kw):
    B, H = Q.shape[:2]
    out = None
    for b in range(B):
        for h in range(H):
            o = fn(Q[b, h], K[b, h], V[b, h], Om[h], *args, **kw)
            if out is None:
                out = np.zeros((B, H) + o.shape)
            out[b, h] = o
    return out


def favor_attention(Q, K, V, Om, kind, causal):
    """FAVOR forward for Q, K, V [B, H, L, d] and Omega [H, M, d] (fp64 arrays)."""
    fn = favor_causal_head if causal else favor_bidirectional_head
    return _per_head(fn, Q, K, V, Om, kind)


def favor_explicit(Q, K, V, Om, kind, causal, rows=None):
    return _per_head(favor_explicit_head, Q, K, V, Om, kind, causal, rows)


def softmax_attention(Q, K, V, causal, rows=None):
    B, H = Q.shape[:2]
    return np.stack([np.stack([softmax_attention_head(Q[b, h], K[b, h], V[b, h], causal, rows)
                               for h in range(H)]) for b in range(B)])


def row_diagnostics(Q, K, V, Om, kind, causal, rows=None):
    B, H = Q.shape[:2]
    kap, s = [], []
    for b in range(B):
        for h in range(H):
            a, c = row_diagnostics_head(Q[b, h], K[b, h], V[b, h], Om[h], kind, causal, rows)
            kap.append(a)
            s.append(c)
    L_rows = kap[0].shape[0]
    return np.stack(kap).reshape(B, H, L_rows), np.stack(s).reshape(B, H, L_rows)


def row_condition(Q, K, V, Om, kind, causal, rows=None):
    B, H = Q.shape[:2]
    return np.stack([np.stack([row_condition_head(Q[b, h], K[b, h], V[b, h], Om[h], kind, causal, rows)
                               for h in range(H)]) for b in range(B)])
