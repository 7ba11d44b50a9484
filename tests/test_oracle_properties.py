"""Property tests of the oracle over random small shapes (hypothesis), complementing the fixed
cases of test_oracle_pins.py: each draws the shape and the seed, then checks a fact that the
definitions fix (no value from the CUDA path is involved)."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import favor_oracle as O

SETTINGS = settings(max_examples=25, deadline=None)


def _inputs(L, d, M, seed):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((L, d)) * 0.4 for _ in range(3))
    nb = -(-M // d)
    om = O.orf_matrix(rng.standard_normal((nb, d, d)), rng.standard_normal((M, d)), M)
    return q, k, v, om


@SETTINGS
@given(L=st.integers(1, 24), d=st.integers(1, 6), M=st.integers(1, 12), kind=st.sampled_from([O.TRIG, O.RELU]),
       seed=st.integers(0, 2**31 - 1))
def test_decode_calls_equal_causal_rows(L, d, M, kind, seed):
    q, k, v, om = _inputs(L, d, M, seed)
    S, z = O.favor_decode_state(M, d, kind)
    rows = np.stack([O.favor_decode_step_head(S, z, q[i], k[i], v[i], om, kind) for i in range(L)])
    ref = O.favor_explicit_head(q, k, v, om, kind, causal=True)
    np.testing.assert_allclose(rows, ref, rtol=1e-8, atol=1e-10 * max(1.0, np.abs(ref).max()))


@SETTINGS
@given(L=st.integers(2, 8), d=st.integers(1, 4), M=st.integers(1, 6), kind=st.sampled_from([O.TRIG, O.RELU]),
       causal=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_backward_equals_central_differences(L, d, M, kind, causal, seed):
    q, k, v, om = _inputs(L, d, M, seed)
    dout = np.random.default_rng(seed + 1).standard_normal((L, d))
    fq, fk = O.phi(q, om, kind), O.phi(k, om, kind)
    A = fq @ fk.T
    if causal:
        A = np.tril(A)
    # keep away from vanishing denominators and from ReLU kinks, where differences are ill-posed
    if np.any(np.abs(A.sum(axis=1)) < 1e-3) or (kind == O.RELU and np.any(np.abs(np.concatenate([q, k]) @ om.T) < 1e-3)):
        return
    g = O.favor_backward_head(q, k, v, om, kind, causal, dout)
    h = 1e-6
    for which in range(3):
        x = (q, k, v)[which]
        idx = tuple(np.random.default_rng(seed + 2 + which).integers(0, s) for s in x.shape)
        args_p, args_m = [q.copy(), k.copy(), v.copy()], [q.copy(), k.copy(), v.copy()]
        args_p[which][idx] += h
        args_m[which][idx] -= h
        lp = np.sum(dout * O.favor_explicit_head(*args_p, om, kind, causal))
        lm = np.sum(dout * O.favor_explicit_head(*args_m, om, kind, causal))
        fd = (lp - lm) / (2 * h)
        scale = max(1.0, np.abs(g[which]).max())
        assert abs(g[which][idx] - fd) <= 1e-5 * scale


@SETTINGS
@given(key=st.integers(0, 2**128 - 1), counter=st.integers(0, 2**256 - 8))
def test_philox_equals_numpy_bit_generator(key, counter):
    raw = np.random.Philox(key=key, counter=counter).random_raw(8)
    mine = []
    for i in range(2):
        c = counter + 1 + i
        mine += O.philox4x64_10([(c >> (64 * w)) & (2**64 - 1) for w in range(4)],
                                [(key >> (64 * w)) & (2**64 - 1) for w in range(2)])
    assert [int(x) for x in raw] == mine


@SETTINGS
@given(M=st.integers(1, 40), d=st.integers(1, 12), seed=st.integers(0, 2**31 - 1))
def test_orf_blocks_are_orthogonal_with_chi_lengths(M, d, seed):
    G, R = O.seeded_orf_gaussians(seed, 1, M, d)
    om = O.orf_matrix(G[0], R[0], M)
    lengths = np.linalg.norm(om, axis=1)
    np.testing.assert_allclose(lengths, np.linalg.norm(R[0], axis=1), rtol=1e-12)
    for b in range(0, M, d):
        blk = om[b:b + d] / lengths[b:b + d, None]
        np.testing.assert_allclose(blk @ blk.T, np.eye(blk.shape[0]), atol=1e-10)
