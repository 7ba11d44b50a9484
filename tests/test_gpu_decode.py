"""Causal decode step (one token per head per call, carried fp32 state) vs the fp64 oracle.

Calls on tokens 0 .. L-1 from an empty state must return the oracle's causal rows 0 .. L-1,
and the state after them must equal the oracle's prefix sums (descaled by the stored
stabiliser reference). The decode arithmetic is fp32 with bf16 inputs and a bf16 output, so
the row tolerance is the output rounding with headroom: 5e-3 of the row's max. The cond branch
uses u = 2^-16: fp32 roundoff 2^-24 times up to 256 accumulated roundings (the sequential
state sums and the angle roundings).
"""
import math

import numpy as np
import pytest

import favor_inputs as fi
from cases import Case
from oracle import favor_oracle as O
from parity_util import TOL_BF16, U_CAUSAL16, check_rows

pytestmark = pytest.mark.gpu

TOL_DEC, U_DEC = 5e-3, 2.0 ** -16


def _decode_all(case, kind):
    """Run L decode calls; returns (rows [B*H, L, d] fp64, state tensor)."""
    import torch
    import linear_kernelized_attention_b200 as F
    q, k, v, om = case.device()
    B, H, L, d, M = case.B, case.H, case.L, case.d, case.M
    qt, kt, vt = (x.permute(2, 0, 1, 3).contiguous() for x in (q, k, v))   # [L, B, H, d]
    st = F.favor_decode_new_state(B, H, d, M, kind)
    outs = torch.empty_like(qt)
    for t in range(L):
        F.favor_decode_step(qt[t], kt[t], vt[t], om, st, out=outs[t], feature_kind=kind)
    assert F.favor_sync_status() == 0
    rows = fi.as_f64(outs.permute(1, 2, 0, 3).reshape(B * H, L, d))
    return rows, st


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("B,H,L,d,M", [
    (1, 1, 1, 64, 64),       # a single token: the row is v_0
    (1, 2, 300, 64, 64),     # cluster of 2 per head
    (2, 3, 200, 64, 256),    # cluster of 8 per head, 32 angles each
    (1, 2, 120, 32, 71),     # ragged last angle slice (36 + 35)
    (1, 1, 100, 128, 512),   # d = 128, the largest trig state (1024 rows)
    (1, 3, 150, 16, 40),     # d = 16, one CTA per head
])
def test_decode_matches_causal_oracle(kind, B, H, L, d, M):
    c = Case(B, H, L, d, M, seed=B * 7 + L + M + d)
    g, _ = _decode_all(c, kind)
    ref, cond, _ = c.oracle(kind, True)
    st = check_rows(g.reshape(B * H, L, d), ref.reshape(B * H, L, d), cond.reshape(B * H, L),
                    TOL_DEC, U_DEC, f"decode kind={kind} {B}x{H}x{L} d={d} M={M}", trig=kind == 0, headroom=1.0)
    print(st)


def test_decode_relu_1024_features():
    c = Case(1, 1, 64, 32, 1024, seed=31)
    g, _ = _decode_all(c, 1)
    ref, cond, _ = c.oracle(1, True)
    check_rows(g, ref, cond, TOL_DEC, U_DEC, "decode relu M=1024", trig=False)


@pytest.mark.parametrize("kind", [0, 1])
def test_decode_many_heads(kind):
    # B*H = 512 heads: one CTA per head, several CTAs per SM
    c = Case(64, 8, 24, 64, 256, seed=41)
    g, _ = _decode_all(c, kind)
    heads = [(0, 0), (17, 3), (63, 7)]
    ref, cond, _ = c.oracle(kind, True, heads=heads)
    sel = np.stack([g[b * 8 + h] for b, h in heads])
    check_rows(sel, ref, cond, TOL_DEC, U_DEC, f"decode many heads kind={kind}", trig=kind == 0, headroom=1.0)


def test_decode_state_matches_oracle_prefix_sums():
    # after L calls: S = e^c / sqrt(M) * S_stored (trig), S_stored / sqrt(M) (ReLU), same for z
    import linear_kernelized_attention_b200 as F
    B, H, L, d, M = 1, 2, 160, 64, 128
    c = Case(B, H, L, d, M, seed=51)
    for kind in (0, 1):
        _, st = _decode_all(c, kind)
        S, z, cref = (fi.as_f64(x.cpu()) for x in F.favor_decode_state_views(st, B, H, d, M, kind))
        for h in range(H):
            q, k, v, om = c.q[0, h], c.k[0, h], c.v[0, h], c.om[h]
            So, zo = O.favor_decode_state(M, d, kind)
            for t in range(L):
                O.favor_decode_step_head(So, zo, q[t], k[t], v[t], om, kind)
            scale = (math.exp(cref[h]) if kind == 0 else 1.0) / math.sqrt(M)
            fk = np.abs(O.phi(k, om, kind))
            magS = fk.T @ np.abs(v)               # sum_j |phi(k_j)| |v_j|, elementwise
            magz = fk.sum(axis=0)
            assert np.all(np.abs(S[h] * scale - So) <= 2e-5 * magS + 1e-30), f"S kind={kind} h={h}"
            assert np.all(np.abs(z[h] * scale - zo) <= 2e-5 * magz + 1e-30), f"z kind={kind} h={h}"
            if kind == 0:
                assert cref[h] == pytest.approx(0.5 * np.max(np.sum(k * k, axis=1)), rel=1e-5)
            else:
                assert cref[h] == -np.inf


def test_decode_key_norm_jumps():
    # keys far above everything before them: the stored state is rescaled by exp(c_old - c_new)
    c = Case(1, 1, 400, 64, 128, seed=3)
    k = c.t[1].float()
    k[0, 0, 50, :] *= 6.0
    k[0, 0, 200, :] *= 4.0
    k[0, 0, 201, :] *= 7.0
    c.t[1] = k.to(c.t[1].dtype)
    c.k = fi.as_f64(c.t[1])
    c._dev = None
    g, _ = _decode_all(c, 0)
    ref, cond, _ = c.oracle(0, True)
    check_rows(g, ref, cond, TOL_DEC, U_DEC, "decode norm jumps", headroom=1.0)


def test_decode_matches_tensor_core_causal_path():
    # the decode rows and the chunked tensor-core kernel's rows agree with each other
    import linear_kernelized_attention_b200 as F
    c = Case(2, 4, 260, 64, 256, seed=61)
    q, k, v, om = c.device()
    for kind in (0, 1):
        g, _ = _decode_all(c, kind)
        p = fi.as_f64(F.favor_attention(q, k, v, om, feature_kind=kind, causal=True)).reshape(8, 260, 64)
        ref, cond, _ = c.oracle(kind, True)
        check_rows(g, ref, cond, TOL_DEC, U_DEC, "decode", trig=kind == 0, headroom=1.0)
        check_rows(p, ref, cond, TOL_BF16, U_CAUSAL16, "chunked", trig=kind == 0)


def test_decode_zero_query_relu_and_reinit():
    import torch
    import linear_kernelized_attention_b200 as F
    c = Case(1, 2, 30, 64, 64, seed=71)
    q, k, v, om = c.device()
    st = F.favor_decode_new_state(1, 2, 64, 64, 1)
    z = torch.zeros_like(q[:, :, 0].contiguous())
    for t in range(5):
        o = F.favor_decode_step(z, k[:, :, t].contiguous(), v[:, :, t].contiguous(), om, st, feature_kind=1)
        assert torch.all(o == 0)
    # re-initialising gives a fresh sequence: the first row is that token's v
    F.favor_decode_init(st, 1, 2, 64, 64, 1)
    o = F.favor_decode_step(q[:, :, 7].contiguous(), k[:, :, 7].contiguous(), v[:, :, 7].contiguous(), om, st,
                            feature_kind=1)
    assert F.favor_sync_status() == 0
    np.testing.assert_allclose(fi.as_f64(o)[0], c.v[0, :, 7], rtol=5e-3, atol=5e-3 * np.abs(c.v[0, :, 7]).max())


def test_decode_rejects_unsupported_on_device():
    import torch
    import linear_kernelized_attention_b200 as F
    x = torch.zeros(1, 1, 48, dtype=torch.bfloat16, device="cuda")
    om = torch.zeros(1, 64, 48, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    with pytest.raises(F.FavorError) as e:
        F.favor_decode_step(x, x, x, om, st, feature_kind=0)
    assert e.value.code == -5
