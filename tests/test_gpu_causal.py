"""bf16 tensor-core path, causal: CUDA output vs the fp64 oracle on the same inputs.

The causal kernel splits the features of a head over a cluster of G CTAs of 64 angles each
(G = 1, 2, 4, 8) and scans 128-token chunks. Sizes cover one and many chunks, ragged tails, each cluster size, both
feature maps, padded feature counts, heavy-norm keys (the stabiliser's per-row references),
the bench workload and a 65536-token sequence.
"""
import numpy as np
import pytest

import favor_inputs as fi
from cases import Case
from parity_util import TOL_BF16, U_CAUSAL16, check_rows

pytestmark = pytest.mark.gpu


def _run(case, kind, chunk=0):
    import linear_kernelized_attention_b200 as F
    q, k, v, om = case.device()
    out = F.favor_attention(q, k, v, om, feature_kind=kind, causal=True, chunk=chunk)
    assert F.favor_sync_status() == 0
    return fi.as_f64(out)


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("B,H,L,M", [
    (1, 1, 1, 64),         # a single token
    (1, 2, 300, 64),       # 3 chunks, ragged tail; G = 1
    (1, 1, 129, 16),       # a full chunk + 1 token, 16 features (padded angles)
    (2, 3, 1000, 256),     # 8 chunks; G = 4
    (1, 4, 127, 128),      # one ragged chunk; G = 2
    (1, 1, 400, 192),      # 3 blocks round up to G = 4 with a padded block
])
def test_causal_small(kind, B, H, L, M):
    c = Case(B, H, L, 64, M, seed=B * 100 + L + M + 7)
    g = _run(c, kind).reshape(B * H, L, 64)
    ref, cond, _ = c.oracle(kind, True)
    check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, f"causal kind={kind} {B}x{H}x{L} M={M}", trig=kind == 0)


def test_causal_relu_512_features():
    # ReLU M = 512: G = 8 CTAs of 64 features (16-row ownership blocks, one per CTA)
    c = Case(1, 2, 640, 64, 512, seed=11)
    g = _run(c, 1).reshape(2, 640, 64)
    ref, cond, _ = c.oracle(1, True)
    check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, "causal relu M=512", trig=False)


def test_causal_relu_384_features():
    # ReLU M = 384: 6 blocks of 64 angles rounded up to G = 8 (two blocks are all padding)
    c = Case(1, 2, 300, 64, 384, seed=12)
    g = _run(c, 1).reshape(2, 300, 64)
    ref, cond, _ = c.oracle(1, True)
    check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, "causal relu M=384", trig=False)


@pytest.mark.parametrize("kind", [0, 1])
def test_causal_more_heads_than_sms(kind):
    # B*H = 160 heads, 2 CTAs each: several waves of clusters
    c = Case(2, 80, 200, 64, 128, seed=13)
    g = _run(c, kind).reshape(160, 200, 64)
    heads = [(0, 0), (0, 79), (1, 40), (1, 79)]
    ref, cond, _ = c.oracle(kind, True, heads=heads)
    sel = np.stack([g[b * 80 + h] for b, h in heads])
    check_rows(sel, ref, cond, TOL_BF16, U_CAUSAL16, f"causal many heads kind={kind}", trig=kind == 0)


def test_causal_first_row_is_v0():
    # row 0 attends to key 0 only, so out_0 = v_0 for either map (non-zero denominator)
    c = Case(1, 2, 256, 64, 128, seed=21)
    for kind in (0, 1):
        g = _run(c, kind).reshape(2, 256, 64)
        np.testing.assert_allclose(g[:, 0], c.v[0, :, 0], rtol=2e-2, atol=2e-2 * np.abs(c.v[0, :, 0]).max())


@pytest.mark.parametrize("kind", [0, 1])
def test_causal_bench_workload(kind):
    # the bench configuration B=4, H=8, L=4096, d=64, M=256, every row
    c = Case(4, 8, 4096, 64, 256, seed=0)
    g = _run(c, kind).reshape(32, 4096, 64)
    ref, cond, _ = c.oracle(kind, True)
    st = check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, f"causal bench kind={kind}", trig=kind == 0)
    print(st)


def test_causal_heavy_norm_decoder():
    # B=2, H=8, L=8192, d=64, M=128, trig, 5% of rows scaled by 4: sampled rows of two heads
    c = Case(2, 8, 8192, 64, 128, seed=4, heavy=0.05)
    g = _run(c, 0).reshape(16, 8192, 64)
    rows = fi.sample_rows(8192, 512, seed=4)
    heads = [(0, 0), (1, 7)]
    ref, cond, _ = c.oracle(0, True, heads=heads, rows=rows)
    sel = np.stack([g[b * 8 + h][rows] for b, h in heads])
    st = check_rows(sel, ref, cond, TOL_BF16, U_CAUSAL16, "causal heavy-norm")
    print(st)


def test_causal_key_norm_jump_inside_a_chunk():
    # keys far above everything before them, in the middle of chunks: the rows before such a
    # key in its chunk keep their own reference, the rows after it take the new one
    c = Case(1, 1, 1024, 64, 128, seed=3)
    k = c.t[1].float()
    k[0, 0, 200, :] *= 6.0
    k[0, 0, 700, :] *= 4.0
    k[0, 0, 701, :] *= 7.0
    c.t[1] = k.to(c.t[1].dtype)
    c.k = fi.as_f64(c.t[1])
    c._dev = None
    g = _run(c, 0).reshape(1, 1024, 64)
    ref, cond, _ = c.oracle(0, True)
    check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, "causal norm jump")


def test_causal_constant_v_and_zero_queries():
    import torch
    c = Case(1, 2, 500, 64, 256, seed=5)
    val = torch.linspace(-1, 1, 64).to(torch.bfloat16)
    c.t[2] = val.expand(1, 2, 500, 64).contiguous()
    c.v = fi.as_f64(c.t[2])
    c._dev = None
    for kind in (0, 1):
        g = _run(c, kind).reshape(2, 500, 64)
        ref, cond, _ = c.oracle(kind, True)
        check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, f"causal constant v kind={kind}", trig=kind == 0)
    # ReLU with q = 0: every query feature is 0, the denominator is 0 and the row is 0
    c.t[0] = torch.zeros_like(c.t[0])
    c._dev = None
    assert np.all(_run(c, 1) == 0.0)


def test_causal_long_sequence_sampled_rows():
    # B=1, H=16, L=65536 trig: 512 sampled rows of the first and last head
    c = Case(1, 16, 65536, 64, 256, seed=0)
    g = _run(c, 0).reshape(16, 65536, 64)
    rows = fi.sample_rows(65536, 512, seed=0)
    heads = [(0, 0), (0, 15)]
    ref, cond, _ = c.oracle(0, True, heads=heads, rows=rows)
    sel = np.stack([g[h][rows] for _, h in heads])
    check_rows(sel, ref, cond, TOL_BF16, U_CAUSAL16, "causal L=65536 sampled")


def test_causal_chunk_argument():
    import linear_kernelized_attention_b200 as F
    c = Case(1, 1, 300, 64, 64, seed=9)
    a = _run(c, 0, chunk=0)
    b = _run(c, 0, chunk=128)
    assert np.array_equal(a, b)
    q, k, v, om = c.device()
    with pytest.raises(F.FavorError) as e:
        F.favor_attention(q, k, v, om, feature_kind=0, causal=True, chunk=64)
    assert e.value.code == -5


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("d,M", [(16, 32), (32, 96), (16, 256)])
def test_causal_head_sizes(kind, d, M):
    # head sizes 16 and 32 ride in the 64-column boxes: zeros past d, d values stored per row
    B, H, L = 2, 2, 600
    c = Case(B, H, L, d, M, seed=d * 5 + M)
    g = _run(c, kind).reshape(B * H, L, d)
    ref, cond, _ = c.oracle(kind, True)
    check_rows(g, ref, cond, TOL_BF16, U_CAUSAL16, f"causal d={d} M={M} kind={kind}", trig=kind == 0)
