"""bf16 tensor-core path, bidirectional: CUDA output vs the fp64 oracle on the same inputs.

Sizes span several 128-token tiles with ragged tails, cluster sizes P = 1 .. 8, both feature
maps, padded feature counts, and the full bench workload (B=4, H=8, L=4096, d=64, M=256).
"""
import numpy as np
import pytest

import favor_inputs as fi
from cases import Case
from parity_util import TOL_BF16, U_BIDIR16, check_rows

pytestmark = pytest.mark.gpu


def _run(case, kind, causal=False):
    import torch
    import linear_kernelized_attention_b200 as F
    q, k, v, om = case.device()
    out = F.favor_attention(q, k, v, om, feature_kind=kind, causal=causal)
    assert F.favor_sync_status() == 0
    return fi.as_f64(out)


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("B,H,L,M", [
    (2, 3, 1000, 256),     # 8 tiles, ragged tail of 104; P = 8
    (1, 2, 300, 64),       # 3 tiles, M padded to 128
    (1, 1, 129, 16),       # one full tile + 1 token, 16 features
    (1, 1, 1, 128),        # a single token
    (1, 4, 127, 256),      # one ragged tile per head: P = 1
])
def test_bidir_small(kind, B, H, L, M):
    c = Case(B, H, L, 64, M, seed=B * 100 + L + M)
    g = _run(c, kind).reshape(B * H, L, 64)
    ref, cond, _ = c.oracle(kind, False)
    check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, f"kind={kind} {B}x{H}x{L} M={M}", trig=kind == 0)


@pytest.mark.parametrize("kind", [0, 1])
def test_bidir_many_heads_single_cta_per_head(kind):
    # B*H = 160 > SM count: one CTA per head, no cross-CTA reduction
    c = Case(2, 80, 200, 64, 128, seed=7)
    g = _run(c, kind).reshape(160, 200, 64)
    heads = [(0, 0), (0, 79), (1, 40), (1, 79)]
    ref, cond, _ = c.oracle(kind, False, heads=heads)
    sel = np.stack([g[b * 80 + h] for b, h in heads])
    check_rows(sel, ref, cond, TOL_BF16, U_BIDIR16, f"many heads kind={kind}", trig=kind == 0)


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("B,H,L", [(4, 64, 128), (2, 128, 256), (1, 30, 384)])
def test_bidir_runs_crossing_many_short_pairs(kind, B, H, L):
    # one to three tiles per (head, angle block) pair and up to seven tiles per CTA run, so runs
    # cross several pair boundaries and a feature group can hold no item of a pair; every row of
    # every head is checked
    c = Case(B, H, L, 64, 256, seed=B * 7 + H + L)
    g = _run(c, kind).reshape(B * H, L, 64)
    ref, cond, _ = c.oracle(kind, False)
    check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, f"short pairs kind={kind} {B}x{H}x{L}", trig=kind == 0)


def test_bidir_protein_mlm_shape_trig():
    # B=8, H=8, L=1024, d=64, M=256 trig: every row of every head
    c = Case(8, 8, 1024, 64, 256, seed=0)
    g = _run(c, 0).reshape(64, 1024, 64)
    ref, cond, _ = c.oracle(0, False)
    st = check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, "B8 H8 L1024 trig")
    print(st)


@pytest.mark.parametrize("kind", [0, 1])
def test_bidir_bench_workload(kind):
    # the bench configuration B=4, H=8, L=4096, d=64, M=256, every row
    c = Case(4, 8, 4096, 64, 256, seed=0)
    g = _run(c, kind).reshape(32, 4096, 64)
    ref, cond, _ = c.oracle(kind, False)
    st = check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, f"bench kind={kind}", trig=kind == 0)
    print(st)


def test_bidir_stabiliser_rescale():
    # a key in the last tile with |k|^2/2 far above the first tile's forces the running
    # reference up mid-stream, so the accumulated state is rescaled in TMEM
    c = Case(1, 1, 1024, 64, 128, seed=3)
    k = c.t[1].float()
    k[0, 0, 1000, :] *= 6.0
    k[0, 0, 700, :] *= 4.0
    c.t[1] = k.to(c.t[1].dtype)
    c.k = fi.as_f64(c.t[1])
    c._dev = None
    g = _run(c, 0).reshape(1, 1024, 64)
    ref, cond, _ = c.oracle(0, False)
    check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, "rescale")


def test_bidir_constant_v_and_zero_queries():
    import torch
    c = Case(1, 2, 500, 64, 256, seed=5)
    val = torch.linspace(-1, 1, 64).to(torch.bfloat16)
    c.t[2] = val.expand(1, 2, 500, 64).contiguous()
    c.v = fi.as_f64(c.t[2])
    c._dev = None
    for kind in (0, 1):
        g = _run(c, kind).reshape(2, 500, 64)
        ref, cond, _ = c.oracle(kind, False)
        # the exact answer is the constant row; trig rows with heavy cancellation get the
        # condition-aware allowance like every other parity check
        np.testing.assert_allclose(ref, np.broadcast_to(fi.as_f64(val), ref.shape), rtol=1e-9, atol=1e-9)
        check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, f"constant v kind={kind}", trig=kind == 0)
    # ReLU with q = 0: every feature of q is 0, so the denominator is 0 and the row is 0
    c.t[0] = torch.zeros_like(c.t[0])
    c._dev = None
    g = _run(c, 1)
    assert np.all(g == 0.0)


def test_bidir_long_sequence_sampled_rows():
    # B=1, H=16, L=65536 trig: 512 sampled rows of the first and last head
    c = Case(1, 16, 65536, 64, 256, seed=0)
    g = _run(c, 0).reshape(16, 65536, 64)
    rows = fi.sample_rows(65536, 512, seed=0)
    heads = [(0, 0), (0, 15)]
    ref, cond, _ = c.oracle(0, False, heads=heads, rows=rows)
    sel = np.stack([g[h][rows] for _, h in heads])
    check_rows(sel, ref, cond, TOL_BF16, U_BIDIR16, "L=65536 sampled")


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("d,M", [(16, 32), (32, 96), (128, 128), (16, 256), (128, 40)])
def test_bidir_head_sizes(kind, d, M):
    # head sizes 16 and 32 ride in the 64-column box (zeros past d, stores clipped); 128 takes two
    # boxes. Several tiles with a ragged tail, two heads per batch entry, padded angle blocks.
    B, H, L = 2, 2, 700
    c = Case(B, H, L, d, M, seed=d * 7 + M)
    g = _run(c, kind).reshape(B * H, L, d)
    ref, cond, _ = c.oracle(kind, False)
    check_rows(g, ref, cond, TOL_BF16, U_BIDIR16, f"d={d} M={M} kind={kind}", trig=kind == 0)


def test_bidir_unsupported_shapes_are_refused():
    import torch
    import linear_kernelized_attention_b200 as F
    # beyond every kernel: d > 128, or M > 512. (d = 128 with trig M = 256, whose state image and
    # operand tiles do not fit one CTA's shared memory, and d = 48 take the CUDA-core route.)
    for (d, M, kind) in ((136, 64, 0), (64, 528, 1)):
        q = torch.zeros((1, 1, 128, d), dtype=torch.bfloat16, device="cuda")
        om = torch.zeros((1, M, d), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(F.FavorError) as e:
            F.favor_attention(q, q, q, om, feature_kind=kind)
        assert e.value.code == -5
