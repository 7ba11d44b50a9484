"""ORF redrawn on the device from a seed vs the oracle's Philox4x64-10 draws.

The raw generator must agree bit for bit. The Gaussians go through double log, sqrt and
sin/cos on both sides, whose last-bit rounding may differ between CUDA and the host library:
they must agree to 1e-13 relative. Omega is then Gram-Schmidt in fp64 on both sides and is
compared after the output rounding (fp32: 2 ulp of the row's max; bf16: 1 ulp).
"""
import numpy as np
import pytest

from oracle import favor_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,first", [(0, 0), (5, 1), (2**64 - 1, 2**64 - 7), (0x243F6A8885A308D3, 123456789)])
def test_philox_raw_is_bit_exact(key, first):
    import linear_kernelized_attention_b200 as F
    n = 64
    got = F.favor_philox4x64(key, first, n).cpu().numpy().view(np.uint64)
    want = np.array([O.philox4x64_10([(first + i) % 2**64, 0, 0, 0], [key, 0]) for i in range(n)], dtype=np.uint64)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("seed,H,M,d", [(1, 2, 72, 16), (2**40 + 7, 3, 256, 64), (3, 1, 130, 128)])
def test_seeded_gaussians_match_oracle(seed, H, M, d):
    import linear_kernelized_attention_b200 as F
    G, R = F.favor_orf_gaussians_seeded(seed, H, M, d)
    Go, Ro = O.seeded_orf_gaussians(seed, H, M, d)
    np.testing.assert_allclose(G.cpu().numpy(), Go, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(R.cpu().numpy(), Ro, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed,H,M,d", [(1, 2, 72, 16), (2**40 + 7, 3, 256, 64), (3, 1, 130, 128)])
def test_seeded_omega_matches_oracle_and_the_explicit_path(seed, H, M, d):
    import torch
    import linear_kernelized_attention_b200 as F
    Go, Ro = O.seeded_orf_gaussians(seed, H, M, d)
    ref = O.orf_matrices(Go, Ro, M)
    om32 = F.favor_orf_omega_seeded(seed, H, M, d, dtype=torch.float32)
    got = om32.cpu().numpy().astype(np.float64)
    scale = np.abs(ref).max(axis=2, keepdims=True)
    assert np.all(np.abs(got - ref) <= 2 * 2.0 ** -24 * scale + 1e-30)
    # the seeded kernel draws exactly what favor_orf_gaussians_seeded writes out
    G, R = F.favor_orf_gaussians_seeded(seed, H, M, d)
    for dt in (torch.float32, torch.bfloat16):
        a = F.favor_orf_omega_seeded(seed, H, M, d, dtype=dt)
        b = F.favor_orf_omega(G, R, M, dtype=dt)
        assert torch.equal(a, b)
    omb = F.favor_orf_omega_seeded(seed, H, M, d, dtype=torch.bfloat16).float().cpu().numpy()
    assert np.all(np.abs(omb - ref) <= 2.0 ** -8 * scale)


def test_seed_redraws():
    import torch
    import linear_kernelized_attention_b200 as F
    a = F.favor_orf_omega_seeded(10, 2, 128, 64, dtype=torch.float32)
    b = F.favor_orf_omega_seeded(11, 2, 128, 64, dtype=torch.float32)
    c = F.favor_orf_omega_seeded(10, 2, 128, 64, dtype=torch.float32)
    assert torch.equal(a, c) and not torch.allclose(a, b)
    # rows of one d x d block are orthogonal, with chi_d lengths (about sqrt(d))
    w = a[0, :64].double()
    n = w.norm(dim=1)
    gram = (w / n[:, None]) @ (w / n[:, None]).T
    assert torch.allclose(gram, torch.eye(64, dtype=torch.float64, device=gram.device), atol=1e-5)
    assert 5.0 < float(n.mean()) < 11.0
    assert F.favor_sync_status() == 0


def test_seeded_omega_drives_attention():
    # a seeded Omega feeds the bf16 path like any other Omega
    import torch
    import favor_inputs as fi
    import linear_kernelized_attention_b200 as F
    from parity_util import TOL_BF16, U_CAUSAL16, RowCond, check_rows
    B, H, L, d, M = 1, 2, 300, 64, 128
    om = F.favor_orf_omega_seeded(77, H, M, d, dtype=torch.bfloat16)
    q, k, v = (fi.round_to(x, "bf16") for x in fi.qkv(B, H, L, d, seed=3))
    out = F.favor_attention(q.cuda(), k.cuda(), v.cuda(), om, feature_kind=0, causal=True)
    Q, K, V, OM = fi.as_f64(q), fi.as_f64(k), fi.as_f64(v), fi.as_f64(om.cpu())
    for h in range(H):
        ref = O.favor_causal_head(Q[0, h], K[0, h], V[0, h], OM[h], O.TRIG)
        a = (Q[0, h], K[0, h], V[0, h], OM[h], O.TRIG, True)
        cond, kden = O.row_condition_head(*a, with_den=True)
        t = O.row_rounding_terms_head(*a)
        check_rows(fi.as_f64(out[0, h].cpu())[None], ref[None],
                   RowCond(cond[None], kden[None], {key: x[None] for key, x in t.items()}),
                   TOL_BF16, U_CAUSAL16, "seeded omega")
