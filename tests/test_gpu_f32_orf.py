"""fp32 accuracy path and the on-device ORF builder vs the oracle; device status checks."""
import numpy as np
import pytest

import favor_inputs as fi
from cases import Case
from oracle import favor_oracle as O
from parity_util import TOL_F32, U_F32, check_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,L,d,M", [(1, 1, 256, 16, 32), (2, 2, 200, 64, 64), (1, 3, 65, 8, 40)])
def test_f32_matches_oracle(kind, causal, B, H, L, d, M):
    import linear_kernelized_attention_b200 as F
    c = Case(B, H, L, d, M, dtype="f32", seed=L + d)
    q, k, v, om = c.device()
    out = fi.as_f64(F.favor_attention_f32(q, k, v, om, feature_kind=kind, causal=causal))
    assert F.favor_sync_status() == 0
    ref, cond, _ = c.oracle(kind, causal)
    st = check_rows(out.reshape(B * H, L, d), ref, cond, TOL_F32, U_F32, f"f32 {kind} {causal}", trig=kind == 0)
    print(st)


@pytest.mark.parametrize("M,d", [(32, 16), (256, 64), (40, 16), (96, 64)])
def test_orf_builder_matches_oracle(M, d):
    import torch
    import linear_kernelized_attention_b200 as F
    G, R = fi.orf_gaussians(3, M, d, seed=M + d)
    om = F.favor_orf_omega(torch.from_numpy(G).cuda(), torch.from_numpy(R).cuda(), M, dtype=torch.float32)
    ref = O.orf_matrices(G, R, M)
    np.testing.assert_allclose(fi.as_f64(om), ref, rtol=2e-6, atol=2e-6)
    omb = F.favor_orf_omega(torch.from_numpy(G).cuda(), torch.from_numpy(R).cuda(), M, dtype=torch.bfloat16)
    np.testing.assert_allclose(fi.as_f64(omb), ref, rtol=2 ** -8, atol=1e-6)


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    import linear_kernelized_attention_b200 as F
    assert F.favor_selftest_timeout(2_000_000) == 0
    assert F.favor_sync_status() == -7        # FAVOR_ERR_TIMEOUT
    assert F.favor_sync_status() == 0         # cleared
    x = torch.ones(1000, device="cuda")
    assert float(x.sum()) == 1000.0           # context still usable


def test_host_buffer_entry_matches_device_entry():
    import torch
    import linear_kernelized_attention_b200 as F
    c = Case(1, 2, 300, 64, 128, seed=11)
    q, k, v, om = c.device()
    dev = F.favor_attention(q, k, v, om, feature_kind=0).cpu()
    hq, hk, hv, hom = (t.pin_memory() for t in c.t)
    out = torch.empty_like(hq).pin_memory()
    F.favor_attention_host(hq, hk, hv, hom, out, feature_kind=0)
    assert torch.equal(out, dev)


@pytest.mark.parametrize("kind,causal", [(0, False), (1, True), (0, True)])
def test_host_buffer_entry_pipelines_batch_slices(kind, causal):
    # B = 6 runs as four batch slices (1, 2, 1, 2 entries) whose copies overlap the compute: each
    # slice must equal the device entry run on that slice alone
    import torch
    import linear_kernelized_attention_b200 as F
    c = Case(6, 2, 300, 64, 128, seed=12)
    q, k, v, om = c.device()
    hq, hk, hv, hom = (t.pin_memory() for t in c.t)
    out = torch.full_like(hq, float("nan")).pin_memory()
    F.favor_attention_host(hq, hk, hv, hom, out, feature_kind=kind, causal=causal)
    for b0, b1 in [(0, 1), (1, 3), (3, 4), (4, 6)]:
        want = F.favor_attention(q[b0:b1].contiguous(), k[b0:b1].contiguous(), v[b0:b1].contiguous(), om,
                                 feature_kind=kind, causal=causal).cpu()
        assert torch.equal(out[b0:b1], want), (b0, b1)
    assert F.favor_sync_status() == 0


def test_host_buffer_entry_unaligned_batch_entries_run_as_one_slice():
    # H = 1, L = 50, d = 33 in fp32: a batch entry is 6600 bytes, not a multiple of 16, so the
    # entry keeps the whole batch in one slice (every device entry needs 16-byte aligned pointers)
    import torch
    import linear_kernelized_attention_b200 as F
    c = Case(3, 1, 50, 33, 40, dtype="f32", seed=13)
    q, k, v, om = c.device()
    want = F.favor_attention_f32(q, k, v, om, feature_kind=0).cpu()
    hq, hk, hv, hom = (t.pin_memory() for t in c.t)
    out = torch.empty_like(hq).pin_memory()
    F.favor_attention_host(hq, hk, hv, hom, out, feature_kind=0)
    assert torch.equal(out, want)
