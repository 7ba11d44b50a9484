"""The allocation-free fp32 entry point against the existing fp32 entry point.

favor_attention_f32_noalloc launches the same kernels as favor_attention_f32 with the
workspace in a static device array, so two calls in a row (the second reusing the array the
first wrote) must reproduce favor_attention_f32 bit for bit. This file is collected last so it
also runs after every other test has used the library.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _inputs(B, H, L, d, M, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, L, d, generator=g) * d ** -0.25 for _ in range(3))
    om = torch.randn(H, M, d, generator=g)
    return [t.cuda() for t in (q, k, v, om)]


def test_noalloc_matches_f32_entry_on_two_calls_in_a_row():
    import torch
    import linear_kernelized_attention_b200 as F
    # the second call is smaller, so stale workspace from the first would show up
    for (B, H, L, d, M, kind, causal, seed) in [(2, 4, 700, 64, 128, 0, True, 1),
                                                (1, 2, 300, 32, 64, 1, False, 2)]:
        q, k, v, om = _inputs(B, H, L, d, M, seed)
        ref = F.favor_attention_f32(q, k, v, om, feature_kind=kind, causal=causal)
        assert F.favor_sync_status() == 0
        got = F.favor_attention_f32_noalloc(q, k, v, om, feature_kind=kind, causal=causal)
        assert F.favor_sync_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (B, H, L, d, M, kind, causal)


def test_noalloc_rejects_oversize_workspace():
    import torch
    import linear_kernelized_attention_b200 as F
    cap = F.favor_noalloc_scratch_bytes()
    assert cap == 32 << 20
    # B*H*ceil(L/64)*2M*(d+1)*4 bytes: 8*128*512*65*4 = 136 MB > 32 MiB
    q, k, v, om = _inputs(1, 8, 8192, 64, 256, 3)
    out = torch.full_like(q, 7.0)
    with pytest.raises(F.FavorError) as e:
        F.favor_attention_f32_noalloc(q, k, v, om, out=out, feature_kind=0, causal=True)
    assert e.value.code == -5
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())   # nothing was launched
