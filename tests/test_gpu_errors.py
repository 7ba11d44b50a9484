"""The bf16 entry point rejects shapes its kernels do not cover, before any launch, and the
output buffer is left untouched."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,M,kind,causal", [
    (48, 64, 0, False), (48, 64, 1, True),        # d not 16, 32, 64 or 128
    (128, 64, 0, True), (128, 64, 1, True),       # causal d = 128
    (128, 256, 0, False),                         # trig d = 128 with M = 256: no shared-memory plan
    (64, 272, 0, False), (64, 272, 0, True),      # trig M > 256
    (64, 528, 1, False), (64, 528, 1, True),      # relu M > 512
])
def test_unsupported_shapes_return_status_and_launch_nothing(d, M, kind, causal):
    import torch
    import linear_kernelized_attention_b200 as F
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(1, 2, 100, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    om = torch.randn(2, M, d, generator=g).to(torch.bfloat16).cuda()
    out = torch.full_like(q, 3.0)
    with pytest.raises(F.FavorError) as e:
        F.favor_attention(q, k, v, om, out=out, feature_kind=kind, causal=causal)
    assert e.value.code == -5
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    assert F.favor_sync_status() == 0
