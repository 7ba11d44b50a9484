"""The bf16 entry point rejects shapes no kernel covers, before any launch, and the output buffer
is left untouched. (Shapes the tensor-core kernels leave out, but the fp32 CUDA-core kernels
cover, take that route: tests/test_gpu_cuda_core_route.py.)"""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,M,kind,causal,chunk", [
    (136, 64, 0, False, 0), (136, 64, 1, True, 0),  # d > 128
    (64, 528, 1, False, 0), (64, 528, 1, True, 0),  # M > 512
    (64, 528, 0, False, 0), (64, 528, 0, True, 0),
    (64, 64, 0, True, 64), (64, 64, 1, True, 256),  # causal chunks other than 128
    (128, 64, 0, True, 128),                        # an explicit chunk on the CUDA-core route
])
def test_unsupported_shapes_return_status_and_launch_nothing(d, M, kind, causal, chunk):
    import torch
    import linear_kernelized_attention_b200 as F
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(1, 2, 100, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    om = torch.randn(2, M, d, generator=g).to(torch.bfloat16).cuda()
    out = torch.full_like(q, 3.0)
    with pytest.raises(F.FavorError) as e:
        F.favor_attention(q, k, v, om, out=out, feature_kind=kind, causal=causal, chunk=chunk)
    assert e.value.code == -5
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    assert F.favor_sync_status() == 0
