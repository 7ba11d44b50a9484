"""bf16 shapes the tensor-core kernels leave out (causal d = 128, bidirectional trig d = 128 with
M > 128, d outside {16, 32, 64, 128}, trig M > 256) run the fp32 CUDA-core kernels on exact fp32
copies of the bf16 inputs and round the result to bf16 once. Compared with the oracle on the same
bf16 inputs: the bf16 tolerance (2e-2 per row, the trig rows' fp32 conditioning allowance), and
the rounding of the output itself, 2^-8 of a row's largest entry, above the fp32 path's error."""
import pytest

import favor_inputs as fi
from cases import Case
from parity_util import TOL_BF16, U_F32, check_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,L,d,M,kind,causal", [
    (1, 2, 300, 128, 64, 0, True),    # causal d = 128
    (1, 2, 300, 128, 64, 1, True),
    (2, 1, 200, 128, 256, 0, False),  # bidirectional trig d = 128, M = 256
    (1, 2, 130, 48, 64, 0, False),    # d = 48
    (1, 2, 130, 48, 64, 1, False),
    (1, 2, 130, 48, 64, 0, True),
    (1, 2, 130, 48, 64, 1, True),
    (1, 1, 97, 64, 384, 0, True),     # trig M = 384
    (1, 1, 97, 64, 384, 0, False),
])
def test_cuda_core_route_matches_oracle(B, H, L, d, M, kind, causal):
    import torch
    import linear_kernelized_attention_b200 as F
    c = Case(B, H, L, d, M, seed=L + d + M)
    q, k, v, om = c.device()
    ws = F.favor_workspace_bytes(B, H, L, d, M, kind, causal)
    assert ws >= 4 * 4 * B * H * L * d
    out = torch.full_like(q, float("nan"))
    F.favor_attention(q, k, v, om, out=out, feature_kind=kind, causal=causal)
    assert F.favor_sync_status() == 0
    got = fi.as_f64(out).reshape(B * H, L, d)
    ref, cond, _ = c.oracle(kind, causal)
    label = f"route {kind} {causal} {B}x{H}x{L} d{d} M{M}"
    st = check_rows(got, ref, cond, TOL_BF16, U_F32, label, trig=kind == 0)
    # beyond the fp32 path's conditioning term, only the output's rounding to bf16
    assert st["max_rel"] <= 2.0 ** -8 + U_F32 * st["max_cond"], f"{label}: {st}"
    print(st)
