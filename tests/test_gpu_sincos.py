"""The FMA-pipe sine and cosine on the device (favor_selftest_sincos) against the mathematics.

Angles span |u| <= 400, beyond what the inputs reach (|omega . x| stays below about 100 even for
the heavy-norm rows, whose norms are four times the others'). The device values must stay within
the bound the header states (1e-6 for sin, 2e-7 for cos, absolute, against fp64) and agree with
the CPU emulation of the same float32 evaluation order to within one float32 unit in the last
place (the emulation rounds each fused multiply-add from float64, which can differ from a single
rounding in rare ties).
"""
import importlib.util
import os

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs_module():
    path = os.path.join(ROOT, "linear_kernelized_attention_b200", "csrc", "sincos_coeffs.py")
    spec = importlib.util.spec_from_file_location("sincos_coeffs", path)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_device_sincos_error_bound_and_emulation():
    import torch
    import linear_kernelized_attention_b200 as F
    u = np.concatenate([np.linspace(-400.0, 400.0, 2_000_001),
                        np.random.default_rng(7).uniform(-100.0, 100.0, 1_000_000)]).astype(np.float32)
    s, c = F.favor_selftest_sincos(torch.from_numpy(u).cuda())
    assert F.favor_sync_status() == 0
    s = s.cpu().numpy().astype(np.float64)
    c = c.cpu().numpy().astype(np.float64)
    ud = u.astype(np.float64)
    assert np.max(np.abs(s - np.sin(ud))) <= 1e-6
    assert np.max(np.abs(c - np.cos(ud))) <= 2e-7
    m = _coeffs_module()
    co_s, co_c, _, _ = m.derive()
    hi, lo = m.split_pi()
    es, ec = m.emulate_f32(u, co_s, co_c, hi, lo)
    ulp = np.spacing(np.float32(1.0)).astype(np.float64)
    assert np.max(np.abs(s - es)) <= ulp and np.max(np.abs(c - ec)) <= ulp
    assert np.mean(s == es) > 0.999 and np.mean(c == ec) > 0.999


def test_device_sincos_rejects_bad_arguments():
    import ctypes
    import linear_kernelized_attention_b200 as F
    lib = F.lib()
    assert lib.favor_selftest_sincos(None, None, None, 4, None) == -1
    import torch
    u = torch.zeros(8, device="cuda")
    assert lib.favor_selftest_sincos(u.data_ptr(), u.data_ptr(), u.data_ptr(), 0, None) == -3
    assert lib.favor_selftest_sincos(u.data_ptr() + 2, u.data_ptr(), u.data_ptr(), 4, None) == -2
