"""The FMA-pipe sine and cosine of csrc/sincos_poly.cuh, on the CPU.

The header's constants must be the ones csrc/sincos_coeffs.py derives (a Remez exchange written
from the algorithm, not copied from any library), and the kernel's float32 evaluation order,
emulated operation by operation, must stay within the error the header states for |u| <= 400:
1e-6 for sin and 2e-7 for cos, absolute.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_kernelized_attention_b200", "csrc")


def _coeffs_module():
    spec = importlib.util.spec_from_file_location("sincos_coeffs", os.path.join(CSRC, "sincos_coeffs.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_constants():
    text = open(os.path.join(CSRC, "sincos_poly.cuh")).read()
    vals = dict(re.findall(r"(k(?:PiHi|PiLo|S1|S2|S3|C1|C2|C3|C4)) = ([-+0-9.e]+)f", text))
    return {k: np.float32(float(v)) for k, v in vals.items()}


def test_header_constants_are_the_derived_ones():
    m = _coeffs_module()
    s, c, es, ec = m.derive()
    hi, lo = m.split_pi()
    h = _header_constants()
    assert len(h) == 9
    assert h["kPiHi"] == np.float32(hi) and h["kPiLo"] == np.float32(lo)
    for name, val in zip(("kS1", "kS2", "kS3"), s):
        assert h[name] == np.float32(val), name
    for name, val in zip(("kC1", "kC2", "kC3", "kC4"), c):
        assert h[name] == np.float32(val), name
    # the fit itself: a few 1e-7 in float64, far below the 16-bit rounding of the features
    assert es < 1e-6 and ec < 3e-7
    # Cody-Waite head: its trailing bits are zero, so n * kPiHi is exact for |n| < 256
    mant = int(np.float32(hi).view(np.int32)) & 0x7FFFFF
    assert mant & ((1 << 12) - 1) == 0


def test_float32_evaluation_error_bound():
    m = _coeffs_module()
    s, c, _, _ = m.derive()
    hi, lo = m.split_pi()
    u = np.linspace(-400.0, 400.0, 400_001).astype(np.float32)
    sr, cr = m.emulate_f32(u, s, c, hi, lo)
    ud = u.astype(np.float64)
    assert np.max(np.abs(sr - np.sin(ud))) <= 1e-6
    assert np.max(np.abs(cr - np.cos(ud))) <= 2e-7
    # signs across the reduction: sin(-u) = -sin(u), cos(-u) = cos(u), and the pi-periodic flip
    sn, cn = m.emulate_f32(-u, s, c, hi, lo)
    np.testing.assert_array_equal(sn, -sr)
    np.testing.assert_array_equal(cn, cr)


def test_fit_equioscillates():
    # a minimax fit of k coefficients has k + 1 alternating extrema of equal size
    m = _coeffs_module()
    s, c, es, ec = m.derive()
    x = np.linspace(1e-6, np.pi / 2, 200_001)
    err = np.sin(x) - x - x ** 3 * (s[0] + s[1] * x ** 2 + s[2] * x ** 4)
    peaks = [i for i in range(1, len(x) - 1) if abs(err[i]) >= abs(err[i - 1]) and abs(err[i]) >= abs(err[i + 1])]
    big = [i for i in peaks + [len(x) - 1] if abs(err[i]) > 0.9 * np.max(np.abs(err))]
    assert len(big) >= 3
    assert np.all(np.diff(np.sign(err[big])) != 0)
