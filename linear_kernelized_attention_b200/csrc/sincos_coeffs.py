"""Derive the polynomial coefficients of the FMA-pipe sine and cosine in ``sincos_poly.cuh``.

The trig feature map needs cos(u) and sin(u) for every projected angle u. The SFU evaluates
them at 16 results per SM per clock; the FMA pipe evaluates 128 fused multiply-adds per SM per
clock. The kernels split the angles between the two, and this script gives the FMA-pipe half
its polynomials.

Method (classical argument reduction plus minimax approximation):
  * Reduction. n = round(u / pi) and r = u - n pi in [-pi/2, pi/2], with pi split as
    PI_HI + PI_LO (Cody and Waite, "Software Manual for the Elementary Functions", 1980):
    PI_HI keeps the leading bits of pi with the trailing ones zero, so n * PI_HI is exact
    in float32 for |n| < 2^(24 - bits(PI_HI)); PI_LO = fl32(pi - PI_HI). Then
    sin u = (-1)^n sin r and cos u = (-1)^n cos r.
  * Approximation. sin r = r + r^3 (s1 + s2 r^2 + s3 r^4) and
    cos r = 1 + r^2 (c1 + c2 r^2 + c3 r^4 + c4 r^6) on [-pi/2, pi/2]. The coefficients
    minimise the maximum absolute error (sin, cos take values in [-1, 1], and the kernels
    round them to 16-bit operands whose error is absolute near zero). They come from the
    Remez exchange algorithm (E. Remez, 1934): solve for the coefficients that equioscillate
    on a reference set of points, move the reference to the error's extrema, repeat.
Running this file prints the constants as C++ and the maximum errors in float64 and in a
float32 emulation of the kernel's evaluation order.
"""
from __future__ import annotations

import numpy as np

HALF_PI = np.pi / 2


def remez(basis, target, a, b, n_iter=40, grid=20001):
    """Minimax fit of target(x) by sum_i c_i basis_i(x) on [a, b] (absolute error)."""
    n = len(basis)
    xs = np.linspace(a, b, grid)
    # initial reference: Chebyshev extrema
    k = np.arange(n + 1)
    ref = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k / n)[::-1]
    for _ in range(n_iter):
        A = np.stack([f(ref) for f in basis] + [(-1.0) ** np.arange(n + 1)], axis=1)
        sol = np.linalg.solve(A, target(ref))
        c = sol[:n]
        err = target(xs) - sum(ci * f(xs) for ci, f in zip(c, basis))
        # new reference: the extremum of each sign-constant run of the error
        sgn = np.sign(err)
        runs, start = [], 0
        for i in range(1, len(xs) + 1):
            if i == len(xs) or sgn[i] != sgn[start]:
                j = start + int(np.argmax(np.abs(err[start:i])))
                runs.append(j)
                start = i
        if len(runs) < n + 1:
            break
        # keep n + 1 alternating extrema with the largest errors
        while len(runs) > n + 1:
            drop = min(range(len(runs)), key=lambda t: abs(err[runs[t]]))
            runs.pop(drop)
        ref = xs[runs]
    return c, np.max(np.abs(err))


def derive():
    # sin r - r = r^3 (s1 + s2 r^2 + s3 r^4): fit on r in (0, pi/2] (odd symmetry)
    sin_basis = [lambda x, p=p: x ** (2 * p + 3) for p in range(3)]
    s, es = remez(sin_basis, lambda x: np.sin(x) - x, 1e-6, HALF_PI)
    # cos r - 1 = r^2 (c1 + c2 r^2 + c3 r^4 + c4 r^6): even, fit on [0, pi/2]
    cos_basis = [lambda x, p=p: x ** (2 * p + 2) for p in range(4)]
    c, ec = remez(cos_basis, lambda x: np.cos(x) - 1.0, 0.0, HALF_PI)
    return s, c, es, ec


def split_pi(bits=16):
    hi = np.float32(np.round(np.pi * 2.0 ** (bits - 2)) / 2.0 ** (bits - 2))
    lo = np.float32(np.pi - np.float64(hi))
    return hi, lo


def emulate_f32(u, s, c, hi, lo):
    """The kernel's float32 evaluation order (fused multiply-adds emulated in float64, then
    rounded to float32 after each operation)."""
    f = np.float32
    u = u.astype(np.float32)
    magic = f(12582912.0)  # 1.5 * 2^23
    t = (u.astype(np.float64) * np.float64(f(1.0 / np.pi)) + np.float64(magic)).astype(np.float32)
    n = (t - magic).astype(np.float32)
    r = (n.astype(np.float64) * -np.float64(hi) + u.astype(np.float64)).astype(np.float32)
    r = (n.astype(np.float64) * -np.float64(lo) + r.astype(np.float64)).astype(np.float32)
    r2 = (r * r).astype(np.float32)
    ps = (r2.astype(np.float64) * np.float64(f(s[2])) + np.float64(f(s[1]))).astype(np.float32)
    ps = (r2.astype(np.float64) * ps.astype(np.float64) + np.float64(f(s[0]))).astype(np.float32)
    r3 = (r2 * r).astype(np.float32)
    sr = (r3.astype(np.float64) * ps.astype(np.float64) + r.astype(np.float64)).astype(np.float32)
    pc = (r2.astype(np.float64) * np.float64(f(c[3])) + np.float64(f(c[2]))).astype(np.float32)
    pc = (r2.astype(np.float64) * pc.astype(np.float64) + np.float64(f(c[1]))).astype(np.float32)
    pc = (r2.astype(np.float64) * pc.astype(np.float64) + np.float64(f(c[0]))).astype(np.float32)
    cr = (r2.astype(np.float64) * pc.astype(np.float64) + 1.0).astype(np.float32)
    odd = (n.astype(np.int64) & 1) == 1
    sr = np.where(odd, -sr, sr)
    cr = np.where(odd, -cr, cr)
    return sr.astype(np.float64), cr.astype(np.float64)


if __name__ == "__main__":
    s, c, es, ec = derive()
    hi, lo = split_pi()
    print("// minimax on [-pi/2, pi/2]; max abs error (float64): sin %.3g, cos %.3g" % (es, ec))
    print("constexpr float kPiHi = %.9ef, kPiLo = %.9ef;" % (hi, lo))
    print("constexpr float kS1 = %.9ef, kS2 = %.9ef, kS3 = %.9ef;" % tuple(np.float32(s)))
    print("constexpr float kC1 = %.9ef, kC2 = %.9ef, kC3 = %.9ef, kC4 = %.9ef;" % tuple(np.float32(c)))
    u = np.linspace(-400.0, 400.0, 2_000_001).astype(np.float32)
    sr, cr = emulate_f32(u, s, c, hi, lo)
    ud = u.astype(np.float64)
    print("// float32 emulation on |u| <= 400: max abs error sin %.3g, cos %.3g"
          % (np.max(np.abs(sr - np.sin(ud))), np.max(np.abs(cr - np.cos(ud)))))
