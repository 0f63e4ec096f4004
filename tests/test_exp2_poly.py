"""The FMA-pipe 2^x used for part of the softmax exponentials.

* The kernel header's coefficients are the degree-3 minimax polynomial of 2^f
  on [-1/2, 1/2] in relative error, rounded to fp32: the Remez exchange below
  re-derives them from that definition (Cody-Waite reduction x = n + f with
  n = round(x), so 2^x = 2^n * P(f)).
* The header's reduction and coefficients, evaluated step by step in fp32 on
  the CPU, stay within the stated relative error of 2^x over the whole input
  range the kernels feed it (clamped at -125, so results stay normal fp32)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_compression_cas_b200", "csrc", "vark_common.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("VARK_DEV void exp2_poly2"):]
    body = body[:body.index("\n}\n")]
    vals = dict(re.findall(r"(c[0-3]) = ([0-9.eE+-]+)f", body))
    return [np.float32(vals[f"c{i}"]) for i in range(4)]


def _remez_exp2(deg=3, a=-0.5, b=0.5, iters=30):
    """Minimax polynomial of 2^f on [a, b] in relative error: solve for
    equioscillating relative error E at deg + 2 reference points, move the
    references to the extrema of the new error curve, repeat."""
    n = deg + 2
    x = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (b - a) / 2 + (a + b) / 2
    grid = np.linspace(a, b, 20001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        idx = [0] + [i for i in range(1, len(grid) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) < 0] + [len(grid) - 1]
        if len(idx) != n:
            break
        x = grid[idx]
    return c, float(np.abs(err).max())


def test_coefficients_are_the_remez_fit():
    c, e = _remez_exp2()
    assert 7.0e-5 < e < 8.0e-5           # the minimax error of degree 3 on [-1/2, 1/2]
    hdr = np.array(_coefficients(), dtype=np.float64)
    np.testing.assert_allclose(hdr, c.astype(np.float32).astype(np.float64), rtol=2e-6)


def _device_exp2(x):
    """fp32 emulation of exp2_poly2: clamp, round via 1.5*2^23, Horner, add n
    into the exponent field."""
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) \
        & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_poly_exp2_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 12.0, 2_000_001), np.linspace(-1.0, 1.0, 200_001)]).astype(np.float32)
    got = _device_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_poly_exp2_reduction_edges():
    x = np.array([0.0, 0.5, -0.5, 1.5, -1.5, 7.999, 8.0, -124.5, -125.0, -125.5, -200.0, -np.inf],
                 dtype=np.float32)
    got = _device_exp2(x)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    np.testing.assert_allclose(got[:9], np.exp2(x[:9].astype(np.float64)), rtol=1e-4)
    assert np.all(got[9:] <= 2.0 ** -124)          # clamped far tail stays tiny and positive
