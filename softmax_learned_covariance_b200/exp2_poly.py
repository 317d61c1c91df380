"""Derivation of the polynomial 2^x the prefill kernel uses for part of its exponentials.

The prefill kernels (``csrc/softmax_sm100.cuh``, ``exp2_poly2``) reduce 2^x = 2^j * 2^f with
j = round(x) and f = x - j in [-1/2, 1/2], and evaluates 2^f with a degree-3
polynomial.  The coefficients are the minimax fit of 2^f on [-1/2, 1/2] in
relative error, found here with the Remez exchange algorithm (alternation of
the weighted error at n + 2 reference points, references moved to the error
extrema until they settle).  ``kernel_coefficients`` reads the constants back
from the CUDA source so a test can check that both agree.
"""
import os
import re

import numpy as np

_CU = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc", "softmax_sm100.cuh")


def remez_exp2(degree=3, lo=-0.5, hi=0.5, iters=40, grid=200001):
    """Coefficients c[0..degree] (ascending powers) minimising max |p(f)/2^f - 1| on [lo, hi]."""
    n = degree
    f = np.exp2
    k = np.arange(n + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    g = np.linspace(lo, hi, grid)
    c = None
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        A[:, :n + 1] = x[:, None] ** np.arange(n + 1)[None, :]
        A[:, n + 1] = -((-1.0) ** np.arange(n + 2)) * f(x)
        sol = np.linalg.solve(A, f(x))
        c = sol[:n + 1]
        err = np.polyval(c[::-1], g) / f(g) - 1.0
        sign_change = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], sign_change + 1, [grid]])
        ext = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n + 2:
            break
        x_new = g[ext]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    err = np.polyval(c[::-1], g) / f(g) - 1.0
    return c, float(np.max(np.abs(err)))


def kernel_coefficients(path=_CU):
    """EXP2_C0..EXP2_C3 as written in the CUDA source."""
    src = open(path).read()
    vals = {}
    for i in range(4):
        m = re.search(r"EXP2_C%d\s*=\s*([-+0-9.eE]+)f" % i, src)
        if m is None:
            raise ValueError("EXP2_C%d not found in %s" % (i, path))
        vals[i] = float(m.group(1))
    return np.array([vals[i] for i in range(4)])


def emulate_kernel_exp2(x, coeffs):
    """float32 emulation of the kernel's range reduction and polynomial (separate
    multiply and add, so each step may differ from the fused form by one ulp)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    kround = np.float32(12582912.0)
    t = (x + kround).astype(np.float32)
    r = (t - kround).astype(np.float32)
    f = (x - r).astype(np.float32)
    c = coeffs.astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)
