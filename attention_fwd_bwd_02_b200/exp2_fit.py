"""Fits the polynomial of the forward kernel's FMA-pipe exp2.

The forward kernel evaluates part of its 2^x values without the MUFU unit:
x is split as x = j + f with j = rint(x) and f in [-1/2, 1/2]; 2^f comes
from a cubic polynomial and 2^j is added to the exponent field.  This
script finds the cubic that minimises the maximum RELATIVE error of
p(f) ~ 2^f on [-1/2, 1/2] with the Remez exchange algorithm (a textbook
method; nothing here is taken from a math library), rounds the
coefficients to fp32 and reports the error:

    python -m attention_fwd_bwd_02_b200.exp2_fit

The coefficients printed are the ones in csrc/fwd_sm100.cu (exp2_fma); the
CPU test tests/test_exp2_poly.py checks both facts.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(nodes):
    # p(x_i) - 2^x_i = (-1)^i * E * 2^x_i  (equioscillating relative error)
    n = DEGREE + 1
    A = np.zeros((n + 1, n + 1))
    b = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, :n] = [x ** k for k in range(n)]
        A[i, n] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:n], sol[n]


def fit(iters: int = 30):
    """Minimax-relative cubic for 2^f on [LO, HI]; returns fp64 coefficients
    c0..c3 (p(f) = c0 + c1 f + c2 f^2 + c3 f^3)."""
    n = DEGREE + 2
    k = np.arange(n)
    nodes = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(nodes)
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extremum of each sign-alternating run
        sign = np.sign(err)
        idx = [0] + list(np.nonzero(np.diff(sign))[0] + 1) + [len(grid)]
        ext = []
        for a, bnd in zip(idx[:-1], idx[1:]):
            seg = np.abs(err[a:bnd])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) >= n:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:n]
            nodes = np.sort(grid[ext])
    return c


def coefficients_f32():
    return [np.float32(x) for x in fit()]


def emulate(x, c):
    """fp32 evaluation of the kernel's exp2 (same operation order; each fma
    rounded once)."""
    f32 = np.float32
    x = np.maximum(np.asarray(x, dtype=np.float32), f32(-126.0))
    y = (x.astype(np.float64) + 12582912.0).astype(np.float32)
    j = (y.astype(np.float64) - 12582912.0).astype(np.float32)
    f = (x.astype(np.float64) - j.astype(np.float64)).astype(np.float32)

    def fma(a, b, d):
        return (a.astype(np.float64) * b.astype(np.float64) + d.astype(np.float64)).astype(np.float32)

    c0, c1, c2, c3 = (np.full_like(f, v) for v in c)
    p = fma(fma(fma(c3, f, c2), f, c1), f, c0)
    bits = p.view(np.int32) + (y.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c = coefficients_f32()
    xs = np.linspace(-126.0, 8.0, 2000001).astype(np.float32)
    rel = np.abs(emulate(xs, c).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error of the fp32 evaluation on [-126, 8]: {rel.max():.3e}")
