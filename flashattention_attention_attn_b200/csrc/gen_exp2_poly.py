"""Generate the coefficients of the software 2^x used by the prefill softmax.

Method (Cody-Waite style range reduction + minimax polynomial):
    x = j + f,  j = round-to-nearest(x),  f in [-1/2, 1/2]
    2^x = 2^j * p(f),  p ~ 2^f  (degree 3)
The exponent j is added to the bits of p(f) with an integer add.  p is the
minimax approximation of 2^f in *relative* error on [-1/2, 1/2], found with
a Remez exchange on the error function e(f) = p(f) / 2^f - 1.  (2^0 is
therefore not exact: p(0) differs from 1 by the levelled error.)

Running this file prints the coefficients (as float32 literals) and the
maximum relative error of the float32 evaluation; the values are pasted
into prefill_sm100.cuh and pinned by tests/test_exp2_poly.py.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 40):
    """Minimax p of the given degree for 2^f in relative error on [LO, HI]."""
    n = degree + 1  # coefficients c0..c_degree; n + 1 reference points
    k = np.arange(n + 1)
    ref = (LO + HI) / 2 - (HI - LO) / 2 * np.cos(np.pi * k / n)  # Chebyshev extrema
    grid = np.linspace(LO, HI, 400001)
    c = None
    for _ in range(iters):
        # p(f_k) - 2^f_k = (-1)^k E 2^f_k  at the n + 1 reference points
        A = np.zeros((n + 1, n + 1))
        for r, f in enumerate(ref):
            A[r, :n] = [f ** i for i in range(n)]
            A[r, n] = -((-1) ** r) * np.exp2(f)
        sol = np.linalg.solve(A, np.exp2(ref))
        c = sol[:n]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: one extremum of |err| per interval of constant sign
        bounds = np.flatnonzero(np.diff(np.sign(err)) != 0) + 1
        pieces = np.split(np.arange(len(grid)), bounds)
        ext = [pc[np.argmax(np.abs(err[pc]))] for pc in pieces if len(pc)]
        while len(ext) > n + 1:  # drop the smaller end extremum
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext.pop(0)
            else:
                ext.pop()
        if len(ext) == n + 1:
            ref = grid[ext]
    return c


def eval_f32(c, x):
    """Emulate the kernel's float32 evaluation of 2^x for x <= 0 arrays."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23: x + magic rounds x to an integer
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    c32 = [np.float32(v) for v in c]
    p = np.float32(c32[3])
    p = (p * f + c32[2]).astype(np.float32)
    p = (p * f + c32[1]).astype(np.float32)
    p = (p * f + c32[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def main():
    c = remez_relative()
    c32 = [float(np.float32(v)) for v in c]
    x = np.linspace(-126.0, 8.0, 4_000_001, dtype=np.float64)
    got = eval_f32(c32, x).astype(np.float64)
    rel = np.abs(got / np.exp2(x) - 1.0)
    for i, v in enumerate(c32):
        print(f"c{i} = {v:.9e}f")
    print(f"max relative error (float32 evaluation on [-126, 8]): {rel.max():.3e}")


if __name__ == "__main__":
    main()
