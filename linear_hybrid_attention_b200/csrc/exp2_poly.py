"""Coefficients of the degree-3 polynomial used for 2^f, f in [0, 1), in the
softmax of the tile-sparse attention kernel (part of the exponentials run on
the FMA pipes instead of the MUFU unit).

Method: Cody-Waite style range reduction 2^x = 2^floor(x) * 2^f, f = x - floor(x)
in [0, 1); 2^f is approximated by the cubic that minimises the maximum
RELATIVE error on [0, 1] (Remez exchange on the equioscillation points),
with the constraint p(0) = 1 so that integer x give exact powers of two.
Run this file to re-derive the constants written in attn.cu:

    python linear_hybrid_attention_b200/csrc/exp2_poly.py
"""
import numpy as np


def remez_exp2(deg: int = 3, iters: int = 30):
    """Minimax-relative polynomial p(f) = 1 + a1 f + ... + ad f^d for 2^f on [0, 1]."""
    n = deg  # unknowns a1..ad plus the level E -> deg + 1 equations on deg + 1 points
    # initial reference: Chebyshev-like points in (0, 1]
    pts = 0.5 - 0.5 * np.cos(np.pi * (np.arange(1, n + 2)) / (n + 1))
    grid = np.linspace(0.0, 1.0, 200001)
    a = None
    for _ in range(iters):
        # solve (1 + sum a_k f^k - 2^f) / 2^f = (-1)^i E at the reference points
        A = np.zeros((n + 1, n + 1))
        rhs = np.zeros(n + 1)
        for i, f in enumerate(pts):
            w = 2.0 ** f
            A[i, :n] = [f ** k / w for k in range(1, n + 1)]
            A[i, n] = -((-1.0) ** i)
            rhs[i] = 1.0 - 1.0 / w
        sol = np.linalg.solve(A, rhs)
        a = sol[:n]
        err = (1.0 + sum(a[k - 1] * grid ** k for k in range(1, n + 1))) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        idx = [int(np.argmax(np.abs(err[(grid >= lo) & (grid <= hi)]))) + int(np.searchsorted(grid, lo))
               for lo, hi in zip(np.r_[0.0, (pts[:-1] + pts[1:]) / 2], np.r_[(pts[:-1] + pts[1:]) / 2, 1.0])]
        pts = grid[idx]
    err = (1.0 + sum(a[k - 1] * grid ** k for k in range(1, n + 1))) / 2.0 ** grid - 1.0
    return [1.0] + [float(v) for v in a], float(np.abs(err).max())


def eval_f32(coef, x):
    """The kernel's arithmetic in float32: Horner in fp32, then 2^floor(x) by exponent add."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    j = np.floor(x).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(coef[3])
    for c in (coef[2], coef[1], coef[0]):
        p = (p * f + np.float32(c)).astype(np.float32)
    bits = p.view(np.int32) + (j.astype(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    coef, e = remez_exp2()
    print("coefficients c0..c3:", ", ".join(f"{float(np.float32(c)):.9g}f" for c in coef))
    print(f"max relative error on [0,1]: {e:.3e}")
