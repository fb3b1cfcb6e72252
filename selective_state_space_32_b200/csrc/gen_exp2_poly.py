"""Derive the polynomial used for 2^f on the FMA pipe (|f| <= 1/2).

p(f) = 1 + f * q(f) with q of degree DEG-1, so that p(0) = 1 exactly (a zero
step keeps the state unchanged).  q comes from a Remez exchange for the minimax
relative error of p against 2^f on [-1/2, 1/2], i.e. the weighted minimax of
q(f) - (2^f - 1)/f with weight |f| / 2^f, in float64.  Prints c0..cDEG
(c0 = 1) as fp32 values with their bit patterns, and the error of the fp32
Horner evaluation (fused multiply-add, as on the GPU) against float64.

    python selective_state_space_32_b200/csrc/gen_exp2_poly.py [DEG]
"""
import sys

import numpy as np

DEG = int(sys.argv[1]) if len(sys.argv) > 1 else 5
LO, HI = -0.5, 0.5


def remez(deg, iters=60):
    m = deg                      # q has m coefficients (degree m-1); m+1 reference points
    n = m + 1
    g = lambda t: np.where(np.abs(t) < 1e-12, np.log(2.0), np.expm1(t * np.log(2.0)) / np.where(t == 0, 1, t))
    w = lambda t: np.abs(t) / np.exp2(t)
    grid = np.linspace(LO, HI, 400001)
    grid = grid[np.abs(grid) > 1e-9]
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (k[::-1] + 0.5) / n)
    for _ in range(iters):
        M = np.zeros((n, n))
        for i in range(n):
            M[i, :m] = x[i] ** np.arange(m)
            M[i, m] = -((-1) ** i) / w(x[i])
        sol = np.linalg.solve(M, g(x))
        q = sol[:m]
        err = (np.polyval(q[::-1], grid) - g(grid)) * w(grid)
        s = np.sign(err)
        idx = np.where(np.diff(s) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = np.array([b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])])
        if len(ext) < n:
            break
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[ext]
    return np.concatenate([[1.0], q]), np.abs(err).max()


c, e = remez(DEG)
c32 = c.astype(np.float32)
grid = np.linspace(LO, HI, 1000001).astype(np.float32)
def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


p = np.full_like(grid, c32[DEG])
for k in range(DEG - 1, -1, -1):
    p = fma32(p, grid, np.full_like(grid, c32[k]))
rel = np.abs(p.astype(np.float64) - np.exp2(grid.astype(np.float64))) / np.exp2(grid.astype(np.float64))
print(f"degree {DEG}: minimax relative error {e:.3e} (float64), fp32 Horner max {rel.max():.3e}")
for k, v in enumerate(c32):
    print(f"c{k} = {float(v)!r:>24}  ({np.float32(v).view(np.uint32):#010x})")
