"""Derive the polynomial used for phi(z) = (exp(z) - 1) / z on |z| <= Z.

Remez exchange for the minimax RELATIVE error of a degree-DEG polynomial
against phi on [-Z, Z], in float64 (phi > 0 there).  Prints the coefficients
(lowest first) as fp32 values and the error of the fp32 Horner evaluation
(fused multiply-add, as on the GPU) against float64.

    python selective_state_space_32_b200/csrc/gen_phi_poly.py [DEG] [Z] [--log2]

With --log2 the polynomial's variable is e = z / ln 2 (the exponent of 2^e =
exp(z) that the kernels already compute), i.e. the fit is of phi(e ln 2) on
|e| <= Z / ln 2.
"""
import sys

import numpy as np

ARGS = [a for a in sys.argv[1:] if not a.startswith("--")]
DEG = int(ARGS[0]) if len(ARGS) > 0 else 4
Z = float(ARGS[1]) if len(ARGS) > 1 else 0.25
LOG2 = "--log2" in sys.argv
SCALE = np.log(2.0) if LOG2 else 1.0  # z = SCALE * variable
if LOG2:
    Z = Z / np.log(2.0)


def phi(v):
    z = np.asarray(v, dtype=np.float64) * SCALE
    out = np.ones_like(z)
    nz = np.abs(z) > 1e-12
    out[nz] = np.expm1(z[nz]) / z[nz]
    return out


def remez(deg, lo, hi, iters=60):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 400001)
    for _ in range(iters):
        M = np.zeros((n, n))
        for i in range(n):
            M[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            M[i, deg + 1] = -((-1) ** i) * phi(x[i:i + 1])[0]
        sol = np.linalg.solve(M, phi(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - phi(grid)) / phi(grid)
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
    return c, np.abs(err).max()


c, e = remez(DEG, -Z, Z)
c32 = c.astype(np.float32)
g = np.linspace(-Z, Z, 1000001).astype(np.float32)
p = np.full_like(g, c32[DEG])
for k in range(DEG - 1, -1, -1):
    p = (p.astype(np.float64) * g.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
rel = np.abs(p.astype(np.float64) - phi(g.astype(np.float64))) / phi(g.astype(np.float64))
print(f"degree {DEG} on |{'e' if LOG2 else 'z'}| <= {Z:.8f}: minimax relative error {e:.3e} (float64), fp32 Horner max {rel.max():.3e}")
for k, v in enumerate(c32):
    print(f"c{k} = {float(v)!r:>24}  ({np.float32(v).view(np.uint32):#010x})")
