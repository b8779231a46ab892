"""Fit the polynomial the kernel uses to evaluate part of its exp2 on the FMA
pipe instead of the MUFU (special-function) unit.

Method (Cody-Waite range reduction + minimax polynomial):

    2^x = 2^n * 2^f,   n = round-to-nearest(x),   f = x - n in [-1/2, 1/2]

2^n is formed exactly by adding n to the IEEE exponent field; 2^f is a
degree-3 polynomial p(f) whose coefficients minimise the maximum *relative*
error max |p(f) / 2^f - 1| over [-1/2, 1/2].  They are found here with a
plain Remez exchange (equioscillation of the weighted error at deg + 2
reference points), then rounded to fp32 and checked on a dense grid with the
fp32 Horner evaluation the kernel performs.

The kernel only needs the bf16 precision of P (half an ulp = 2^-9
relative), so a degree-3 fit (about 9e-5 relative) is far inside the budget.

Run:  python gen_exp2_poly.py   -> prints the fp32 coefficients (hex floats)
that attn_fwd_kernel.cuh embeds, and the measured error bound.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def _solve(ref):
    # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}  for the deg + 2 reference points
    n = len(ref)
    A = np.zeros((n, n))
    b = np.exp2(ref)
    for i, x in enumerate(ref):
        A[i, :DEG + 1] = x ** np.arange(DEG + 1)
        A[i, DEG + 1] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:DEG + 1], sol[DEG + 1]


def rel_err(c, x):
    p = np.polynomial.polynomial.polyval(x, c)
    return p / np.exp2(x) - 1.0


def remez(iters: int = 30):
    k = np.arange(DEG + 2)
    ref = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * (DEG + 1 - k) / (DEG + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        c, _ = _solve(ref)
        e = rel_err(c, grid)
        # split the grid into sign-constant runs; keep each run's extremum
        s = np.sign(e)
        cuts = np.flatnonzero(np.diff(s) != 0) + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = [r[np.argmax(np.abs(e[r]))] for r in runs if r.size]
        while len(ext) > DEG + 2:  # drop the smallest end extremum
            if abs(e[ext[0]]) < abs(e[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        if len(ext) < DEG + 2:
            break
        ref = grid[ext]
    return c


def fp32_horner_error(c32, n=1 << 20):
    """Max relative error of the kernel's fp32 evaluation over [-1/2, 1/2]."""
    f = np.linspace(LO, HI, n).astype(np.float32)
    p = np.float32(c32[DEG])
    for k in range(DEG - 1, -1, -1):
        # fused multiply-add: one rounding of the exact p * f + c
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c32[k])
             ).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


def coefficients():
    c = remez()
    c32 = np.array(c, dtype=np.float32)
    return c, c32, fp32_horner_error(c32)


if __name__ == "__main__":
    c, c32, err = coefficients()
    print("degree", DEG, "minimax relative error (exact coefficients):",
          float(np.max(np.abs(rel_err(c, np.linspace(LO, HI, 200001))))))
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v).hex()}f  // {float(v):.9g}")
    print("fp32 Horner max relative error:", err)
