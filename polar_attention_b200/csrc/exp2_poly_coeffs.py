"""Derives the minimax polynomial used by the tensor-core prefill for part of
its exponentials (2^f on [-1/2, 1/2], relative error), and prints the fp32
coefficients that fwd_tc.cu holds.

Method: Cody-Waite range reduction 2^x = 2^n * 2^f with n = round(x), and a
Remez exchange for the polynomial p of degree D minimising
max |p(f) / 2^f - 1| on [-1/2, 1/2]; the constant term is then pinned to 1 so
that 2^0 is exact.  Run:  python polar_attention_b200/csrc/exp2_poly_coeffs.py
"""
import numpy as np

D = 4
LO, HI = -0.5, 0.5


def remez(deg, iters=30):
    n = deg + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative error)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, grid.size - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        # keep n extrema with alternating sign, largest magnitude
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = sorted(cand[:n])
        x = grid[chosen]
    return c, np.max(np.abs(err))


def fp32_eval(c32, f):
    """Horner in fp32 with fused multiply-adds (as the kernel does)."""
    f = f.astype(np.float64)
    p = np.full_like(f, np.float64(c32[-1]))
    for ci in c32[-2::-1]:
        p = (p * f + np.float64(ci)).astype(np.float32).astype(np.float64)
    return p


if __name__ == "__main__":
    c, e = remez(D)
    c32 = c.astype(np.float32)
    c32[0] = np.float32(1.0)
    f = np.linspace(LO, HI, 1000001).astype(np.float32)
    rel = np.abs(fp32_eval(c32, f) / 2.0 ** f.astype(np.float64) - 1.0)
    print(f"degree {D}: minimax relative error {e:.3e}; fp32 Horner max {rel.max():.3e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci):.9e}f  ({ci.view(np.uint32):#010x})")
