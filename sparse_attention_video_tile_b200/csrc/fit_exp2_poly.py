"""Fits the cubic used by the attention kernel's software base-2 exponential.

Method: Cody-Waite style range reduction x = j + f with j = round(x) and
f in [-1/2, 1/2], so 2^x = 2^j * 2^f; 2^j is applied by adding j to the
exponent field and 2^f comes from a degree-3 polynomial whose coefficients are
the minimax (equioscillating) fit of 2^f on [-1/2, 1/2] under relative error,
found with the Remez exchange algorithm below.  The coefficients are rounded
to fp32 and the final relative error is measured on a dense grid in fp64.

The kernel rounds P to bf16 (relative spacing 2^-8), so a relative error
around 1e-4 is far below what the kernel keeps.

Run: python fit_exp2_poly.py  (prints the coefficients and the error).
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i * E * 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        b = 2.0 ** x
        sol = np.linalg.solve(A, b)
        coef = sol[:deg + 1]
        # new extrema of the relative error
        g = np.linspace(LO, HI, 200001)
        err = (np.polyval(coef[::-1], g) - 2.0 ** g) / 2.0 ** g
        # pick alternating extrema: split at sign changes
        idx = [0]
        sgn = np.sign(err)
        for i in range(1, len(g)):
            if sgn[i] != sgn[idx[-1]] and sgn[i] != 0:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) >= n:
            # keep the n consecutive extrema with the largest minimum magnitude
            best = None
            for s in range(len(idx) - n + 1):
                cand = idx[s:s + n]
                m = min(abs(err[c]) for c in cand)
                if best is None or m > best[0]:
                    best = (m, cand)
            x = g[best[1]]
    return coef


def main():
    c = remez()
    c32 = c.astype(np.float32).astype(np.float64)
    g = np.linspace(LO, HI, 1000001)
    rel = np.abs((np.polyval(c32[::-1], g) - 2.0 ** g) / 2.0 ** g)
    print("coefficients c0..c3 (fp32):")
    for i, v in enumerate(c.astype(np.float32)):
        print(f"  c{i} = {float(v)!r}f  ({float(v).hex()})")
    print(f"max relative error on [-1/2, 1/2]: {rel.max():.3e}")


if __name__ == "__main__":
    main()
