"""Fits the minimax polynomial the CUDA kernels use for 2^f on [-1/2, 1/2].

Method: Remez exchange for the best uniform approximation of the *relative*
error of a degree-n polynomial p(f) ~ 2^f (minimise max |p(f)/2^f - 1|),
starting from Chebyshev nodes.  2^x for general x is then 2^round(x) *
p(x - round(x)), the integer part going into the float's exponent field
(Cody-Waite style range reduction with a single split).

Run: python -m rank_latent_attention_flare_b200.fit_exp2_poly (prints coefficients and error)
"""
import numpy as np


def remez_exp2(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (equioscillating relative error)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new extremal points: one per sign-alternating segment
        sgn = np.sign(err)
        idx = np.where(np.diff(sgn) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [grid.size]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_exp2()
    c32 = np.float32(c)
    grid = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c32[3] * grid + c32[2]) * grid + c32[1]) * grid + c32[0]
    e32 = float(np.abs(p.astype(np.float64) / 2.0 ** grid.astype(np.float64) - 1).max())
    print("coefficients c0..c3:", [float(v) for v in c32])
    print(f"max relative error: {e:.3e} (float32 Horner: {e32:.3e})")
