"""Fit the minimax polynomials behind the kernels' software exp2.

    python bf16_causal_prefill_02_b200/csrc/exp2_poly_fit.py

Method: Cody-Waite style range reduction 2^z = 2^n * 2^f with n = rne(z) and
f = z - n in [-1/2, 1/2], and a polynomial p(f) ~ 2^f whose maximum
*relative* error on that interval is minimised by the Remez exchange
algorithm (equioscillation of (p(f) - 2^f) / 2^f at degree + 2 points).
The coefficients are rounded to fp32 and printed with the resulting error
bound; attn_fwd.cu carries the degree-3 and degree-4 sets verbatim and the
GPU test of the polynomial checks the device against CUDA's exp2f with these
bounds.
"""
import numpy as np


def remez_exp2(deg: int, iters: int = 60):
    a, b = -0.5, 0.5
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  sum_k c_k x_i^k - (-1)^i E 2^x_i = 2^x_i
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[: deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extremum of each sign-alternating segment
        s = np.sign(err)
        s[s == 0] = 1
        bounds = np.flatnonzero(np.diff(s)) + 1
        segs = np.split(np.arange(grid.size), bounds)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitudes
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


def fp32_error(c):
    c32 = np.array(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.zeros_like(f)
    for ck in c32[::-1]:  # Horner in fp32, as the kernel evaluates it
        p = (p * f + ck).astype(np.float32)
    return c32, float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c, e = remez_exp2(deg)
        c32, e32 = fp32_error(c)
        print("degree %d: minimax rel. error %.3e, with fp32 coefficients and Horner %.3e" % (deg, e, e32))
        print("   c0..c%d =" % deg, ", ".join("%.9ef" % v for v in c32))
