"""Fit of the degree-5 polynomial for 2^f on [-1/2, 1/2] used by the
prefill kernels (exp2_poly2 in prefill_common.cuh) to take part of the exponentials
off the MUFU unit.

Method: Remez exchange for the minimax RELATIVE error, i.e. minimise
max |p(f) / 2^f - 1| over f in [-1/2, 1/2]. Each iteration solves
p(x_i) - (-1)^i E 2^(x_i) = 2^(x_i) at 7 reference points (6 coefficients
and the levelled error E), then moves the references to the extrema of the
error curve found on a dense grid, until the extrema are level. The
coefficients are then rounded to float32.

    python block_quantized_precision_b200/csrc/exp2_poly_fit.py

prints the coefficients c0..c5 (2^f ~ c0 + c1 f + ... + c5 f^5) and the
relative error of the float32 polynomial evaluated in Horner form with
fused multiply-adds (as the kernel does).
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def _error_extrema(coef, grid):
    e = np.polyval(coef[::-1], grid) / np.exp2(grid) - 1.0
    # interior local extrema of e plus the end points, one per sign run
    idx = [0]
    for i in range(1, len(grid) - 1):
        if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
            idx.append(i)
    idx.append(len(grid) - 1)
    # keep the largest |e| within each run of equal sign
    runs = []
    for i in idx:
        if runs and np.sign(e[i]) == np.sign(e[runs[-1]]):
            if abs(e[i]) > abs(e[runs[-1]]):
                runs[-1] = i
        else:
            runs.append(i)
    return np.array(runs), e


def remez(iters=30):
    n = DEG + 2
    # Chebyshev extrema as the first references
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :DEG + 1] = x[i] ** np.arange(DEG + 1)
            A[i, DEG + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        coef = sol[:DEG + 1]
        ext, e = _error_extrema(coef, grid)
        if len(ext) < n:
            break
        # the n extrema with the largest error, kept in order
        if len(ext) > n:
            keep = np.sort(np.argsort(-np.abs(e[ext]))[:n])
            ext = ext[keep]
        x_new = grid[ext]
        if np.allclose(x_new, x, atol=1e-9):
            break
        x = x_new
    return coef


def eval_f32_horner(c32, f):
    """Horner with one float32 rounding per fused multiply-add (the product
    of two float32 values is exact in float64, so fma = one rounding of the
    float64 sum, up to a double-rounding tie that float64 makes vanishingly
    rare)."""
    f = f.astype(np.float32)
    q = np.full_like(f, c32[DEG])
    for k in range(DEG - 1, -1, -1):
        q = (q.astype(np.float64) * f.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
    return q


def max_rel_error_f32(c32, n=1 << 20):
    f = np.linspace(LO, HI, n).astype(np.float32)
    got = eval_f32_horner(c32, f).astype(np.float64)
    return float(np.max(np.abs(got / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = remez()
    c32 = c.astype(np.float32)
    for k, v in enumerate(c32):
        print("c%d = %.8e" % (k, v))
    print("max relative error, float64 polynomial: %.3e" % float(
        np.max(np.abs(np.polyval(c[::-1], np.linspace(LO, HI, 100001)) / np.exp2(np.linspace(LO, HI, 100001)) - 1))))
    print("max relative error, float32 Horner/FMA: %.3e" % max_rel_error_f32(c32))
