"""Fit the polynomials of the kernels' FMA-pipe exponentials (``exp2_poly2_x2``
for the e4m3 path, ``exp2_poly3_x2`` for the bf16 path).

2^x is split as 2^n * 2^f with n = round-to-nearest(x) and f = x - n in
[-1/2, 1/2] (Cody-Waite range reduction: W. J. Cody and W. Waite, "Software
Manual for the Elementary Functions", 1980).  2^f is approximated by a
polynomial whose coefficients minimise the maximum RELATIVE error over
[-1/2, 1/2] (the Remez exchange algorithm, weighted by 1 / 2^f).  2^n is applied by adding n to the
float32 exponent field.

Degree 2 is enough for the e4m3 path: its P is rounded to e4m3 (relative step
2^-4) right after, and the fit's 1.73e-3 is far below that.  The bf16 path
rounds P to bf16 (half step 2^-9, about 2e-3) and takes degree 3 (7.5e-5).

The printed coefficients are the kExp2P2C* and kExp2P3C* constants of
fwd_common.cuh; the second figure of each simulates the kernel's float32
steps (magic-number rounding, Horner steps, exponent add) against float64
exp2 over [-126, 8].

    python context_blocks_b200/csrc/gen_exp2_poly.py
"""

import numpy as np

MAGIC = np.float32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer


def fit(degree: int = 2, iters: int = 30):
    """Coefficients c_0..c_degree (float64) and their max relative error:
    the Remez exchange algorithm for the weighted (relative) error
    (p(f) - 2^f) / 2^f on [-1/2, 1/2], started from Chebyshev extrema."""
    m = degree + 2
    ref = -0.5 * np.cos(np.pi * np.arange(m) / (m - 1))   # reference points
    grid = np.linspace(-0.5, 0.5, 200001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  at the m reference points
        y = np.exp2(ref)
        a = np.hstack([np.vander(ref, degree + 1, increasing=True), (-(-1.0) ** np.arange(m) * y)[:, None]])
        sol = np.linalg.solve(a, y)
        c = sol[:-1]
        err = (np.vander(grid, degree + 1, increasing=True) @ c - np.exp2(grid)) / np.exp2(grid)
        # new reference: the extremum of each run of equal sign
        sign_change = np.nonzero(np.sign(err[1:]) != np.sign(err[:-1]))[0]
        bounds = np.concatenate([[0], sign_change + 1, [len(grid)]])
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(ext) != m:
            break
        new_ref = grid[ext]
        if np.allclose(new_ref, ref, atol=1e-12, rtol=0):
            break
        ref = new_ref
    err = (np.vander(grid, degree + 1, increasing=True) @ c - np.exp2(grid)) / np.exp2(grid)
    return c, float(np.max(np.abs(err)))


def simulate(c32: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The kernel's float32 steps, bit for bit where numpy allows: clamp at
    -126, t = x + MAGIC, n = t - MAGIC, f = x - n, Horner in float32, then the
    low bits of t (which hold n) shifted into the exponent field."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    fr = (x - n).astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * fr + np.float32(c32[k])).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    for degree in (2, 3):
        c, e = fit(degree)
        c32 = c.astype(np.float32)
        print(f"degree {degree} coefficients (c0..c{degree}):", ", ".join(f"{v:.9e}f" for v in c32))
        print(f"  max relative error of the polynomial on [-1/2, 1/2]: {e:.3e}")
        x = np.linspace(-126.0, 8.0, 400001)
        r = simulate(c32, x)
        print(f"  max relative error of the float32 emulation on [-126, 8]: "
              f"{np.max(np.abs(r - np.exp2(x)) / np.exp2(x)):.3e}")
