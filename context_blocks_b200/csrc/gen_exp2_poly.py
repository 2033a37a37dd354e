"""Fit the polynomial used by the kernels' FMA-pipe exp2 (``exp2_poly_x2``).

2^x is split as 2^n * 2^f with n = round-to-nearest(x) and f = x - n in
[-1/2, 1/2] (Cody-Waite style range reduction).  2^f is approximated by a
degree-3 polynomial whose coefficients minimise the maximum RELATIVE error
over [-1/2, 1/2]; the fit is an iteratively re-weighted least-squares
(Lawson) iteration on Chebyshev nodes.  2^n is applied by adding n to the
float32 exponent field.

The printed coefficients are pasted into fwd_common.cuh (kExp2C0..3).  The
second figure simulates the kernel's float32 arithmetic (magic-number
rounding, Horner steps, exponent add) and reports its max relative error
against float64 exp2 over [-126, 8].

    python context_blocks_b200/csrc/gen_exp2_poly.py
"""

import numpy as np


def fit(degree: int = 3, iters: int = 300):
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        wt = w / y
        c, *_ = np.linalg.lstsq(a * wt[:, None], y * wt, rcond=None)
        err = np.abs(a @ c - y) / y
        w = np.maximum(w * err / err.mean(), 1e-12)
    return c, float(np.max(np.abs(a @ c - y) / y))


def simulate(c32: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The kernel's float32 steps, bit for bit where numpy allows."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)                  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    fr = (x - n).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * fr + np.float32(c32[k])).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    print("coefficients (c0..c3):", ", ".join(f"{v:.9e}f" for v in c32))
    print(f"max relative error of the polynomial on [-1/2, 1/2]: {e:.3e}")
    x = np.linspace(-126.0, 8.0, 400001)
    r = simulate(c32, x)
    print(f"max relative error of the float32 emulation on [-126, 8]: "
          f"{np.max(np.abs(r - np.exp2(x)) / np.exp2(x)):.3e}")
