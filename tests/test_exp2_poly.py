"""The FMA-pipe exp2 used for a share of the softmax exponentials.

The kernel computes 2^x = 2^n * p(f) with n = round(x), f = x - n and a
degree-3 polynomial p (coefficients in fwd_common.cuh, fitted by
csrc/gen_exp2_poly.py).  Here the same float32 steps are simulated in NumPy
and held against float64 exp2: the relative error must stay far below the
bf16 rounding step (2^-9) that P is stored with.
"""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "context_blocks_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def _kernel_coeffs():
    text = open(os.path.join(CSRC, "fwd_common.cuh")).read()
    vals = [float(re.search(rf"kExp2C{i}\s*=\s*([-0-9.eE+]+)f", text).group(1)) for i in range(4)]
    return np.array(vals, dtype=np.float32)


def test_kernel_coefficients_match_the_fit():
    c, err = gen_exp2_poly.fit()
    assert err < 1e-4
    assert np.allclose(_kernel_coeffs(), c.astype(np.float32), rtol=1e-6, atol=0)


def test_emulated_exp2_error_bound():
    c = _kernel_coeffs()
    x = np.linspace(-120.0, 8.0, 1_000_001)
    r = gen_exp2_poly.simulate(c, x).astype(np.float64)
    rel = np.abs(r - np.exp2(x)) / np.exp2(x)
    assert rel.max() < 1.2e-4           # vs 2^-9 ~ 2e-3 for the bf16 P it feeds


def test_emulated_exp2_exact_points_and_underflow():
    c = _kernel_coeffs()
    ints = np.arange(-100, 9, dtype=np.float64)
    r = gen_exp2_poly.simulate(c, ints).astype(np.float64)
    assert np.allclose(r, np.exp2(ints), rtol=1e-4, atol=0)
    tiny = gen_exp2_poly.simulate(c, np.array([-200.0, -1e9, -np.inf]))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)
