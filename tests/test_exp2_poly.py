"""The FMA-pipe exponentials of the forward kernel (``exp2_poly2_x2`` for e4m3
inputs, ``exp2_poly3_x2`` for bf16).

The kernel computes 2^x = 2^n * p(f) with n = round(x), f = x - n and a
degree-2 or degree-3 polynomial p whose coefficients live in fwd_common.cuh
and are fitted by csrc/gen_exp2_poly.py.  Here the same float32 steps are
simulated in NumPy and held against float64 exp2: the relative error must
stay far below the rounding step P is stored with right after (2^-4 for
e4m3, 2^-9 for bf16).
"""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "context_blocks_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def _kernel_coeffs(degree=2):
    text = open(os.path.join(CSRC, "fwd_common.cuh")).read()
    vals = [float(re.search(rf"kExp2P{degree}C{i}\s*=\s*([-0-9.eE+]+)f", text).group(1))
            for i in range(degree + 1)]
    return np.array(vals, dtype=np.float32)


def test_kernel_coefficients_match_the_fit():
    c, err = gen_exp2_poly.fit(2)
    assert err < 2e-3
    assert np.allclose(_kernel_coeffs(), c.astype(np.float32), rtol=1e-6, atol=0)


def test_fit_is_equioscillating():
    # A minimax fit of degree 2 has 4 alternating extrema of equal size.
    c, err = gen_exp2_poly.fit(2)
    f = np.linspace(-0.5, 0.5, 20001)
    r = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    ext = [r[0]] + [r[i] for i in range(1, len(r) - 1) if (r[i] - r[i - 1]) * (r[i + 1] - r[i]) < 0] + [r[-1]]
    assert len(ext) == 4
    assert np.all(np.sign(ext[:-1]) != np.sign(ext[1:]))
    assert np.allclose(np.abs(ext), err, rtol=1e-4)


def test_emulated_exp2_error_bound():
    c = _kernel_coeffs()
    x = np.linspace(-120.0, 8.0, 1_000_001)
    r = gen_exp2_poly.simulate(c, x).astype(np.float64)
    rel = np.abs(r - np.exp2(x)) / np.exp2(x)
    assert rel.max() < 1.75e-3         # vs 2^-4 for the e4m3 P it feeds


def test_emulated_exp2_exact_points_and_underflow():
    c = _kernel_coeffs()
    ints = np.arange(-100, 9, dtype=np.float64)
    r = gen_exp2_poly.simulate(c, ints).astype(np.float64)
    # at integers f = 0 and the result is c0 * 2^n
    assert np.allclose(r, c[0] * np.exp2(ints), rtol=1e-7, atol=0)
    tiny = gen_exp2_poly.simulate(c, np.array([-200.0, -1e9, -np.inf]))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)


def test_degree3_coefficients_match_the_fit_and_error_bound():
    c, err = gen_exp2_poly.fit(3)
    assert err < 8e-5
    k = _kernel_coeffs(3)
    assert np.allclose(k, c.astype(np.float32), rtol=1e-6, atol=0)
    x = np.linspace(-120.0, 8.0, 1_000_001)
    r = gen_exp2_poly.simulate(k, x).astype(np.float64)
    rel = np.abs(r - np.exp2(x)) / np.exp2(x)
    assert rel.max() < 1.6e-4          # vs 2^-9 ~ 2e-3 for the bf16 P it feeds
    tiny = gen_exp2_poly.simulate(k, np.array([-200.0, -1e9, -np.inf]))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)


def test_degree3_fit_is_equioscillating():
    c, err = gen_exp2_poly.fit(3)
    f = np.linspace(-0.5, 0.5, 20001)
    r = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    ext = [r[0]] + [r[i] for i in range(1, len(r) - 1) if (r[i] - r[i - 1]) * (r[i + 1] - r[i]) < 0] + [r[-1]]
    assert len(ext) == 5
    assert np.all(np.sign(ext[:-1]) != np.sign(ext[1:]))
    assert np.allclose(np.abs(ext), err, rtol=1e-3)
