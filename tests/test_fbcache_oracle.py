"""Pins of the First Block Cache residual-difference oracle (oracle/fbcache.py)
to things other than itself: closed forms, hand-worked values, an invariance,
the zero conventions, and planted mistakes that each fail a pin (diffusers
"ParaAttention" guide, section "First Block Cache"; the relative L1 reading
stated in the oracle)."""

import numpy as np
import pytest

from oracle.fbcache import residual_diff


def _pins(f):
    rng = np.random.default_rng(11)
    prev = rng.standard_normal(1000)
    out = []
    out.append(f(prev, prev) == 0.0)                                    # unchanged residual
    out.append(abs(f(2 * prev, prev) - 1.0) < 1e-12)                    # doubled: |2p - p| = |p|
    out.append(abs(f(np.zeros(1000), prev) - 1.0) < 1e-12)              # vanished
    out.append(abs(f(-prev, prev) - 2.0) < 1e-12)                       # sign flip
    out.append(abs(f([1.0, -2.0, 3.0], [2.0, 2.0, 2.0]) - 1.0) < 1e-12)  # (1 + 4 + 1) / 6, by hand
    out.append(abs(f([0.5, 1.5], [1.0, 1.0]) - 0.5) < 1e-12)            # (0.5 + 0.5) / 2, by hand
    out.append(abs(f([2.0], [1.0]) - 1.0) < 1e-12 and abs(f([1.0], [2.0]) - 0.5) < 1e-12)  # not symmetric
    cur = rng.standard_normal(1000)
    out.append(abs(f(0.37 * cur, 0.37 * prev) - f(cur, prev)) < 1e-12)  # scale invariance
    return out


def test_oracle_pins():
    assert all(_pins(residual_diff))


def test_zero_conventions():
    assert residual_diff(np.zeros(4), np.zeros(4)) == 0.0
    assert residual_diff(np.ones(4), np.zeros(4)) == float("inf")


@pytest.mark.parametrize("mutant", [
    lambda c, p: float(np.abs(np.subtract(c, p)).sum() / np.abs(c).sum()),        # divides by |cur|
    lambda c, p: float(np.square(np.subtract(c, p)).sum() / np.square(p).sum()),   # squared (L2) differences
    lambda c, p: float(np.abs(np.subtract(c, p)).sum() / abs(np.sum(p))),          # |sum p| instead of sum |p|
    lambda c, p: float(np.abs(np.subtract(p, c)).sum() / np.abs(p).sum()) * 0.5,   # a stray factor
])
def test_planted_mistakes_fail_a_pin(mutant):
    def guarded(c, p):
        with np.errstate(divide="ignore", invalid="ignore"):
            return mutant(np.asarray(c, dtype=np.float64), np.asarray(p, dtype=np.float64))
    assert not all(_pins(guarded))
