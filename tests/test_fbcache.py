"""pa_residual_diff (First Block Cache's residual difference, diffusers
"ParaAttention" guide, section "First Block Cache") against the fp64 oracle
on the GPU: sizes around the 8-element vector width and its ragged tails up
to a FLUX-sized residual, closed forms that hold exactly in fp32, the zero
conventions, and bitwise determinism."""

import math

import pytest
import torch

import context_blocks_b200 as pa
from oracle.fbcache import residual_diff as oracle_diff

pytestmark = pytest.mark.gpu

REL = 1e-4  # fp32 accumulation of up to ~1e7 terms in a fixed tree


def _pair(n, seed, noise=0.05):
    g = torch.Generator(device="cuda").manual_seed(seed)
    prev = torch.randn(n, generator=g, device="cuda")
    cur = prev + noise * torch.randn(n, generator=g, device="cuda")
    return cur.to(torch.bfloat16), prev.to(torch.bfloat16)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 4097, 1_000_003, 4096 * 3072])
def test_matches_oracle(n):
    cur, prev = _pair(n, seed=n % 1000)
    got = float(pa.residual_diff(cur, prev, check=True).item())
    want = oracle_diff(cur, prev)
    assert math.isfinite(got) and abs(got - want) <= REL * max(want, 1e-30), (n, got, want)


def test_closed_forms_exact():
    cur, prev = _pair(1_000_003, seed=3)
    assert float(pa.residual_diff(prev, prev).item()) == 0.0             # unchanged (same buffer)
    assert float(pa.residual_diff(prev.clone(), prev).item()) == 0.0
    assert float(pa.residual_diff(-prev, prev).item()) == 2.0            # 2|p| summed as |p|, times 2
    z = torch.zeros_like(prev)
    assert float(pa.residual_diff(z, prev).item()) == 1.0                # vanished residual


def test_zero_conventions():
    z = torch.zeros(1000, dtype=torch.bfloat16, device="cuda")
    assert float(pa.residual_diff(z, z).item()) == 0.0
    assert float(pa.residual_diff(torch.ones_like(z), z).item()) == float("inf")


def test_deterministic_and_threshold_use():
    cur, prev = _pair(4096 * 3072, seed=5, noise=0.08)
    a = pa.residual_diff(cur, prev)
    b = pa.residual_diff(cur, prev)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    # the cache decision of the guide: reuse while the difference is below the threshold
    want = oracle_diff(cur, prev)
    assert (float(a.item()) < 0.08) == (want < 0.08) or abs(want - 0.08) < REL
