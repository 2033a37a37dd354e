"""fp64 CPU oracle for First Block Cache's residual difference.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: it is used by ``tests/`` and by ``bench.py``'s CPU legs.
It shares no code with the CUDA library and imports nothing from this
project.

What it computes, and the passage it follows
--------------------------------------------
The diffusers "ParaAttention" guide, section "First Block Cache": the change
of the model's output between two denoising steps is approximated by the
difference of the residual output of the first transformer block between the
two steps, and the cached residuals are reused while that difference is
small enough (a threshold, 0.08 by default for FLUX models).  The guide
gives no formula; the reading taken here is the plainest one with a
dimensionless threshold, the relative L1 difference

    diff = sum_i |cur_i - prev_i| / sum_i |prev_i|

(equivalently mean |cur - prev| / mean |prev|) over every element of the two
residual tensors, with diff = 0 when both sums are 0 and +inf when only the
denominator is.

Inputs are the exact values the GPU receives (bf16 upcast to float64).
"""

import numpy as np


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").double().numpy()
    except ImportError:
        pass
    return np.asarray(x, dtype=np.float64)


def residual_diff(cur, prev) -> float:
    """sum |cur - prev| / sum |prev| in float64 (see the module docstring)."""
    c = _f64(cur).reshape(-1)
    p = _f64(prev).reshape(-1)
    if c.shape != p.shape:
        raise ValueError("cur and prev must have the same number of elements")
    num = float(np.abs(c - p).sum())
    den = float(np.abs(p).sum())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den
