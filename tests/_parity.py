"""Comparison helpers shared by the GPU parity tests.

Tolerances (the acceptance bar for floating point, stated by the task's
workload definition): on O, max |o_gpu - o_ref| <= 1e-2 and mean |o_gpu -
o_ref| <= 1e-3; on LSE, |lse_gpu - lse_ref| / max(|lse_ref|, 1) <= 1e-3 for
every row.  As a stricter diagnostic, the relative L2 error of O is also held
to <= 1e-2 (derivation: P is rounded to bf16 before P.V, a relative error of
at most 2^-9 per weight that averages out over keys, and O is rounded to bf16
on output, 2^-9 relative; together well under 1e-2).
"""

from __future__ import annotations

import numpy as np

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_REL = 1e-3
O_REL_L2 = 1e-2


def errors(o_gpu, lse_gpu, o_ref, lse_ref) -> dict:
    o = o_gpu.detach().float().cpu().double().numpy() if hasattr(o_gpu, "detach") else np.asarray(o_gpu, float)
    l = lse_gpu.detach().cpu().double().numpy() if hasattr(lse_gpu, "detach") else np.asarray(lse_gpu, float)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert l.shape == lse_ref.shape, (l.shape, lse_ref.shape)
    d = np.abs(o - o_ref)
    both_ninf = np.isneginf(l) & np.isneginf(lse_ref)
    lrel = np.where(both_ninf, 0.0, np.abs(l - lse_ref) / np.maximum(np.abs(lse_ref), 1.0))
    return {
        "o_max_abs": float(d.max()) if d.size else 0.0,
        "o_mean_abs": float(d.mean()) if d.size else 0.0,
        "o_rel_l2": float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30)) if d.size else 0.0,
        "lse_max_rel": float(lrel.max()) if lrel.size else 0.0,
        "finite": bool(np.all(np.isfinite(o)) and np.all(np.isfinite(l) | both_ninf)),
    }


# Every comparison made in this session, in order (written out by conftest.py
# when PA_PARITY_REPORT names a file).
RECORDED: list = []


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, what: str = "") -> dict:
    e = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    RECORDED.append({"what": what, **e})
    msg = f"{what}: {e}"
    assert e["finite"], msg
    assert e["o_max_abs"] <= O_MAX_ABS, msg
    assert e["o_mean_abs"] <= O_MEAN_ABS, msg
    assert e["lse_max_rel"] <= LSE_REL, msg
    assert e["o_rel_l2"] <= O_REL_L2, msg
    return e
