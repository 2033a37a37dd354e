"""Comparison helpers shared by the GPU parity tests.

Tolerances (the acceptance bar for floating point in this project): on O,
max |o_gpu - o_ref| <= 1e-2 and mean |o_gpu - o_ref| <= 1e-3; on LSE,
|lse_gpu - lse_ref| / max(|lse_ref|, 1) <= 1e-3 for every row.  As a
stricter diagnostic, the relative L2 error of O is also held
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


# e4m3 forward (pa_attn_fwd_fp8), against the oracle on the dequantised inputs.
# The inputs' own quantisation is exact on both sides; what remains is P
# rounded to e4m3 before P.V: a relative error of at most 2^-4 per weight,
# about 2^-4/sqrt(3) = 3.6% rms.  So O's error is bounded elementwise by
# 2^-4 * sum_j w_j |v_j| <= 2^-4 max|v| (plus the bf16 rounding of O,
# 2^-8 max|o| with margin), and on average it is a few per cent of |o|.  The
# bounds are therefore relative: relative L2 <= 6e-2, mean-abs <= 6e-2 of the
# mean |o_ref|, max-abs <= 2^-4 max|v| + 2^-8 max|o_ref|.  LSE uses the fp32
# exponentials and keeps the bf16 bound.
FP8_O_REL_L2 = 6e-2
FP8_O_MEAN_REL = 6e-2

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


def assert_close_fp8(o_gpu, lse_gpu, o_ref, lse_ref, v_max: float, what: str = "") -> dict:
    """The e4m3 bounds above; v_max = max |v| of the dequantised V."""
    e = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    RECORDED.append({"what": what, **e})
    o_ref = np.asarray(o_ref, dtype=np.float64)
    msg = f"{what}: {e}"
    assert e["finite"], msg
    assert e["o_max_abs"] <= 2.0 ** -4 * v_max + 2.0 ** -8 * float(np.abs(o_ref).max()), msg
    assert e["o_mean_abs"] <= FP8_O_MEAN_REL * float(np.abs(o_ref).mean()), msg
    assert e["lse_max_rel"] <= LSE_REL, msg
    assert e["o_rel_l2"] <= FP8_O_REL_L2, msg
    return e
