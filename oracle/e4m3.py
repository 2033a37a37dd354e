"""e4m3 (OCP FP8 E4M3FN) rounding, written from the format's definition.

TEST INFRASTRUCTURE ONLY, under the same rules as ``blockwise.py``: used by
``tests/`` and nothing on the product path; it imports nothing from this
project.

The fp8 path applies the storage format that the diffusers "ParaAttention"
guide quantises activations to (its fp8 section) to the attention inputs.
The format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
Exponent fields 1..15 are normal numbers (1 + m/8) * 2^(e - 7); field 0 holds
the subnormals (m/8) * 2^-6.  The code with exponent 15 and mantissa 7 is NaN,
so the largest finite magnitude is 1.75 * 2^8 = 448; there is no infinity.

Quantisation as the library does it (the plain per-tensor reading):

    amax  = max |x|                      (x as given, bf16 values)
    scale = amax / 448   in float32      (scale = 1 when amax = 0)
    inv   = 448 / amax   in float32      (inv = 1 when amax = 0)
    y     = x * inv      in float32      (one multiply per element)
    code  = e4m3 nearest to y, ties to the even code, saturated to +-448

so that x ~= scale * decode(code).
"""

from __future__ import annotations

import numpy as np

__all__ = ["decode_table", "encode_rne", "quantize", "E4M3_MAX"]

E4M3_MAX = 448.0


def decode_table() -> np.ndarray:
    """float64 value of every code 0..255 (NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_POS = decode_table()[:0x7F]  # codes 0x00 .. 0x7E: 0 .. 448, increasing


def encode_rne(y) -> np.ndarray:
    """Nearest e4m3 code to each finite y, ties to the even code, magnitudes
    above 448 saturated to 448.  Returns uint8 codes; -0.0 gives 0x80."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")          # first value >= a
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    neg = np.signbit(y)
    return np.where(neg, code | np.uint8(0x80), code).astype(np.uint8)


def quantize(x) -> tuple:
    """(codes uint8, scale float32) for a tensor of bf16-representable values,
    in the steps listed in the module docstring."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    scale = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))
    inv = np.float32(1.0) if amax == 0 else np.float32(np.float32(E4M3_MAX) / amax)
    y = (x32 * inv).astype(np.float32)
    return encode_rne(y), scale
