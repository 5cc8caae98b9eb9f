"""MXFP8 (E4M3 elements, one power-of-two scale per 32-element block) quantisation.

TEST INFRASTRUCTURE ONLY (see the package docstring).  The torchtitan page lists
MXFP8 routed experts as a training option; this module states the block-scaled format
the way the OCP Microscaling (MX) v1.0 specification defines it, so that a future
MXFP8 expert path can be compared against an oracle that quantises the same values by
the same rule (the products of two quantised values are exact in float64, so parity
then reduces to accumulation order).

Format (OCP MX v1.0, "MXFP8 (E4M3)"):
  * element: FP8 E4M3 - 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
    infinities; the largest finite magnitude is 1.75 * 2^8 = 448, the smallest normal
    2^-6, subnormals are k * 2^-9 for k = 1..7;
  * block: 32 consecutive elements along the reduction axis share one E8M0 scale
    X = 2^s (an 8-bit biased exponent, s in [-127, 127]);
  * scale choice: s = floor(log2(max |v| over the block)) - 8, where 8 is the largest
    exponent of an E4M3 normal, so the block's largest magnitude lands in [256, 512)
    before its element conversion;
  * element conversion: round to nearest, ties to even; magnitudes above 448 (the
    [448, 512) range the scale choice can produce) clamp to 448 - the reading taken
    here, since the format has no infinity and the specification leaves overflow
    handling to the implementation; an all-zero block takes s = -127.
"""
from __future__ import annotations

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_round", "mx_block_exponent", "quantize_mxfp8", "dequantize_mxfp8"]

E4M3_MAX = 448.0          # 1.75 * 2^8
_E4M3_EMIN = -6           # exponent of the smallest normal
_E4M3_EMAX = 8            # exponent of the largest normal
_MANT_BITS = 3
MX_BLOCK = 32


def _round_half_even(v: np.ndarray) -> np.ndarray:
    """Nearest integer, ties to the even one (numpy's rint does exactly this)."""
    return np.rint(v)


def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value to each element of v (float64 in, float64 out), ties to even,
    magnitudes above 448 clamped to 448; NaN stays NaN."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    nz = a > 0
    # exponent of the binade each magnitude falls in, never below the subnormal range's
    e = np.full_like(a, _E4M3_EMIN)
    e[nz] = np.maximum(np.floor(np.log2(a[nz])), _E4M3_EMIN)
    e = np.minimum(e, _E4M3_EMAX)
    quantum = np.exp2(e - _MANT_BITS)              # spacing of representable values there
    out = _round_half_even(a / quantum) * quantum
    out = np.minimum(out, E4M3_MAX)
    out = np.where(np.isnan(v), np.nan, np.copysign(out, v))
    return out


def mx_block_exponent(amax) -> np.ndarray:
    """E8M0 scale exponent s of a block whose largest magnitude is amax (see the module
    docstring): floor(log2 amax) - 8, clamped to [-127, 127]; -127 for an all-zero block."""
    amax = np.asarray(amax, dtype=np.float64)
    s = np.full(amax.shape, -127, dtype=np.int64)
    pos = amax > 0
    s[pos] = np.floor(np.log2(amax[pos])).astype(np.int64) - _E4M3_EMAX
    return np.clip(s, -127, 127)


def quantize_mxfp8(x, axis: int = -1):
    """Quantise x along `axis` (its length a multiple of 32) to MXFP8.  Returns
    (q, s): q has x's shape and holds E4M3 values, s has one int exponent per block
    (x's shape with `axis` divided by 32); the represented value is q * 2^s."""
    x = np.moveaxis(np.asarray(x, dtype=np.float64), axis, -1)
    n = x.shape[-1]
    if n % MX_BLOCK:
        raise ValueError("the blocked axis must be a multiple of 32")
    xb = x.reshape(x.shape[:-1] + (n // MX_BLOCK, MX_BLOCK))
    s = mx_block_exponent(np.abs(xb).max(axis=-1))
    q = e4m3_round(xb / np.exp2(s)[..., None])
    q = np.moveaxis(q.reshape(x.shape), -1, axis)
    s = np.moveaxis(s, -1, axis)
    return q, s


def dequantize_mxfp8(q, s, axis: int = -1) -> np.ndarray:
    """q * 2^s, the scale broadcast over each block of 32 along `axis`."""
    q = np.moveaxis(np.asarray(q, dtype=np.float64), axis, -1)
    s = np.moveaxis(np.asarray(s), axis, -1)
    scale = np.repeat(np.exp2(s.astype(np.float64)), MX_BLOCK, axis=-1)
    return np.moveaxis(q * scale, -1, axis)
