"""FP8 E4M3 ("e4m3fn") codec written from the OCP 8-bit floating point format.

Test infrastructure only (see the package docstring).

The pages say only "FP8 quantization for PV" (SageAttention README, "Current
Features"); the reading adopted is the E4M3 format of the OCP FP8 spec:

* bit 7 sign, bits 6..3 exponent E (bias 7), bits 2..0 mantissa M;
* E = 0:          value = M/8 * 2^-6            (subnormals, and +-0);
* E = 1..15:      value = (1 + M/8) * 2^(E - 7);
* E = 15, M = 7:  NaN (the only NaN pattern); there are no infinities;
* largest finite magnitude 448 (E = 15, M = 6).

Encoding is round-to-nearest, ties to the even code, with saturation to
+-448 for finite inputs beyond the range ("satfinite").  The encoder below
does this by brute force against the table of all 127 finite non-negative
values, so it follows the definition rather than any bit trick.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
NAN_CODE = 0x7F


def decode(code) -> np.ndarray:
    """Code(s) in 0..255 -> float64 values (NaN for the NaN patterns)."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * mag
    return np.where((e == 15) & (m == 7), np.nan, val)


# All finite non-negative values in code order; code i <-> _POS[i] for i in 0..126.
_POS = decode(np.arange(127))
assert np.all(np.diff(_POS) > 0)


def encode(x) -> np.ndarray:
    """float32/float64 array -> uint8 E4M3 codes (RNE, ties to even code, saturating).

    The sign bit is copied from the input, so negative values that round to
    zero give the negative-zero code 0x80, as IEEE conversion does.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # index of the largest table value <= a
    lo = np.searchsorted(_POS, a, side="right") - 1
    lo = np.clip(lo, 0, 126)
    hi = np.minimum(lo + 1, 126)
    vlo, vhi = _POS[lo], _POS[hi]
    mid = (vlo + vhi) / 2.0          # exact in float64
    pick_hi = (a > mid) | ((a == mid) & (lo % 2 == 1))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)       # saturate finite overflow
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), NAN_CODE, code)
    return code.astype(np.uint8)
