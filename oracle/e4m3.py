"""FP8 E4M3FN decoder, written from the format definition (oracle; test infrastructure only).

The history-attention page ("Prefill Context-Parallel Attention POC for
Trainium2", section "Current POC constraints") stores K/V as FP8 E4M3FN. That
format (OCP 8-bit floating point, "FN" = finite, no infinities) is:

  bit 7      sign s
  bits 6..3  exponent e, bias 7
  bits 2..0  mantissa m

  e == 0              -> subnormal: (-1)^s * 2^(1-7) * (m / 8)
  0 < e, not all-ones -> normal:    (-1)^s * 2^(e-7) * (1 + m / 8)
  e == 15, m < 7      -> normal as above (the FN variant reuses the top binade)
  e == 15, m == 7     -> NaN (codes 0x7F and 0xFF); there is no infinity.

So the largest finite magnitude is 2^8 * 1.75 = 448 and the smallest
subnormal is 2^-9.
"""

from __future__ import annotations

import numpy as np


def _decode_one(code: int) -> float:
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    sign = -1.0 if s else 1.0
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (2.0 ** (1 - 7)) * (m / 8.0)
    return sign * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


# 256-entry table built by evaluating the definition above code by code.
E4M3FN_TABLE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)


def e4m3fn_to_float64(codes: np.ndarray) -> np.ndarray:
    """Decode an array of E4M3FN byte codes (uint8) to exact float64 values."""
    codes = np.asarray(codes)
    if codes.dtype != np.uint8:
        raise TypeError("e4m3fn codes must be uint8")
    return E4M3FN_TABLE[codes]
