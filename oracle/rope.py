"""Rotary position embedding (RoPE) applied to Q or K rows, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows "vit-encoder-neuron-kernels", section "Kernels": the encoder attention
takes per-token rotation tables, and the two supported pairings of head-dim
lanes are
  * "half":        lane j pairs with lane j + D/2   (DINOv3, EVA-02, HF Llama),
  * "interleaved": lane 2j pairs with lane 2j + 1   (V-JEPA2).
A pair (a, b) at token position s, pair index j, is rotated by the angle whose
cosine and sine the tables hold at [s, j]:
    a' = a cos - b sin,   b' = a sin + b cos.
The page's tables come from the model (V-JEPA2 builds them from a 3-D
time / height / width grid); here they are inputs, [S, D/2] each.
"""

from __future__ import annotations

import numpy as np


def pair_lanes(D: int, mode: str):
    """(first, second) lane index of every pair j = 0 .. D/2 - 1."""
    j = np.arange(D // 2)
    if mode == "half":
        return j, j + D // 2
    if mode == "interleaved":
        return 2 * j, 2 * j + 1
    raise ValueError(f"unknown RoPE pairing {mode!r}")


def rope_apply(x, cos, sin, mode: str) -> np.ndarray:
    """x [..., S, D] (any float type, read exactly) -> rotated copy in float64.

    cos, sin: [S, D/2]; row s of x is rotated with row s of the tables."""
    x = np.asarray(x, dtype=np.float64)
    cos = np.asarray(cos, dtype=np.float64)
    sin = np.asarray(sin, dtype=np.float64)
    D = x.shape[-1]
    if D % 2 or cos.shape != (x.shape[-2], D // 2) or sin.shape != cos.shape:
        raise ValueError("tables must be [S, D/2] for x [..., S, D]")
    ia, ib = pair_lanes(D, mode)
    a, b = x[..., ia], x[..., ib]
    out = np.empty_like(x)
    out[..., ia] = a * cos - b * sin
    out[..., ib] = a * sin + b * cos
    return out
