"""Float64 replay of the paged FP8 kernel's roundings (oracle; test infrastructure only).

Tensor cores multiply FP8 only by FP8, while the history-attention page ("Prefill
Context-Parallel Attention POC for Trainium2", "Current POC constraints") keeps Q
and the softmax numerator in bf16 against FP8 K / V. The kernel therefore writes
the bf16 operand of each matmul as two E4M3FN terms, x ~ hi + lo with
hi = e4m3(x) and lo = e4m3(x - hi), each term a separate FP8 MMA into the same
fp32 accumulator:

  * Q row r is scaled by sq_r = amax_r / 448 before the split (S = sq_r (Qh + Ql) K^T);
  * P = 2^(s - m) in fp32, times 2^7, rounded to f16, then hi = e4m3(P), lo =
    e4m3(f16(P - hi)); the running max is refreshed only when it grows by more
    than 1 (log2 units), so P * 2^7 <= 256 < 448 stays in range.

This module replays those steps in the same order with plain NumPy roundings
(E4M3FN nearest-even from the format's value table, IEEE f16 / f32 casts), so the
error of each design choice -- both splits, one, or none -- can be measured
against the exact attention on the CPU. It shares no code with the kernel.
"""

from __future__ import annotations

import numpy as np

from .e4m3 import E4M3FN_TABLE

_FINITE = np.sort(np.unique(np.abs(E4M3FN_TABLE[np.isfinite(E4M3FN_TABLE)])))   # 0 .. 448
_CODES_OF = {float(v): c for c, v in enumerate(E4M3FN_TABLE) if np.isfinite(v) and v >= 0}


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3FN value, ties to the even code, saturating at +-448 (values as float64)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), _FINITE[-1])
    i = np.clip(np.searchsorted(_FINITE, a), 1, len(_FINITE) - 1)
    lo, hi = _FINITE[i - 1], _FINITE[i]
    pick_hi = (hi - a) < (a - lo)
    tie = (hi - a) == (a - lo)
    hi_even = np.array([_CODES_OF[float(v)] % 2 == 0 for v in hi.ravel()]).reshape(hi.shape)
    r = np.where(pick_hi | (tie & hi_even), hi, lo)
    r = np.where(a >= _FINITE[-1], _FINITE[-1], r)
    return np.copysign(r, x)


def f16_round(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def f32_round(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def paged_history_emulated(q, k_vals, v_vals, k_scale, v_scale, softmax_scale, split_q=True,
                           split_p=True, p_scale_log2=7.0, threshold=1.0, tile=128):
    """Replay of the kernel for one query head against one kv head.

    q [Sq, D] (bf16 values); k_vals, v_vals [L, D]: the decoded E4M3FN code values
    (unscaled) of the history in logical order. Returns out [Sq, D] as the kernel
    would produce it before its final bf16 rounding."""
    q = np.asarray(q, dtype=np.float64)
    amax = np.abs(q).max(axis=1, keepdims=True)
    sq = np.where(amax > 0, amax / 448.0, 1.0)
    qh = e4m3_round(q / sq)
    ql = e4m3_round(q / sq - qh) if split_q else np.zeros_like(qh)
    c_row = sq[:, 0] * k_scale * softmax_scale * np.log2(np.e)
    p_scale = 2.0 ** p_scale_log2
    m = np.full(q.shape[0], -np.inf)
    l = np.zeros(q.shape[0])
    o = np.zeros_like(q)
    for j0 in range(0, k_vals.shape[0], tile):
        K, V = k_vals[j0:j0 + tile], v_vals[j0:j0 + tile]
        s = f32_round(qh @ K.T + ql @ K.T) * c_row[:, None]
        mt = s.max(axis=1)
        upd = mt > m + threshold
        mn = np.where(upd, mt, m)
        alpha = np.where(upd, np.exp2(m - mn), 1.0)
        p = f32_round(np.exp2(s - mn[:, None]))
        l = l * alpha + p.sum(axis=1)
        o *= alpha[:, None]
        m = mn
        ps = f16_round(p * p_scale)
        ph = e4m3_round(ps)
        pl = e4m3_round(f16_round(ps - ph)) if split_p else np.zeros_like(ph)
        o += (ph + pl) @ V
    return o * v_scale / (p_scale * l[:, None])


def bf16_round(x) -> np.ndarray:
    """Round to bf16 (nearest even), values returned as float64."""
    a = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def encoder_row_emulated(s_row, v, threshold, tile=128):
    """Online softmax of one query row as the encoder's softmax warps run it.

    s_row [L]: the row's scores already in log2 units (scale * log2 e folded in);
    v [L, D]. Per 128-key tile: the running max m moves only when the tile's max
    exceeds it by more than `threshold`; P = 2^(s - m) is rounded to bf16 for the
    P.V product while the row sum l accumulates the unrounded fp32 values; O is
    rescaled by 2^(m_old - m_new) when m moves. Returns O / l (before the final
    bf16 rounding)."""
    m, l = -np.inf, 0.0
    o = np.zeros(v.shape[1])
    for j0 in range(0, s_row.shape[0], tile):
        s = s_row[j0:j0 + tile]
        mt = s.max()
        if mt > m + threshold:
            alpha = np.exp2(m - mt) if np.isfinite(m) else 0.0
            l *= alpha
            o *= alpha
            m = mt
        p = f32_round(np.exp2(s - m))
        l += p.sum()
        o += bf16_round(p) @ v[j0:j0 + tile]
    return o / l
