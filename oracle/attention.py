"""Plain float64 softmax attention: the definition the three entry points compute.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

The method on the pages is exact softmax attention evaluated tile by tile with a
running ("online") max and sum, so the oracle is the plain definition written
out, with no tiling, no running state and no reordering:

    s[i, j] = softmax_scale * sum_d q[i, d] * k[j, d] + mask[i, j]
    m[i]    = max_j s[i, j]                       (pass 1)
    p[i, j] = exp(s[i, j] - m[i])                 (pass 2)
    l[i]    = sum_j p[i, j]
    o[i, :] = sum_j p[i, j] * v[j, :] / l[i]

Passages followed:
  * "head_dim>128 (256/512) GQA Flash-Decode NKI Kernel for AWS Trainium",
    section "Input contract": q [B, Hq, 1, D], k/v [B, Hkv, S_ctx, D],
    attn_mask [B, 1, 1, S_ctx] additive (0 keep, -inf mask), softmax_scale,
    num_kv_groups = Hq // Hkv; and the sentence after it: flash online-softmax
    accumulation over K tiles (the tiling is the GPU's business, not the
    oracle's).
  * "Prefill Context-Parallel Attention POC for Trainium2", sections "Layout"
    (Q [Hq, q_len, D], K/V [blocks, Hkv, block_size, D], O [Hq, q_len, D]),
    the history-only rule (queries attend to history only, no causal mask),
    the additive bias derived from actual_history_len, and "Current POC
    constraints" (FP8 E4M3FN K/V, fp32 max/sum).

Readings where the pages are silent (each is also listed in the design notes):
  * GQA mapping: query head h reads kv head h // num_kv_groups (contiguous
    groups; "Q heads sharing a KV head are packed" on the history page).
  * A -inf mask entry removes the key outright (s = -inf whatever q.k is).
  * A row whose every key is masked has l = 0; its output is defined as 0 and
    its log-sum-exp as -inf.
  * softmax_scale multiplies Q K^T before the additive mask is added.
"""

from __future__ import annotations

import numpy as np

from .e4m3 import e4m3fn_to_float64

_ROW_CHUNK = 256  # query rows per matmul; rows are independent, so chunking rows changes nothing


def _as_f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _weighted_rows(p, v_head, removed):
    """num[i] = sum over the keys j that row i keeps of p[i, j] * v[j].

    A removed key (score -inf) takes no part at all, so its V row is never
    multiplied, not even by p = 0: a non-finite V row at a removed position
    (an unwritten cache slot) leaves the result finite, while one at a kept
    position propagates as the definition says.
    """
    bad = ~np.isfinite(v_head).all(axis=1)        # keys whose V row holds NaN / inf
    if not bad.any():
        return p @ v_head
    v_fin = np.where(bad[:, None], 0.0, v_head)
    num = p @ v_fin
    for j in np.flatnonzero(bad):
        kept = ~removed[:, j]
        num[kept] += p[kept, j][:, None] * v_head[j][None, :]
    return num


def _rows_attention(q_rows, k_head, v_head, softmax_scale, mask_rows):
    """Two-pass softmax attention for a block of query rows against one kv head.

    q_rows [R, D], k_head/v_head [L, D], mask_rows [R, L] or [1, L] or None.
    Returns (o [R, D], lse [R]) in float64; lse = m + log(l).
    """
    with np.errstate(invalid="ignore"):                         # NaN rows of removed keys
        s = softmax_scale * (q_rows @ k_head.T)                 # scores
    if mask_rows is not None:
        s = np.where(np.isneginf(mask_rows), -np.inf, s + mask_rows)
    m = s.max(axis=1) if s.shape[1] > 0 else np.full(s.shape[0], -np.inf)
    live = np.isfinite(m)
    m_safe = np.where(live, m, 0.0)
    p = np.exp(s - m_safe[:, None])                             # exp(-inf) = 0 for removed keys
    l = p.sum(axis=1)
    num = _weighted_rows(p, v_head, np.isneginf(s))
    o = np.zeros_like(num)
    nz = l > 0
    o[nz] = num[nz] / l[nz, None]
    with np.errstate(divide="ignore"):
        lse = np.where(nz, m_safe + np.log(np.where(nz, l, 1.0)), -np.inf)
    return o, lse


def softmax_attention(q, k, v, softmax_scale, num_kv_groups=1, mask=None,
                      return_lse=False, rows=None):
    """out[b, h] = softmax(softmax_scale * q[b,h] k[b,g]^T + mask[b,h]) v[b,g], g = h // groups.

    q [B, Hq, Sq, D]; k, v [B, Hkv, L, D]; mask additive, broadcastable to
    [B, Hq, Sq, L] (None = no mask). ``rows`` optionally restricts the query
    rows evaluated (an index array into Sq); the result then has Sq = len(rows).
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, L, Dk = k.shape
    if Bk != B or Dk != D or v.shape != k.shape:
        raise ValueError("shape mismatch between q, k, v")
    if Hq != Hkv * num_kv_groups:
        raise ValueError("num_q_heads must equal num_kv_heads * num_kv_groups")
    row_idx = np.arange(Sq) if rows is None else np.asarray(rows)
    if mask is not None:
        mask = np.broadcast_to(_as_f64(mask), (B, Hq, Sq, L))
    out = np.zeros((B, Hq, len(row_idx), D), dtype=np.float64)
    lse = np.zeros((B, Hq, len(row_idx)), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // num_kv_groups
            for c0 in range(0, len(row_idx), _ROW_CHUNK):
                ridx = row_idx[c0:c0 + _ROW_CHUNK]
                mrows = None if mask is None else mask[b, h][ridx]
                o, ls = _rows_attention(q[b, h][ridx], k[b, g], v[b, g], softmax_scale, mrows)
                out[b, h, c0:c0 + len(ridx)] = o
                lse[b, h, c0:c0 + len(ridx)] = ls
    return (out, lse) if return_lse else out


def encoder_attention(q, k, v, softmax_scale, key_bias=None, rows=None):
    """Non-causal multi-head encoder attention (the ViT / NewBERT encoder pages).

    q, k, v [B, H, S, D]; key_bias optional [B, S] additive per-key bias
    (a 0 / -inf right-padding mask is the special case the gte page uses).
    """
    mask = None
    if key_bias is not None:
        kb = _as_f64(key_bias)
        mask = kb[:, None, None, :]
    return softmax_attention(q, k, v, softmax_scale, 1, mask, rows=rows)


def gqa_decode_attention(q, k, v, attn_mask, softmax_scale, num_kv_groups, return_lse=False):
    """Single-token GQA decode per the decode page's input contract.

    q [B, Hq, 1, D]; k, v [B, Hkv, S_ctx, D]; attn_mask [B, 1, 1, S_ctx] or None.
    """
    return softmax_attention(q, k, v, softmax_scale, num_kv_groups, attn_mask,
                             return_lse=return_lse)


def paged_logical_kv(k_codes, v_codes, k_scale, v_scale, block_table, block_size,
                     actual_history_len):
    """Gather the logical history K/V (float64) through the block table.

    k_codes, v_codes: uint8 E4M3FN codes [num_phys_blocks, Hkv, block_size, D].
    Logical position t < actual_history_len lives in physical block
    block_table[t // block_size] at offset t % block_size; its value is the
    decoded code times the per-tensor scale. Returns K, V as [Hkv, L, D].
    """
    k_codes = np.asarray(k_codes)
    v_codes = np.asarray(v_codes)
    table = np.asarray(block_table, dtype=np.int64)
    L = int(actual_history_len)
    t = np.arange(L)
    phys = table[t // block_size]
    off = t % block_size
    # [L, Hkv, D] -> [Hkv, L, D]
    kl = e4m3fn_to_float64(k_codes[phys, :, off, :]).transpose(1, 0, 2) * float(k_scale)
    vl = e4m3fn_to_float64(v_codes[phys, :, off, :]).transpose(1, 0, 2) * float(v_scale)
    return kl, vl


def paged_history_attention(q, k_codes, v_codes, k_scale, v_scale, block_table, block_size,
                            actual_history_len, softmax_scale, num_kv_groups, rows=None):
    """History-only attention over a paged FP8 cache (the PCP history page).

    q [Hq, Sq, D] (bf16 values as float64). Every query attends to every
    logical history position < actual_history_len; nothing else. Returns
    [Hq, Sq or len(rows), D].
    """
    kl, vl = paged_logical_kv(k_codes, v_codes, k_scale, v_scale, block_table, block_size,
                              actual_history_len)
    out = softmax_attention(_as_f64(q)[None], kl[None], vl[None], softmax_scale,
                            num_kv_groups, None, rows=rows)
    return out[0]


def paged_prefill_attention(q, k_codes, v_codes, k_scale, v_scale, block_tables, block_size,
                            q_start, hist_lens, softmax_scale, num_kv_groups, rows=None):
    """Prefill attention over a paged FP8 cache: history plus the current tokens, causal
    among the current tokens (the PCP history page's "current tokens do not attend to one
    another yet", completed; several sequences per call).

    q [Hq, total_q, D]: the current tokens of num_seqs sequences, packed; sequence s owns
    rows q_start[s] .. q_start[s+1] - 1. Its K/V, history and current tokens alike, sit in
    the cache at logical positions 0 .. hist_lens[s] + q_len_s - 1 of block_tables[s].
    Query i of sequence s is at logical position hist_lens[s] + i and attends to every
    position t <= hist_lens[s] + i. ``rows`` optionally restricts the evaluated rows of
    each sequence (indices into 0 .. q_len_s - 1, those past q_len_s are skipped); the
    result keeps the [Hq, total_q, D] layout with unevaluated rows left 0.
    """
    q = _as_f64(q)
    Hq, total_q, D = q.shape
    out = np.zeros_like(q)
    starts = [int(x) for x in q_start]
    for s, hist in enumerate(int(x) for x in hist_lens):
        a, b = starts[s], starts[s + 1]
        n = b - a
        if n == 0:
            continue
        kl, vl = paged_logical_kv(k_codes, v_codes, k_scale, v_scale, block_tables[s],
                                  block_size, hist + n)
        i = np.arange(n)[:, None]
        t = np.arange(hist + n)[None, :]
        mask = np.where(t <= hist + i, 0.0, -np.inf)[None, None]
        r = np.arange(n) if rows is None else np.asarray([x for x in rows if x < n], dtype=np.int64)
        o = softmax_attention(q[None, :, a:b], kl[None], vl[None], softmax_scale, num_kv_groups,
                              mask, rows=r)
        out[:, a + r] = o[0]
    return out


def lse_combine(o_parts, m_parts, l_parts):
    """Combine split-KV partial results of one query row.

    o_parts [n, D] are the UNNORMALISED partial numerators sum_j p_ij v_j of
    each key split, computed against that split's own max m_parts[n]; l_parts
    [n] are the matching partial sums. With M = max_i m_i:
        out = sum_i e^(m_i - M) o_i / sum_i e^(m_i - M) l_i
    Splits with m_i = -inf (every key masked) contribute nothing; if all are
    -inf the output is 0.
    """
    o_parts = _as_f64(o_parts)
    m_parts = _as_f64(m_parts)
    l_parts = _as_f64(l_parts)
    M = m_parts.max() if m_parts.size else -np.inf
    if not np.isfinite(M):
        return np.zeros(o_parts.shape[-1])
    w = np.where(np.isneginf(m_parts), 0.0, np.exp(m_parts - M))
    den = (w * l_parts).sum()
    if den == 0:
        return np.zeros(o_parts.shape[-1])
    return (w[:, None] * o_parts).sum(axis=0) / den
