"""Closed-form work counts (oracle package; test infrastructure and bench accounting).

Attention FLOPs follow the accounting of the PCP history page ("Prefill
Context-Parallel Attention POC for Trainium2", section "Profiling-optimized
4-chip case" and the Q-scaling table after it): only the two matmuls count,
QK^T and PV, two flops per multiply-add:

    flops = 2 * Sq * Hq * L * D   (QK^T)  +  2 * Sq * Hq * L * D   (PV)
          = 4 * Sq * Hq * L * D

with L the number of keys each query attends to. The page's MFU figures are
reproduced exactly by this formula (pinned in tests/golden/pcp_mfu_table.txt).
"""

from __future__ import annotations


def attention_flops(batch: int, q_heads: int, q_len: int, kv_len: int, head_dim: int) -> float:
    return 4.0 * batch * q_heads * q_len * kv_len * head_dim


def decode_algorithmic_bytes(lengths, kv_heads: int, head_dim: int, q_heads: int,
                             s_ctx: int, kv_elem_bytes: int = 2, q_elem_bytes: int = 2,
                             out_elem_bytes: int = 2, mask_elem_bytes: int = 4) -> float:
    """Bytes a single-token decode must move: K and V of the valid positions,
    plus Q, O and the additive mask row of every batch entry."""
    B = len(lengths)
    kv = sum(int(x) for x in lengths) * kv_heads * head_dim * kv_elem_bytes * 2
    q = B * q_heads * head_dim * q_elem_bytes
    o = B * q_heads * head_dim * out_elem_bytes
    m = B * s_ctx * mask_elem_bytes
    return float(kv + q + o + m)
