"""CPU fp64 oracle for the online-softmax attention forward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call, link or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s ``cpu_baseline`` leg (and its ``--impl reference`` arm) use
it. The oracle shares no code with the CUDA library: it reads the same stored
input bits (bf16, fp32, e4m3fn bytes) and evaluates the plain definition

    out = softmax(softmax_scale * Q K^T + additive_mask) V

in float64, two passes per query row (row max, then exp / sum / P V).

Modules
-------
attention   -- the definition for the entry points (encoder, GQA decode, paged
               history, paged prefill with causal current tokens) plus the
               split-KV log-sum-exp combine.
e4m3        -- an FP8 E4M3FN decoder written from the format definition.
rope        -- rotary position embedding of Q / K rows (both lane pairings).
projection  -- the QKV projection (+ RoPE) and the output projection around the
               attention core.
precision_model -- float64 replay of the paged FP8 kernel's roundings (hi / lo e4m3
               splits), used to measure that design choice on the CPU.
flops       -- the closed-form work counts used for throughput figures.
"""

from .attention import (  # noqa: F401
    softmax_attention,
    encoder_attention,
    gqa_decode_attention,
    paged_history_attention,
    paged_prefill_attention,
    paged_logical_kv,
    lse_combine,
)
from .e4m3 import e4m3fn_to_float64  # noqa: F401
from .rope import rope_apply, pair_lanes  # noqa: F401
from .projection import qkv_projection, qkv_rope_projection, out_projection  # noqa: F401
from .flops import attention_flops, decode_algorithmic_bytes  # noqa: F401
