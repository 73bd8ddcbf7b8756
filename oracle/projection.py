"""The projections on either side of the attention core, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows "V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2", section
"Repository layout" (the attention block K2: QKV projection + RoPE, the
attention inner, the output projection) and "vit-encoder-neuron-kernels",
section "Kernels" (attention per head group with both RoPE pairings). The
pages fold LayerNorm affines into the weights, so each projection is a plain
affine map y = x W^T + b (a torch.nn.Linear), with every matmul in bf16:

  qkv projection: x [B, S, C] -> t = x W_qkv^T + b_qkv, t [B, S, 3 H D];
                  columns [0, HD) are Q, [HD, 2HD) K, [2HD, 3HD) V, and column
                  h D + d of each is head h, lane d, laid out as [B, H, S, D];
                  RoPE then rotates Q and K (rope.rope_apply), not V.
  out projection: o [B, H, S, D] -> the heads side by side, a[b, s, h D + d] =
                  o[b, h, s, d], then y = a W_o^T + b_o, y [B, S, C_out].

Readings (the pages give the block, not its interface): x is the bf16 input of
the block (the normalised residual stream, cast to bf16 as every matmul runs in
bf16); biases are fp32; Q, K, V come out in bf16 for the attention core; the
output projection's result stays in fp32, the precision of the residual stream
it is added to.
"""

from __future__ import annotations

import numpy as np

from .rope import rope_apply


def qkv_projection(x, w_qkv, b_qkv, H: int, D: int):
    """x [B, S, C], w_qkv [3 H D, C], b_qkv [3 H D] or None -> (q, k, v), each [B, H, S, D]."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    B, S, C = x.shape
    if w.shape != (3 * H * D, C):
        raise ValueError("w_qkv must be [3 H D, C]")
    t = x.reshape(B * S, C) @ w.T
    if b_qkv is not None:
        t = t + np.asarray(b_qkv, dtype=np.float64)[None, :]
    t = t.reshape(B, S, 3, H, D)
    q, k, v = (np.ascontiguousarray(t[:, :, i].transpose(0, 2, 1, 3)) for i in range(3))
    return q, k, v


def qkv_rope_projection(x, w_qkv, b_qkv, H: int, D: int, cos=None, sin=None, mode=None):
    """qkv_projection, then RoPE on q and k with [S, D/2] tables (none if mode is None)."""
    q, k, v = qkv_projection(x, w_qkv, b_qkv, H, D)
    if mode is not None:
        q = rope_apply(q, cos, sin, mode)
        k = rope_apply(k, cos, sin, mode)
    return q, k, v


def out_projection(o, w_o, b_o):
    """o [B, H, S, D], w_o [C_out, H D], b_o [C_out] or None -> y [B, S, C_out]."""
    o = np.asarray(o, dtype=np.float64)
    w = np.asarray(w_o, dtype=np.float64)
    B, H, S, D = o.shape
    if w.shape[1] != H * D:
        raise ValueError("w_o must be [C_out, H D]")
    a = o.transpose(0, 2, 1, 3).reshape(B * S, H * D)
    y = a @ w.T
    if b_o is not None:
        y = y + np.asarray(b_o, dtype=np.float64)[None, :]
    return y.reshape(B, S, w.shape[0])
