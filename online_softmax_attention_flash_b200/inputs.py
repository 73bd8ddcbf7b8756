"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic. Everything is generated on the CPU with a seeded
``torch.Generator`` (fp32 N(0,1) draws rounded to bf16 with round-to-nearest-
even, or quantised to FP8 E4M3FN with a per-tensor scale), so that the CUDA
path and the CPU oracle read exactly the same stored bits.

The shapes mirror the workloads on the pages:
  * "tiny":   B=1, H=4,  S=256,  D=64  non-causal MHA, scale 1/8.
  * "vitl":   B=1, H=16, S=2048, D=64  (V-JEPA2 ViT-L, 16 frames = 2048 tokens),
              24 layers = 24 independent calls with seeds 2000 + layer.
  * "dinov3": B=8, H=16, S=201,  D=64  (ViT-L/16 at 224 px: 1 CLS + 4 register +
              196 patch tokens).
  * "decode": B=8, Hq=16, Hkv=8, D=256, S_ctx=4096, scale 1.0, per-batch valid
              length uniform in [128, 4096], additive 0 / -inf mask.
  * "paged":  32 Q heads x 4096 query tokens, 2 KV heads, D=256, bf16 Q; a pool of
              256 blocks x 512 tokens of E4M3FN K/V, a seeded permutation block
              table, actual_history_len = 100000, scale 1/16.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

E4M3FN_MAX = 448.0


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, g: torch.Generator) -> torch.Tensor:
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def quantize_e4m3fn(x: torch.Tensor):
    """Per-tensor scale amax / 448, round-to-nearest-even, saturating cast.

    Returns (codes uint8, scale float). The stored cache is codes * scale.
    """
    amax = float(x.abs().max())
    scale = amax / E4M3FN_MAX if amax > 0 else 1.0
    scale = float(torch.tensor(scale, dtype=torch.float32))  # the scale is an fp32 value
    codes = (x / scale).clamp(-E4M3FN_MAX, E4M3FN_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale


@dataclass
class EncoderCase:
    q: torch.Tensor            # [B, H, S, D] bf16
    k: torch.Tensor
    v: torch.Tensor
    softmax_scale: float
    key_bias: Optional[torch.Tensor] = None   # [B, S] fp32 additive, or None


def encoder_case(B, H, S, D, seed, softmax_scale=0.125, pad_lengths=None) -> EncoderCase:
    """N(0,1) bf16 q, k, v. ``pad_lengths`` (one per batch entry) adds a 0/-inf
    right-padding key bias, the gte page's 0/1 attention_mask as an additive bias."""
    g = _gen(seed)
    q = randn_bf16((B, H, S, D), g)
    k = randn_bf16((B, H, S, D), g)
    v = randn_bf16((B, H, S, D), g)
    kb = None
    if pad_lengths is not None:
        kb = torch.zeros((B, S), dtype=torch.float32)
        for b, n in enumerate(pad_lengths):
            kb[b, int(n):] = float("-inf")
    return EncoderCase(q, k, v, float(softmax_scale), kb)


@dataclass
class DecodeCase:
    q: torch.Tensor            # [B, Hq, 1, D] bf16
    k: torch.Tensor            # [B, Hkv, S_ctx, D] bf16
    v: torch.Tensor
    attn_mask: Optional[torch.Tensor]   # [B, 1, 1, S_ctx] fp32 additive (0 keep, -inf drop)
    lengths: torch.Tensor      # [B] int64 valid lengths used to build the mask
    softmax_scale: float
    num_kv_groups: int


def decode_case(B, Hq, Hkv, S_ctx, D, seed, softmax_scale=1.0, min_len=128,
                max_len=None, lengths=None) -> DecodeCase:
    g = _gen(seed)
    max_len = S_ctx if max_len is None else max_len
    if lengths is None:
        lengths = torch.randint(min_len, max_len + 1, (B,), generator=g, dtype=torch.int64)
    else:
        lengths = torch.as_tensor(lengths, dtype=torch.int64)
    q = randn_bf16((B, Hq, 1, D), g)
    k = randn_bf16((B, Hkv, S_ctx, D), g)
    v = randn_bf16((B, Hkv, S_ctx, D), g)
    mask = torch.zeros((B, 1, 1, S_ctx), dtype=torch.float32)
    for b in range(B):
        mask[b, :, :, int(lengths[b]):] = float("-inf")
    return DecodeCase(q, k, v, mask, lengths, float(softmax_scale), Hq // Hkv)


@dataclass
class PagedCase:
    q: torch.Tensor            # [Hq, Sq, D] bf16
    k_cache: torch.Tensor      # [num_phys_blocks, Hkv, block_size, D] uint8 (E4M3FN codes)
    v_cache: torch.Tensor
    k_scale: float
    v_scale: float
    block_table: torch.Tensor  # [n_table] int32, logical block -> physical block
    block_size: int
    actual_history_len: int
    softmax_scale: float
    num_kv_groups: int


def paged_case(Hq, Hkv, Sq, D, num_phys_blocks, block_size, actual_history_len, seed,
               softmax_scale=None, n_table=None) -> PagedCase:
    g = _gen(seed)
    n_table = num_phys_blocks if n_table is None else n_table
    q = randn_bf16((Hq, Sq, D), g)
    kf = torch.randn((num_phys_blocks, Hkv, block_size, D), generator=g, dtype=torch.float32)
    vf = torch.randn((num_phys_blocks, Hkv, block_size, D), generator=g, dtype=torch.float32)
    kc, ks = quantize_e4m3fn(kf)
    vc, vs = quantize_e4m3fn(vf)
    perm = torch.randperm(num_phys_blocks, generator=g)[:n_table].to(torch.int32).contiguous()
    scale = (1.0 / D ** 0.5) if softmax_scale is None else float(softmax_scale)
    return PagedCase(q, kc, vc, ks, vs, perm, block_size, int(actual_history_len), scale,
                     Hq // Hkv)


@dataclass
class PagedPrefillCase:
    q: torch.Tensor            # [Hq, total_q, D] bf16, the sequences' current tokens packed
    k_cache: torch.Tensor      # [num_phys_blocks, Hkv, block_size, D] uint8 (E4M3FN codes)
    v_cache: torch.Tensor
    k_scale: float
    v_scale: float
    block_tables: torch.Tensor  # [num_seqs, max_blocks] int32 (-1 past each sequence's blocks)
    block_size: int
    q_start: torch.Tensor      # [num_seqs + 1] int32, row offsets into q
    hist_lens: torch.Tensor    # [num_seqs] int32
    softmax_scale: float
    num_kv_groups: int


def paged_prefill_case(Hq, Hkv, D, block_size, hist_lens, q_lens, seed, softmax_scale=None,
                       spare_blocks=3) -> PagedPrefillCase:
    """Sequences with the given history and current lengths; each owns a disjoint random set
    of physical blocks covering hist + q_len positions (current tokens' K/V included)."""
    g = _gen(seed)
    need = [-(-(int(h) + int(n)) // block_size) for h, n in zip(hist_lens, q_lens)]
    nb = sum(need) + spare_blocks
    kf = torch.randn((nb, Hkv, block_size, D), generator=g, dtype=torch.float32)
    vf = torch.randn((nb, Hkv, block_size, D), generator=g, dtype=torch.float32)
    kc, ks = quantize_e4m3fn(kf)
    vc, vs = quantize_e4m3fn(vf)
    perm = torch.randperm(nb, generator=g).to(torch.int32)
    tables = torch.full((len(need), max(need + [1])), -1, dtype=torch.int32)
    o = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[o:o + n]
        o += n
    starts = [0]
    for n in q_lens:
        starts.append(starts[-1] + int(n))
    q = randn_bf16((Hq, starts[-1], D), g)
    scale = (1.0 / D ** 0.5) if softmax_scale is None else float(softmax_scale)
    return PagedPrefillCase(q, kc, vc, ks, vs, tables.contiguous(), block_size,
                            torch.tensor(starts, dtype=torch.int32),
                            torch.tensor([int(h) for h in hist_lens], dtype=torch.int32), scale,
                            Hq // Hkv)


# The five workloads named by the pages' shapes.
def tiny_case() -> EncoderCase:
    return encoder_case(1, 4, 256, 64, seed=1001, softmax_scale=0.125)


def vitl_layer_case(layer: int) -> EncoderCase:
    return encoder_case(1, 16, 2048, 64, seed=2000 + layer, softmax_scale=0.125)


VITL_LAYERS = 24


def dinov3_case() -> EncoderCase:
    return encoder_case(8, 16, 201, 64, seed=1003, softmax_scale=0.125)


def gqa_decode_full_case() -> DecodeCase:
    return decode_case(8, 16, 8, 4096, 256, seed=1004, softmax_scale=1.0)


def paged_full_case() -> PagedCase:
    return paged_case(32, 2, 4096, 256, num_phys_blocks=256, block_size=512,
                      actual_history_len=100000, seed=1005, softmax_scale=1.0 / 16.0)


def rope_tables(S: int, D: int, base: float = 10000.0):
    """cos / sin tables [S, D/2] fp32 for 1-D positions 0 .. S-1 with angle s * base^(-2j/D)
    (pair j). The rotation kernels take any tables; models with 2-D or 3-D position grids
    (DINOv3, V-JEPA2) only fill them differently."""
    j = torch.arange(D // 2, dtype=torch.float64)
    w = base ** (-2.0 * j / D)
    theta = torch.arange(S, dtype=torch.float64)[:, None] * w[None, :]
    return torch.cos(theta).float(), torch.sin(theta).float()


@dataclass
class ProjectionCase:
    x: torch.Tensor            # [B, S, C] bf16 block input
    w_qkv: torch.Tensor        # [3 H D, C] bf16
    b_qkv: Optional[torch.Tensor]   # [3 H D] fp32
    w_o: torch.Tensor          # [C_out, H D] bf16
    b_o: Optional[torch.Tensor]     # [C_out] fp32
    H: int
    D: int


def projection_case(B, S, C, H, D, seed, C_out=None, bias=True) -> ProjectionCase:
    """Random-init weights of a ViT attention block (no trained weights exist here): entries
    N(0, 1/fan_in) in bf16 like a freshly initialised Linear, biases N(0, 0.02^2) fp32, and a
    block input x ~ N(0, 1) in bf16 (a LayerNorm output has unit variance per channel)."""
    g = _gen(seed)
    C_out = C if C_out is None else C_out
    x = randn_bf16((B, S, C), g)
    w_qkv = (torch.randn((3 * H * D, C), generator=g) / C ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn((C_out, H * D), generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    b_qkv = torch.randn(3 * H * D, generator=g) * 0.02 if bias else None
    b_o = torch.randn(C_out, generator=g) * 0.02 if bias else None
    return ProjectionCase(x, w_qkv, b_qkv, w_o, b_o, H, D)
