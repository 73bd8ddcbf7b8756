"""GPU parity of the projections around the attention core (attn_qkv_rope_proj, attn_out_proj)
against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import assert_bf16_parity, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
# fp32 output of an fp32-accumulated bf16 GEMM (K <= 1024): only accumulation rounding
FP32_OUT_REL_L2 = 1e-5


def _qkv(case, S, mode):
    x, w = case.x.to(DEV), case.w_qkv.to(DEV)
    b = None if case.b_qkv is None else case.b_qkv.to(DEV)
    cos = sin = None
    if mode is not None:
        cos, sin = (t.to(DEV) for t in syn.rope_tables(S, case.D))
    q, k, v = B.attn_qkv_rope_proj(x, w, b, case.H, case.D, cos, sin,
                                   interleaved=(mode == "interleaved"))
    assert B.attn_check() == 0
    return q, k, v


def _qkv_oracle(case, S, mode):
    cos = sin = None
    if mode is not None:
        cos, sin = (t.double().numpy() for t in syn.rope_tables(S, case.D))
    b = None if case.b_qkv is None else case.b_qkv.double().numpy()
    return oracle.qkv_rope_projection(to_f64(case.x), to_f64(case.w_qkv), b, case.H, case.D,
                                      cos, sin, mode)


@pytest.mark.parametrize("mode", ["interleaved", "half"])
def test_qkv_rope_vitl_layer(mode):
    # V-JEPA2 ViT-L: 2048 tokens, hidden 1024, 16 heads of 64
    case = syn.projection_case(1, 2048, 1024, 16, 64, seed=3100)
    got = _qkv(case, 2048, mode)
    ref = _qkv_oracle(case, 2048, mode)
    for g, r, n in zip(got, ref, "qkv"):
        assert_bf16_parity(g, r, 2, f"{n} ({mode})")


@pytest.mark.parametrize("B_,S,C,H,D,mode,bias", [
    (2, 200, 128, 2, 64, "half", False),          # ragged tail, H D = 128 (128-wide tiles)
    (1, 300, 256, 4, 128, "interleaved", True),   # D = 128
    (3, 129, 192, 6, 64, None, True),             # no rotation, 3 batch entries
    (1, 1, 64, 2, 64, "half", True),              # a single token
    (2, 600, 256, 4, 64, "half", True),           # 256-token tiles, ragged third tile
])
def test_qkv_shapes(B_, S, C, H, D, mode, bias):
    case = syn.projection_case(B_, S, C, H, D, seed=3200 + S + D, bias=bias)
    got = _qkv(case, S, mode)
    ref = _qkv_oracle(case, S, mode)
    for g, r, n in zip(got, ref, "qkv"):
        assert_bf16_parity(g, r, 2, f"{n} S={S} D={D} {mode}")


@pytest.mark.parametrize("S,H", [(150, 2), (300, 4)])   # 128- and 256-token tiles
def test_qkv_one_hot_weights_are_bit_exact(S, H):
    # W = three stacked identities (C = H D): q = k = v = x laid out as heads, bit for bit
    Bn, D = 2, 64
    C = H * D
    x = syn.randn_bf16((Bn, S, C), torch.Generator().manual_seed(3300))
    w = torch.cat([torch.eye(C)] * 3).to(torch.bfloat16)
    q, k, v = B.attn_qkv_rope_proj(x.to(DEV), w.to(DEV), None, H, D)
    assert B.attn_check() == 0
    want = x.view(Bn, S, H, D).permute(0, 2, 1, 3)
    for t in (q, k, v):
        assert torch.equal(t.cpu(), want)


def test_out_projection_vitl_layer():
    case = syn.projection_case(1, 2048, 1024, 16, 64, seed=3400)
    o = syn.randn_bf16((1, 16, 2048, 64), torch.Generator().manual_seed(3401))
    y = B.attn_out_proj(o.to(DEV), case.w_o.to(DEV), case.b_o.to(DEV))
    assert B.attn_check() == 0
    ref = oracle.out_projection(to_f64(o), to_f64(case.w_o), case.b_o.double().numpy())
    e = rel_l2(to_f64(y), ref)
    assert e <= FP32_OUT_REL_L2, e


@pytest.mark.parametrize("B_,S,H,D,C_out", [(2, 77, 3, 64, 128), (1, 260, 2, 128, 384)])
def test_out_projection_shapes(B_, S, H, D, C_out):
    g = torch.Generator().manual_seed(3500 + S)
    o = syn.randn_bf16((B_, H, S, D), g)
    w = (torch.randn((C_out, H * D), generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    y = B.attn_out_proj(o.to(DEV), w.to(DEV))
    assert B.attn_check() == 0
    ref = oracle.out_projection(to_f64(o), to_f64(w), None)
    assert rel_l2(to_f64(y), ref) <= FP32_OUT_REL_L2


def test_out_projection_identity_is_bit_exact():
    Bn, H, S, D = 2, 2, 130, 64
    o = syn.randn_bf16((Bn, H, S, D), torch.Generator().manual_seed(3600))
    w = torch.eye(H * D).to(torch.bfloat16)
    y = B.attn_out_proj(o.to(DEV), w.to(DEV))
    assert B.attn_check() == 0
    assert torch.equal(y.cpu(), o.permute(0, 2, 1, 3).reshape(Bn, S, H * D).float())


def test_attention_block_end_to_end():
    # projection -> RoPE -> attention -> out-projection on one DINOv3-sized image batch
    Bn, S, C, H, D = 2, 201, 1024, 16, 64
    case = syn.projection_case(Bn, S, C, H, D, seed=3700)
    q, k, v = _qkv(case, S, "half")
    o = B.attn_encoder_fwd(q, k, v, D ** -0.5)
    y = B.attn_out_proj(o, case.w_o.to(DEV), case.b_o.to(DEV))
    assert B.attn_check() == 0
    qr, kr, vr = _qkv_oracle(case, S, "half")
    orf = oracle.encoder_attention(qr, kr, vr, D ** -0.5)
    yr = oracle.out_projection(orf, to_f64(case.w_o), case.b_o.double().numpy())
    # three bf16 roundings (q/k/v, P, o) on the way: the bf16 path tolerance
    assert rel_l2(to_f64(y), yr) <= 5e-3
