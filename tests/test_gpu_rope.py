"""GPU parity of attn_rope_qk (rotary embedding of Q and K) against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import assert_bf16_parity, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bf16_ulps(got: torch.Tensor, ref64: np.ndarray) -> np.ndarray:
    """|got - ref| in units of the bf16 spacing at ref."""
    r = np.abs(ref64)
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -126)))
    spacing = 2.0 ** (e - 7)
    return np.abs(to_f64(got) - ref64) / spacing


def _case(B_, H, S, D, seed, random_angles=True):
    g = torch.Generator().manual_seed(seed)
    q = syn.randn_bf16((B_, H, S, D), g)
    k = syn.randn_bf16((B_, H, S, D), g)
    if random_angles:
        th = (torch.rand((S, D // 2), generator=g, dtype=torch.float64) * 2 - 1) * 40.0
        c, s = torch.cos(th).float(), torch.sin(th).float()
    else:
        c, s = syn.rope_tables(S, D)
    return q, k, c, s


@pytest.mark.parametrize("mode", ["half", "interleaved"])
@pytest.mark.parametrize("B_,H,S,D", [(1, 2, 7, 16), (2, 3, 129, 64), (1, 4, 300, 128),
                                      (1, 1, 33, 256), (1, 2, 5, 512)])
def test_rotation_matches_oracle_to_one_bf16_ulp(mode, B_, H, S, D):
    q, k, c, s = _case(B_, H, S, D, seed=S * D + B_)
    qo, ko = B.attn_rope_qk(*(t.to(DEV) for t in (q, k, c, s)), interleaved=(mode == "interleaved"))
    assert B.attn_check() == 0
    for got, x in ((qo, q), (ko, k)):
        ref = oracle.rope_apply(to_f64(x), c.double().numpy(), s.double().numpy(), mode)
        ulps = _bf16_ulps(got.cpu(), ref)
        assert ulps.max() <= 1.0, ulps.max()
        assert (ulps <= 0.5).mean() > 0.99   # correctly rounded almost everywhere


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_in_place_equals_out_of_place_and_identity_table_is_exact(mode):
    q, k, c, s = (t.to(DEV) for t in _case(2, 4, 200, 64, seed=9))
    il = mode == "interleaved"
    qo, ko = B.attn_rope_qk(q, k, c, s, interleaved=il)
    q2, k2 = q.clone(), k.clone()
    B.attn_rope_qk(q2, k2, c, s, interleaved=il, q_out=q2, k_out=k2)
    assert torch.equal(q2, qo) and torch.equal(k2, ko)
    qi, ki = B.attn_rope_qk(q, k, torch.ones_like(c), torch.zeros_like(s), interleaved=il)
    assert torch.equal(qi, q) and torch.equal(ki, k)
    assert B.attn_check() == 0


def test_pairings_agree_up_to_a_lane_permutation_bitwise():
    D = 64
    q, k, c, s = (t.to(DEV) for t in _case(1, 3, 77, D, seed=10))
    perm = torch.empty(D, dtype=torch.long)
    perm[0::2], perm[1::2] = torch.arange(D // 2), torch.arange(D // 2) + D // 2
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(D)
    qh, kh = q[..., inv].contiguous(), k[..., inv].contiguous()   # interleaved -> half layout
    yh, zh = B.attn_rope_qk(qh, kh, c, s, interleaved=False)
    yi, zi = B.attn_rope_qk(q, k, c, s, interleaved=True)
    assert torch.equal(yh[..., perm], yi) and torch.equal(zh[..., perm], zi)


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_rope_then_encoder_matches_oracle_attention_of_rotated_inputs(mode):
    """The encoder prologue as a user runs it: rotate Q and K, then attention."""
    Bn, H, S, D = 1, 4, 300, 64
    q, k, c, s = _case(Bn, H, S, D, seed=11, random_angles=False)
    v = syn.randn_bf16((Bn, H, S, D), torch.Generator().manual_seed(12))
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    qr, kr = B.attn_rope_qk(qd, kd, c.to(DEV), s.to(DEV), interleaved=(mode == "interleaved"))
    out = B.attn_encoder_fwd(qr, kr, vd, 0.125)
    assert B.attn_check() == 0
    c64, s64 = c.double().numpy(), s.double().numpy()
    ref = oracle.encoder_attention(oracle.rope_apply(to_f64(q), c64, s64, mode),
                                   oracle.rope_apply(to_f64(k), c64, s64, mode), to_f64(v), 0.125)
    assert_bf16_parity(out, ref, 2, f"rope {mode} + encoder")
