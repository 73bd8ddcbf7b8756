"""GPU parity of attn_encoder_fwd against the fp64 oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import assert_bf16_parity, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(case: syn.EncoderCase):
    q, k, v = (t.to(DEV) for t in (case.q, case.k, case.v))
    kb = None if case.key_bias is None else case.key_bias.to(DEV)
    out = B.attn_encoder_fwd(q, k, v, case.softmax_scale, key_bias=kb)
    assert B.attn_check() == 0
    return out


def _oracle(case: syn.EncoderCase, rows=None):
    kb = None if case.key_bias is None else case.key_bias.double().numpy()
    return oracle.encoder_attention(to_f64(case.q), to_f64(case.k), to_f64(case.v),
                                    case.softmax_scale, key_bias=kb, rows=rows)


def test_tiny_mha_b1_h4_s256_d64():
    case = syn.tiny_case()
    assert_bf16_parity(_run(case), _oracle(case), 2, "tiny")


def test_dinov3_b8_h16_s201_d64_ragged_tail():
    case = syn.dinov3_case()
    assert_bf16_parity(_run(case), _oracle(case), 2, "dinov3")


@pytest.mark.parametrize("layer", [0, 23])
def test_vitl_b1_h16_s2048_d64(layer):
    case = syn.vitl_layer_case(layer)
    assert_bf16_parity(_run(case), _oracle(case), 2, f"vitl layer {layer}")


@pytest.mark.parametrize("S", [1, 7, 63, 64, 65, 127, 128, 129, 192, 193, 255, 256, 257, 300, 513])
@pytest.mark.parametrize("D", [64, 128])
def test_ragged_lengths(S, D):
    case = syn.encoder_case(2, 3, S, D, seed=300 + S + D, softmax_scale=D ** -0.5)
    assert_bf16_parity(_run(case), _oracle(case), 2, f"S={S} D={D}")


@pytest.mark.parametrize("D,with_bias", [(64, False), (64, True), (128, False)])
def test_running_max_grows_across_key_tiles(D, with_bias):
    """Scores that climb from one 128-key tile to the next (the keys of tile t carry 8 t times
    a direction the queries share), so the running max moves by more than 2^8 several times
    after the first tile and O is rescaled in later tiles. A skipped rescale or a wrong factor
    would leave the earlier tiles' share of O off by 2^8 or more."""
    g = torch.Generator().manual_seed(4242 + D)
    nb, nh, S = 2, 2, 700
    w = torch.randn(D, generator=g)
    w = w / w.norm()
    tile = (torch.arange(S) // 128).float()
    q = (torch.randn(nb, nh, S, D, generator=g) * 0.3 + 3.0 * w).to(torch.bfloat16)
    k = (torch.randn(nb, nh, S, D, generator=g) * 0.3 + (8.0 * tile)[:, None] * w).to(torch.bfloat16)
    v = torch.randn(nb, nh, S, D, generator=g).to(torch.bfloat16)
    kb = (torch.rand((nb, S), generator=g) * 0.5).float() if with_bias else None
    case = syn.EncoderCase(q, k, v, 0.125, kb)
    assert_bf16_parity(_run(case), _oracle(case), 2, f"growing max D={D} bias={with_bias}")


def test_head_dim_128_long():
    case = syn.encoder_case(1, 4, 1024, 128, seed=77, softmax_scale=128 ** -0.5)
    assert_bf16_parity(_run(case), _oracle(case), 2, "D=128 S=1024")


@pytest.mark.parametrize("D", [64, 128])
def test_right_padding_key_bias(D):
    case = syn.encoder_case(4, 2, 384, D, seed=91, softmax_scale=0.125,
                            pad_lengths=[384, 200, 129, 6])
    assert_bf16_parity(_run(case), _oracle(case), 2, "padding")


def test_random_finite_key_bias():
    case = syn.encoder_case(2, 2, 300, 64, seed=92)
    g = torch.Generator().manual_seed(5)
    case.key_bias = torch.randn(2, 300, generator=g) * 3.0
    assert_bf16_parity(_run(case), _oracle(case), 2, "finite bias")


def test_single_unmasked_key_is_bit_exact():
    case = syn.encoder_case(2, 2, 200, 64, seed=93, pad_lengths=[1, 1])
    case.key_bias[1, 0] = float("-inf")
    case.key_bias[1, 137] = 0.0
    out = _run(case).cpu()
    assert torch.equal(out[0], case.v[0, :, 0:1].expand(2, 200, 64))
    assert torch.equal(out[1], case.v[1, :, 137:138].expand(2, 200, 64))


def test_fully_masked_rows_are_zero():
    case = syn.encoder_case(1, 1, 140, 64, seed=94, pad_lengths=[0])
    out = _run(case).cpu()
    assert torch.count_nonzero(out) == 0


def test_zero_query_gives_mean_of_values():
    case = syn.encoder_case(1, 2, 333, 64, seed=95)
    case.q.zero_()
    ref = _oracle(case)
    assert np.allclose(ref[0, :, 0], to_f64(case.v)[0].mean(axis=1))
    assert_bf16_parity(_run(case), ref, 2, "q=0")


def test_batch_independence_bitwise():
    a = syn.encoder_case(2, 2, 201, 64, seed=96)
    b = syn.encoder_case(2, 2, 201, 64, seed=97)
    b.q[0], b.k[0], b.v[0] = a.q[0], a.k[0], a.v[0]
    oa, ob = _run(a).cpu(), _run(b).cpu()
    assert torch.equal(oa[0], ob[0])


def test_deterministic_repeat():
    case = syn.encoder_case(1, 4, 700, 64, seed=98)
    assert torch.equal(_run(case).cpu(), _run(case).cpu())


def test_long_sequence_8192_tokens_sampled_rows():
    """V-JEPA2's native 64-frame clip is 8192 tokens; the V-JEPA2 page's kernels could not
    run it (their cross-section combine). Online softmax has no section limit."""
    case = syn.encoder_case(1, 2, 8192, 64, seed=8192, softmax_scale=0.125)
    out = _run(case)
    rows = np.sort(np.random.default_rng(1).choice(8192, 256, replace=False))
    ref = _oracle(case, rows=rows)
    assert_bf16_parity(out[:, :, torch.from_numpy(rows).to(out.device)], ref, 2, "S=8192")


@pytest.mark.parametrize("L", [128, 512, 1024])
def test_gte_shapes_right_padded_batches(L):
    """gte encoders: head_dim 64, 16 heads, right-padded batches of ragged lengths
    (gte page "Accuracy": 6 tokens up to the padded length)."""
    lens = [L, 6, L // 2 + 3, L - 1]
    case = syn.encoder_case(4, 16, L, 64, seed=L, softmax_scale=0.125, pad_lengths=lens)
    out = _run(case)
    ref = _oracle(case)
    # rows of padded positions also attend to the valid keys; all rows are compared
    assert_bf16_parity(out, ref, 2, f"gte L={L}")


def test_all_zero_key_bias_equals_no_bias_bitwise():
    """Tiles whose key bias is all zero take the unbiased path of the same kernel: identical
    results (head dim 128: the two-query-tile kernel)."""
    c = syn.encoder_case(2, 4, 700, 128, seed=77, softmax_scale=128 ** -0.5)
    q, k, v = (t.to(DEV) for t in (c.q, c.k, c.v))
    zero = torch.zeros((2, 700), dtype=torch.float32, device=DEV)
    a = B.attn_encoder_fwd(q, k, v, c.softmax_scale)
    b = B.attn_encoder_fwd(q, k, v, c.softmax_scale, key_bias=zero)
    assert B.attn_check() == 0
    assert torch.equal(a, b)


def test_all_zero_key_bias_d64_equals_no_bias_bitwise():
    """Head dim 64: with an all-zero bias every tile of the one-query-tile kernel's key-bias
    build takes the unbiased path, so the result equals the call without a bias bit for bit
    (the columns past S weigh 0 there instead of 2^-125, against zero-filled V rows and a row
    sum of at least 1: no difference)."""
    c = syn.encoder_case(2, 4, 700, 64, seed=77, softmax_scale=0.125)
    q, k, v = (t.to(DEV) for t in (c.q, c.k, c.v))
    zero = torch.zeros((2, 700), dtype=torch.float32, device=DEV)
    a = B.attn_encoder_fwd(q, k, v, c.softmax_scale)
    b = B.attn_encoder_fwd(q, k, v, c.softmax_scale, key_bias=zero)
    assert B.attn_check() == 0
    assert_bf16_parity(a, _oracle(c), 2, "no bias")
    assert torch.equal(a, b)


def test_general_finite_key_bias():
    """Arbitrary additive per-key biases (not only 0 / -inf), some tiles all zero."""
    c = syn.encoder_case(2, 4, 600, 64, seed=78, softmax_scale=0.125)
    g = torch.Generator().manual_seed(79)
    kb = (torch.rand((2, 600), generator=g) * 6 - 3).float()
    kb[:, 128:256] = 0.0                           # one all-zero tile: the unbiased path
    kb[1, 500:] = float("-inf")
    q, k, v = (t.to(DEV) for t in (c.q, c.k, c.v))
    out = B.attn_encoder_fwd(q, k, v, c.softmax_scale, key_bias=kb.to(DEV))
    assert B.attn_check() == 0
    ref = oracle.encoder_attention(to_f64(c.q), to_f64(c.k), to_f64(c.v), c.softmax_scale,
                                   key_bias=kb.double().numpy())
    assert_bf16_parity(out, ref, 2, "general key bias")


@pytest.mark.parametrize("pattern", ["every_third", "right_padding"])
@pytest.mark.parametrize("D", [64, 128])
def test_dropped_keys_weigh_exactly_zero(D, pattern):
    """Keys dropped by a -inf bias inside tiles that keep other keys: their V rows hold the
    largest finite bf16 value, so any weight above 0 (2^-125 from the polynomial would already
    give ~7) shows in the output; the result must match the oracle, which drops them. Every
    third key dropped takes the biased path; a right-padded entry (zeros, then -inf) takes the
    unbiased one with the padding masked."""
    c = syn.encoder_case(2, 3, 600, D, seed=91, softmax_scale=D ** -0.5)
    kb = torch.zeros((2, 600), dtype=torch.float32)
    if pattern == "every_third":
        kb[:, 1::3] = float("-inf")
    kb[0, 300:] = float("-inf")          # a padded tail in both entries
    kb[1, 450:] = float("-inf")
    v = c.v.clone()
    big = torch.finfo(torch.bfloat16).max
    v[kb.isinf()[:, None, :, None].expand_as(v)] = big
    case = syn.EncoderCase(c.q, c.k, v, c.softmax_scale, kb)
    out = _run(case)
    assert torch.isfinite(out.float()).all()
    assert_bf16_parity(out, _oracle(case), 2, f"dropped keys D={D}")


def test_float32_min_key_bias_keeps_keys():
    # a finite -FLT_MAX bias keeps its keys: all of them give the mean of V, next to 0-biased
    # keys they carry no weight (-inf alone removes a key)
    case = syn.encoder_case(2, 2, 300, 64, seed=94)
    fmin = torch.finfo(torch.float32).min
    case.key_bias = torch.zeros(2, 300)
    case.key_bias[0] = fmin
    case.key_bias[1, 150:] = fmin
    got = _run(case)
    assert_bf16_parity(got, _oracle(case), 2, "finfo.min bias")
    ref = case.v[0].double().mean(dim=1, keepdim=True).expand(2, 300, 64)
    assert torch.allclose(got[0].cpu().double(), ref, atol=2e-3, rtol=0)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [300, 512])
def test_all_scores_far_below_zero(D, S):
    """Every score of every row near -1600 in natural units: the row max must be taken over
    exactly the row's scores (any stray larger value makes every weight underflow to 0)."""
    c = syn.encoder_case(1, 2, S, D, seed=95, softmax_scale=D ** -0.5)
    g = torch.Generator().manual_seed(96)
    k0 = torch.randn(D, generator=g)
    k0 = k0 / k0.norm() * D ** 0.25 * 8.0            # |k0|^2 * scale = 64
    kk = k0 + 0.05 * torch.randn((1, 2, S, D), generator=g)
    c.k = kk.to(torch.bfloat16)
    c.q = (-25.0 * k0).expand(1, 2, S, D).to(torch.bfloat16).contiguous()
    got = _run(c)
    ref = _oracle(c)
    s_max = (to_f64(c.q)[0, 0, 0] @ to_f64(c.k)[0, 0].T).max() * c.softmax_scale
    assert s_max < -1000.0, s_max                     # the case is what it claims
    assert_bf16_parity(got, ref, 2, "scores far below zero")



def test_key_bias_trailing_masked_tiles_are_skipped_bit_exactly():
    """Key tiles holding only -inf-biased keys (right padding) are never read: rows of a
    640-key problem whose keys 384.. carry -inf equal, bit for bit, the same rows of the
    384-key problem, even with NaN K and V in the skipped tiles."""
    B_, H, S, Sl, D = 2, 3, 640, 384, 64
    c = syn.encoder_case(B_, H, S, D, seed=97)
    kb = torch.zeros((B_, S), dtype=torch.float32)
    kb[:, Sl:] = float("-inf")
    k = c.k.clone()
    v = c.v.clone()
    k[:, :, Sl:] = float("nan")
    v[:, :, Sl:] = float("nan")
    q_d, k_d, v_d = (t.to(DEV) for t in (c.q, k, v))
    full = B.attn_encoder_fwd(q_d, k_d, v_d, c.softmax_scale, key_bias=kb.to(DEV))
    q_t, k_t, v_t = (t[:, :, :Sl].contiguous().to(DEV) for t in (c.q, k, v))
    kb_t = torch.zeros((B_, Sl), dtype=torch.float32, device=DEV)
    short = B.attn_encoder_fwd(q_t, k_t, v_t, c.softmax_scale, key_bias=kb_t)
    assert B.attn_check() == 0
    assert torch.isfinite(full.float()).all()
    assert torch.equal(full[:, :, :Sl], short)
    ref = oracle.encoder_attention(to_f64(c.q), to_f64(k), to_f64(v), c.softmax_scale,
                                   key_bias=kb.double().numpy())
    assert_bf16_parity(full, ref, 2, "trailing masked tiles")


@pytest.mark.parametrize("lengths", [[1, 640], [129, 300], [640, 640]])
def test_key_bias_ragged_lengths_per_batch_entry(lengths):
    """Per batch entry a different number of kept keys (1 key, one tile and a bit, all):
    each entry skips its own trailing tiles."""
    S = 640
    c = syn.encoder_case(len(lengths), 2, S, 64, seed=98 + lengths[0])
    kb = torch.zeros((len(lengths), S), dtype=torch.float32)
    for i, L in enumerate(lengths):
        kb[i, L:] = float("-inf")
    q, k, v = (t.to(DEV) for t in (c.q, c.k, c.v))
    got = B.attn_encoder_fwd(q, k, v, c.softmax_scale, key_bias=kb.to(DEV))
    assert B.attn_check() == 0
    ref = oracle.encoder_attention(to_f64(c.q), to_f64(c.k), to_f64(c.v), c.softmax_scale,
                                   key_bias=kb.double().numpy())
    assert_bf16_parity(got, ref, 2, f"lengths {lengths}")
