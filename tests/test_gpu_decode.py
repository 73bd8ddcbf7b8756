"""GPU parity of attn_gqa_decode against the fp64 oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import assert_bf16_parity, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(case: syn.DecodeCase, use_mask=True):
    q, k, v = (t.to(DEV) for t in (case.q, case.k, case.v))
    m = case.attn_mask.to(DEV) if (use_mask and case.attn_mask is not None) else None
    out = B.attn_gqa_decode(q, k, v, m, case.softmax_scale, case.num_kv_groups)
    assert B.attn_check() == 0
    return out


def _oracle(case: syn.DecodeCase, use_mask=True):
    m = case.attn_mask.double().numpy() if (use_mask and case.attn_mask is not None) else None
    return oracle.gqa_decode_attention(to_f64(case.q), to_f64(case.k), to_f64(case.v), m,
                                       case.softmax_scale, case.num_kv_groups)


def test_full_config_b8_16q_8kv_d256_ctx4096():
    case = syn.gqa_decode_full_case()
    assert_bf16_parity(_run(case), _oracle(case), 2, "decode full")


@pytest.mark.parametrize("D", [128, 256, 512])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_head_dims_and_groups(D, G):
    Hkv = 2
    case = syn.decode_case(3, Hkv * G, Hkv, 700, D, seed=10 * D + G, softmax_scale=D ** -0.5,
                           min_len=1, max_len=700)
    if D == 512 and G == 8:   # outside the supported set: rejected before any launch
        with pytest.raises(B.AttnError) as exc:
            _run(case)
        assert exc.value.status == -3
        return
    assert_bf16_parity(_run(case), _oracle(case), 2, f"D={D} G={G}")


@pytest.mark.parametrize("S_ctx", [1, 7, 8, 9, 31, 32, 33, 255, 256, 257, 511, 512, 513, 1000])
def test_ragged_context_without_mask(S_ctx):
    case = syn.decode_case(2, 4, 2, S_ctx, 256, seed=S_ctx, lengths=[S_ctx, S_ctx])
    assert_bf16_parity(_run(case, use_mask=False), _oracle(case, use_mask=False), 2,
                       f"S_ctx={S_ctx}")


def test_random_neg_inf_pattern_and_finite_mask_values():
    case = syn.decode_case(2, 4, 2, 1500, 256, seed=5)
    g = torch.Generator().manual_seed(1)
    m = torch.randn(2, 1, 1, 1500, generator=g)
    m[torch.rand(2, 1, 1, 1500, generator=g) < 0.7] = float("-inf")
    m[0, ..., 256:512] = float("-inf")          # one whole split removed
    case.attn_mask = m
    assert_bf16_parity(_run(case), _oracle(case), 2, "random mask")


def test_single_unmasked_key_is_bit_exact():
    case = syn.decode_case(2, 4, 2, 900, 256, seed=6)
    case.attn_mask.fill_(float("-inf"))
    case.attn_mask[0, ..., 0] = 0.0
    case.attn_mask[1, ..., 777] = 2.5
    out = _run(case).cpu()
    for h in range(4):
        assert torch.equal(out[0, h, 0], case.v[0, h // 2, 0])
        assert torch.equal(out[1, h, 0], case.v[1, h // 2, 777])


def test_masked_tail_equals_truncated_problem_bitwise():
    L = 1337
    full = syn.decode_case(2, 4, 2, 4096, 256, seed=7, lengths=[L, L])
    trunc = syn.DecodeCase(full.q, full.k[:, :, :L].contiguous(), full.v[:, :, :L].contiguous(),
                           None, full.lengths, full.softmax_scale, full.num_kv_groups)
    a = _run(full).cpu()
    b = _run(trunc, use_mask=False).cpu()
    assert torch.equal(a, b)


@pytest.mark.parametrize("G", [2, 4, 8])
def test_gqa_equals_repeated_kv_heads(G):
    # query head h reads kv head h // G. The repeated-KV problem (G = 1) runs the CUDA-core
    # stream step; G >= 4 runs the tensor-core one, so the two agree to rounding, not bitwise
    # (G = 2 runs the same path on both sides and must be bit-exact).
    case = syn.decode_case(2, 2 * G, 2, 600, 256, seed=8)
    rep = syn.DecodeCase(case.q, case.k.repeat_interleave(G, dim=1),
                         case.v.repeat_interleave(G, dim=1), case.attn_mask, case.lengths,
                         case.softmax_scale, 1)
    a, b = _run(case).cpu(), _run(rep).cpu()
    if G == 2:
        assert torch.equal(a, b)
    else:
        assert rel_l2(a.double().numpy(), b.double().numpy()) <= 2e-3
    assert_bf16_parity(a, _oracle(case), 2, f"G={G}")


def test_fully_masked_row_is_zero():
    case = syn.decode_case(1, 2, 1, 300, 256, seed=9)
    case.attn_mask.fill_(float("-inf"))
    out = _run(case).cpu()
    assert torch.count_nonzero(out) == 0


@pytest.mark.parametrize("W", [64, 500, 1024])
def test_sliding_window_mask(W):
    """Sliding-window layers (the decode page's windowed-KV follow-on) as an additive
    mask: only the last W positions before each length are kept; the kernel reads only
    the 8-key groups that hold them."""
    case = syn.decode_case(4, 8, 4, 4096, 256, seed=W, softmax_scale=256 ** -0.5)
    for b in range(4):
        L = int(case.lengths[b])
        case.attn_mask[b, ..., :max(0, L - W)] = float("-inf")
    assert_bf16_parity(_run(case), _oracle(case), 2, f"window {W}")


def test_head_dim_512_gemma_global_layer_shape():
    """Gemma global layers (decode page: head_dim 512), 2 Q heads per KV head."""
    case = syn.decode_case(2, 16, 8, 2048, 512, seed=512, softmax_scale=1.0, min_len=1)
    assert_bf16_parity(_run(case), _oracle(case), 2, "D=512")


def test_one_workspace_reused_across_calls_with_different_split_counts():
    """One workspace serves calls of any size in turn: every call rebuilds the live
    lists and partials it reads, whatever the previous call left there."""
    need = max(B.attn_gqa_decode_workspace_size(2, 8, 4, S, 256) for S in (4096, 700, 1, 2600))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for S in (4096, 700, 1, 2600, 4096):
        case = syn.decode_case(2, 8, 4, S, 256, seed=S, softmax_scale=1 / 16, min_len=1, max_len=S)
        q, k, v, m = (t.to(DEV) for t in (case.q, case.k, case.v, case.attn_mask))
        out = B.attn_gqa_decode(q, k, v, m, case.softmax_scale, case.num_kv_groups, workspace=ws)
        assert B.attn_check() == 0
        assert_bf16_parity(out, _oracle(case), 2, f"reuse S_ctx={S}")


def test_tiny_contexts_many_pairs_per_warp():
    """Short, ragged contexts: each warp's slice of the live sub-tile sequence crosses
    many (batch, kv head) pairs, and with S_ctx = 16 there are fewer sub-tiles than
    warps (most warps idle)."""
    for B_, S, seed in ((64, 64, 71), (2, 16, 72)):
        case = syn.decode_case(B_, 16, 8, S, 256, seed=seed, softmax_scale=1 / 16, min_len=1)
        assert_bf16_parity(_run(case), _oracle(case), 2, f"tiny contexts B={B_} S={S}")


def test_fully_masked_batch_entries_between_live_ones():
    """Batch entries without a live key produce zero rows and shift the numbering of
    the following entries' partials; their neighbours must be unaffected."""
    case = syn.decode_case(7, 8, 4, 1200, 128, seed=73, softmax_scale=128 ** -0.5, min_len=1)
    for b in (0, 3, 4, 6):
        case.attn_mask[b].fill_(float("-inf"))
    out = _run(case)
    ref = _oracle(case)
    assert_bf16_parity(out, ref, 2, "masked entries")
    assert torch.count_nonzero(out[[0, 3, 4, 6]].cpu()) == 0


def test_one_long_pair_spread_over_every_warp():
    """A single (batch, kv head) pair with 32768 keys: its live sub-tiles are split
    over all warps of the wave, so the combine merges well over a thousand partials."""
    case = syn.decode_case(1, 8, 1, 32768, 256, seed=74, softmax_scale=1 / 16,
                           lengths=[32768])
    assert_bf16_parity(_run(case), _oracle(case), 2, "one long pair")


def test_workspace_contents_on_entry_do_not_matter():
    case = syn.decode_case(3, 8, 2, 3000, 256, seed=75, softmax_scale=1 / 16, min_len=1)
    q, k, v, m = (t.to(DEV) for t in (case.q, case.k, case.v, case.attn_mask))
    need = B.attn_gqa_decode_workspace_size(3, 8, 2, 3000, 256)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bit patterns
    out = B.attn_gqa_decode(q, k, v, m, case.softmax_scale, case.num_kv_groups, workspace=ws)
    assert B.attn_check() == 0
    ref = B.attn_gqa_decode(q, k, v, m, case.softmax_scale, case.num_kv_groups)
    assert torch.equal(out.cpu(), ref.cpu())
    assert_bf16_parity(out, _oracle(case), 2, "garbage workspace")


def test_large_batch_long_context():
    """B = 32, 32 Q / 8 KV heads, 16k context, D = 128: many warps per (batch, kv head)."""
    case = syn.decode_case(32, 32, 8, 16384, 128, seed=76, softmax_scale=128 ** -0.5, min_len=1)
    assert_bf16_parity(_run(case), _oracle(case), 2, "large batch long context")


def test_nonfinite_k_v_rows_at_masked_keys_take_no_part():
    # masked slots inside partly live 8-key sub-tiles hold NaN / inf K and V rows (an
    # unwritten cache): the result must equal the oracle and, bitwise, the same call with
    # finite rows there (a -inf entry removes the key whatever its K and V hold)
    case = syn.decode_case(3, 8, 4, 600, 256, seed=61, min_len=200, max_len=590)
    g = torch.Generator().manual_seed(62)
    dead = torch.rand(3, 600, generator=g) < 0.3
    case.attn_mask[:, 0, 0][dead] = float("-inf")
    clean = _run(case)
    bad = dead[:, None, :].expand(3, 4, 600)
    case.k[bad] = float("nan")
    case.v[bad] = float("nan")
    case.v[:, :, 599] = float("inf")       # past every length: dead too
    got = _run(case)
    assert torch.equal(got.cpu(), clean.cpu())
    assert_bf16_parity(got, _oracle(case), 2, "nonfinite masked rows")


def test_float32_min_mask_fill_keeps_keys():
    # finfo(float32).min is a finite fill: a row masked with it everywhere is the mean of V,
    # next to 0-masked keys it carries no weight (as in the oracle; -inf alone removes a key)
    case = syn.decode_case(2, 4, 2, 300, 128, seed=63, lengths=[300, 300])
    fmin = torch.finfo(torch.float32).min
    case.attn_mask[0] = fmin
    case.attn_mask[1, ..., 100:] = fmin
    got = _run(case)
    assert_bf16_parity(got, _oracle(case), 2, "finfo.min fill")
    mean_v = case.v[0].double().mean(dim=1)           # [Hkv, D]
    ref = mean_v.repeat_interleave(2, dim=0)          # [Hq, D]
    assert torch.allclose(got[0, :, 0].cpu().double(), ref, atol=2e-3, rtol=0)
