"""GPU parity of attn_paged_prefill (history + causal current tokens, several sequences)
against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import FP8_REL_L2, FP8_ROW_REL_L2, assert_rows_close, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SPLIT_DESIGN_REL_L2 = 5e-3   # the hi/lo split keeps the FP8 path at bf16-level accuracy


def _dev(c):
    return (c.q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV), c.block_tables.to(DEV),
            c.q_start.to(DEV), c.hist_lens.to(DEV))


def _run(c, **kw):
    q, kc, vc, bt, qs, hl = _dev(c)
    out = B.attn_paged_prefill(q, kc, vc, bt, qs, hl, c.k_scale, c.v_scale, c.softmax_scale,
                               c.num_kv_groups, **kw)
    return out


def _oracle(c):
    return oracle.paged_prefill_attention(to_f64(c.q), c.k_cache.numpy(), c.v_cache.numpy(),
                                          c.k_scale, c.v_scale, c.block_tables.numpy(), c.block_size,
                                          c.q_start.numpy(), c.hist_lens.numpy(), c.softmax_scale,
                                          c.num_kv_groups)


@pytest.mark.parametrize("bs,hist,qlen", [
    (128, [1000], [300]),                       # one sequence, ragged tiles
    (512, [0, 700, 4096], [129, 1, 500]),       # no history, one token, long history
    (256, [37, 0, 255, 1024], [128, 257, 64, 3]),
])
def test_matches_oracle(bs, hist, qlen):
    c = syn.paged_prefill_case(8, 2, 256, bs, hist_lens=hist, q_lens=qlen, seed=sum(hist) + bs,
                               softmax_scale=1 / 16)
    out = _run(c)
    assert B.attn_check() == 0
    ref = _oracle(c)
    e = rel_l2(to_f64(out), ref)
    assert e <= SPLIT_DESIGN_REL_L2 <= FP8_REL_L2, e
    assert_rows_close(to_f64(out), ref, FP8_ROW_REL_L2, f"bs={bs}")


def test_sequences_are_independent_bitwise():
    hist, qlen = [300, 1200, 50], [200, 130, 400]
    c = syn.paged_prefill_case(4, 1, 256, 128, hist_lens=hist, q_lens=qlen, seed=21, softmax_scale=1 / 16)
    whole = _run(c).cpu()
    for s in range(3):
        a, b = int(c.q_start[s]), int(c.q_start[s + 1])
        one = syn.PagedPrefillCase(c.q[:, a:b].contiguous(), c.k_cache, c.v_cache, c.k_scale, c.v_scale,
                                   c.block_tables[s:s + 1].contiguous(), 128,
                                   torch.tensor([0, b - a], dtype=torch.int32), c.hist_lens[s:s + 1].clone(),
                                   c.softmax_scale, 4)
        assert torch.equal(_run(one).cpu(), whole[:, a:b])
    assert B.attn_check() == 0


def test_one_current_token_equals_history_of_one_more_bitwise():
    c = syn.paged_prefill_case(8, 2, 256, 512, hist_lens=[2047], q_lens=[1], seed=22, softmax_scale=1 / 16)
    pre = _run(c)
    q, kc, vc, bt, _, _ = _dev(c)
    n = int((c.block_tables[0] >= 0).sum())
    hist = B.attn_paged_history(q, kc, vc, bt[0, :n].contiguous(), 512, 2048, c.k_scale, c.v_scale,
                                c.softmax_scale, c.num_kv_groups)
    assert B.attn_check() == 0
    assert torch.equal(pre.cpu(), hist.cpu())


def test_bad_sequence_descriptor_is_reported_and_others_are_unaffected():
    c = syn.paged_prefill_case(4, 1, 256, 128, hist_lens=[100, 200], q_lens=[50, 60], seed=23,
                               softmax_scale=1 / 16)
    good = _run(c).cpu()
    assert B.attn_check() == 0
    bad = syn.PagedPrefillCase(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables, 128,
                               c.q_start, torch.tensor([100, 10 ** 6], dtype=torch.int32),
                               c.softmax_scale, 4)
    out = torch.zeros_like(c.q).to(DEV)
    q, kc, vc, bt, qs, hl = _dev(bad)
    B.attn_paged_prefill(q, kc, vc, bt, qs, hl, c.k_scale, c.v_scale, c.softmax_scale, 4, out=out)
    assert B.attn_check() == -9                                    # ATTN_ERR_SEQUENCE
    out = out.cpu()
    assert torch.equal(out[:, :50], good[:, :50])                 # sequence 0 still computed
    assert torch.count_nonzero(out[:, 50:]) == 0                   # sequence 1 left untouched


def test_many_sequences_with_empty_ones_and_block_size_384():
    g = np.random.default_rng(24)
    hist = g.integers(0, 900, size=40).tolist()
    qlen = g.integers(0, 200, size=40).tolist()
    qlen[3] = qlen[17] = 0                      # sequences with nothing to prefill
    c = syn.paged_prefill_case(4, 2, 256, 384, hist_lens=hist, q_lens=qlen, seed=25, softmax_scale=1 / 16)
    out = _run(c)
    assert B.attn_check() == 0
    e = rel_l2(to_f64(out), _oracle(c))
    assert e <= SPLIT_DESIGN_REL_L2, e


def test_sequence_that_fills_its_table_row_exactly():
    c = syn.paged_prefill_case(8, 2, 256, 512, hist_lens=[1536, 1000], q_lens=[512, 24], seed=26,
                               softmax_scale=1 / 16, spare_blocks=0)
    assert int((c.block_tables[0] >= 0).sum()) * 512 == 1536 + 512   # every entry used
    out = _run(c)
    assert B.attn_check() == 0
    assert rel_l2(to_f64(out), _oracle(c)) <= SPLIT_DESIGN_REL_L2


def test_pcp_head_shape_16_query_heads_per_kv_head():
    """The history page's head shape: 32 Q heads sharing 2 KV heads, blocks of 512."""
    c = syn.paged_prefill_case(32, 2, 256, 512, hist_lens=[2048, 700], q_lens=[300, 129], seed=27,
                               softmax_scale=1 / 16)
    out = _run(c)
    assert B.attn_check() == 0
    assert rel_l2(to_f64(out), _oracle(c)) <= SPLIT_DESIGN_REL_L2
