"""Pins for the oracle's paged prefill (history + causal current tokens; no GPU).

* a library special case: with no history, one sequence is causal self-attention,
  checked against torch's scaled_dot_product_attention(is_causal=True) in float64
  on the dequantised K/V;
* a closed form: a single current token sees its history plus itself, i.e. the
  history-only attention over hist + 1 positions;
* causality: changing the cache at positions after a query's own leaves that
  query's output unchanged (and changing its own position does change it);
* batching: several sequences in one call equal one call per sequence;
* brute force: scalar loops, own gather, on a tiny case;
* a planted off-by-one in the causal limit is caught.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from oracle.e4m3 import e4m3fn_to_float64
from online_softmax_attention_flash_b200 import inputs as syn


def _f64(t):
    return t.double().numpy() if t.dtype == torch.bfloat16 else t.numpy()


def _run(c, rows=None):
    return oracle.paged_prefill_attention(_f64(c.q), c.k_cache.numpy(), c.v_cache.numpy(), c.k_scale,
                                          c.v_scale, c.block_tables.numpy(), c.block_size,
                                          c.q_start.numpy(), c.hist_lens.numpy(), c.softmax_scale,
                                          c.num_kv_groups, rows=rows)


def test_no_history_is_causal_self_attention_sdpa():
    c = syn.paged_prefill_case(4, 2, 32, 16, hist_lens=[0], q_lens=[37], seed=1)
    kl, vl = oracle.paged_logical_kv(c.k_cache.numpy(), c.v_cache.numpy(), c.k_scale, c.v_scale,
                                     c.block_tables[0].numpy(), 16, 37)
    q = torch.from_numpy(_f64(c.q))[None]
    k = torch.from_numpy(kl)[None].repeat_interleave(2, dim=1)
    v = torch.from_numpy(vl)[None].repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                           scale=c.softmax_scale)[0].numpy()
    np.testing.assert_allclose(_run(c), ref, rtol=0, atol=1e-12)


def test_single_current_token_sees_history_and_itself():
    c = syn.paged_prefill_case(4, 1, 16, 8, hist_lens=[29], q_lens=[1], seed=2)
    hist = oracle.paged_history_attention(_f64(c.q), c.k_cache.numpy(), c.v_cache.numpy(), c.k_scale,
                                          c.v_scale, c.block_tables[0].numpy(), 8, 30,
                                          c.softmax_scale, 4)
    np.testing.assert_array_equal(_run(c), hist)


def test_future_positions_do_not_matter():
    c = syn.paged_prefill_case(2, 1, 16, 8, hist_lens=[13], q_lens=[11], seed=3)
    base = _run(c)
    i = 5                                   # query 5 sits at logical position 13 + 5 = 18
    t = 13 + i + 1                          # first position it must not see
    blk, off = int(c.block_tables[0, t // 8]), t % 8
    c.k_cache[blk, :, off] = 0x48           # new (valid, finite) K and V codes for that token
    c.v_cache[blk, :, off] = 0xC4
    after = _run(c)
    np.testing.assert_array_equal(after[:, :i + 1], base[:, :i + 1])
    assert not np.array_equal(after[:, i + 1], base[:, i + 1])


def test_batched_sequences_equal_separate_calls():
    hl, ql = [0, 40, 9], [5, 17, 30]
    c = syn.paged_prefill_case(4, 2, 16, 8, hist_lens=hl, q_lens=ql, seed=4)
    whole = _run(c)
    for s in range(3):
        a, b = int(c.q_start[s]), int(c.q_start[s + 1])
        one = syn.PagedPrefillCase(c.q[:, a:b].contiguous(), c.k_cache, c.v_cache, c.k_scale, c.v_scale,
                                   c.block_tables[s:s + 1], 8, torch.tensor([0, b - a], dtype=torch.int32),
                                   c.hist_lens[s:s + 1], c.softmax_scale, 2)
        np.testing.assert_array_equal(whole[:, a:b], _run(one))


def test_brute_force_tiny():
    c = syn.paged_prefill_case(2, 1, 4, 4, hist_lens=[3, 0], q_lens=[4, 3], seed=5)
    out = _run(c)
    kd, vd = e4m3fn_to_float64(c.k_cache.numpy()), e4m3fn_to_float64(c.v_cache.numpy())
    q = _f64(c.q)
    for s in range(2):
        hist = int(c.hist_lens[s])
        for i in range(int(c.q_start[s + 1] - c.q_start[s])):
            row = int(c.q_start[s]) + i
            for h in range(2):
                w, vs = [], []
                for t in range(hist + i + 1):
                    blk, off = int(c.block_tables[s, t // 4]), t % 4
                    kk = [float(x) * c.k_scale for x in kd[blk, 0, off]]
                    vs.append([float(x) * c.v_scale for x in vd[blk, 0, off]])
                    w.append(math.exp(c.softmax_scale * math.fsum(float(q[h, row, d]) * kk[d] for d in range(4))))
                den = math.fsum(w)
                for d in range(4):
                    assert math.isclose(out[h, row, d], math.fsum(w[j] * vs[j][d] for j in range(len(w))) / den,
                                        rel_tol=1e-12, abs_tol=1e-12)


def test_planted_off_by_one_is_caught(monkeypatch):
    c = syn.paged_prefill_case(4, 1, 16, 8, hist_lens=[29], q_lens=[1], seed=2)
    good = _run(c)
    real = oatt.paged_logical_kv

    def short(kc, vc, ks, vs, table, bs, L):   # drops the current token's own key
        return real(kc, vc, ks, vs, table, bs, L - 1)
    monkeypatch.setattr(oatt, "paged_logical_kv", short)
    with pytest.raises(Exception):
        _run(c)                                     # shapes no longer line up
    monkeypatch.setattr(oatt, "paged_logical_kv", real)
    hist = oracle.paged_history_attention(_f64(c.q), c.k_cache.numpy(), c.v_cache.numpy(), c.k_scale,
                                          c.v_scale, c.block_tables[0].numpy(), 8, 29,
                                          c.softmax_scale, 4)
    assert not np.allclose(good, hist)               # "t < hist + i" would have given this
