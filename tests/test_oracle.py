"""Pins for the CPU fp64 oracle, against things other than the oracle itself.

* brute force: pure-Python scalar loops on tiny shapes, written from the
  textbook definition softmax(x)_j = e^{x_j} / sum_k e^{x_k} without the max
  shift the oracle uses, summed with math.fsum;
* a library special case: torch's scaled_dot_product_attention in float64 on
  the CPU (independent code) with GQA and an additive mask;
* closed forms and invariants: all-equal scores give the mean of V, a single
  unmasked key gives its V row, a fully masked tail equals the truncated
  problem, GQA equals repeated KV heads, additive mask shift invariance, key
  permutation invariance, split-KV log-sum-exp combine equals the unsplit row;
* the paged gather: an identity block table over a contiguous pool equals the
  dense problem, a one-hot probe lands on block_table[t // bs] at offset t % bs,
  relabelling the physical pool changes nothing;
* the FP8 decoder against the format's fixed points and torch's e4m3fn cast;
* the FLOP formula against the MFU figures the history page prints.

No GPU is used here.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from oracle.e4m3 import E4M3FN_TABLE, e4m3fn_to_float64
from online_softmax_attention_flash_b200 import inputs as syn


# ---------------------------------------------------------------- brute force
def brute_attention(q, k, v, scale, groups=1, mask=None):
    """Scalar loops straight from the definition, no max subtraction (tiny, well-scaled inputs)."""
    B, Hq, Sq, D = q.shape
    L = k.shape[2]
    out = np.zeros((B, Hq, Sq, D))
    for b in range(B):
        for h in range(Hq):
            g = h // groups
            for i in range(Sq):
                w = []
                for j in range(L):
                    mij = 0.0 if mask is None else float(mask[b, h if mask.shape[1] > 1 else 0,
                                                             i if mask.shape[2] > 1 else 0, j])
                    if mij == -math.inf:
                        w.append(0.0)
                        continue
                    dot = math.fsum(float(q[b, h, i, d]) * float(k[b, g, j, d]) for d in range(D))
                    w.append(math.exp(scale * dot + mij))
                den = math.fsum(w)
                for d in range(D):
                    out[b, h, i, d] = (math.fsum(w[j] * float(v[b, g, j, d]) for j in range(L)) / den
                                       if den > 0 else 0.0)
    return out


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,L,D", [(1, 1, 1, 3, 5, 4), (2, 4, 2, 2, 7, 8),
                                             (1, 4, 1, 1, 9, 8), (2, 2, 2, 4, 6, 3)])
def test_brute_force_dense_and_gqa(B, Hq, Hkv, Sq, L, D):
    r = _rng(B * 100 + Hq * 10 + L)
    q = r.standard_normal((B, Hq, Sq, D))
    k = r.standard_normal((B, Hkv, L, D))
    v = r.standard_normal((B, Hkv, L, D))
    scale = 0.37
    got = oracle.softmax_attention(q, k, v, scale, Hq // Hkv)
    ref = brute_attention(q, k, v, scale, Hq // Hkv)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_brute_force_with_mask():
    r = _rng(7)
    B, Hq, Hkv, L, D = 2, 4, 2, 9, 8
    q = r.standard_normal((B, Hq, 1, D))
    k = r.standard_normal((B, Hkv, L, D))
    v = r.standard_normal((B, Hkv, L, D))
    mask = r.standard_normal((B, 1, 1, L)) * 0.5
    mask[0, 0, 0, [1, 4, 8]] = -np.inf
    mask[1, 0, 0, 5:] = -np.inf
    got = oracle.gqa_decode_attention(q, k, v, mask, 1.0, 2)
    ref = brute_attention(q, k, v, 1.0, 2, mask)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_brute_force_paged():
    r = _rng(11)
    NB, Hkv, BS, D, Hq, Sq = 4, 2, 4, 8, 4, 3
    kc = r.integers(0, 256, (NB, Hkv, BS, D), dtype=np.uint8)
    vc = r.integers(0, 256, (NB, Hkv, BS, D), dtype=np.uint8)
    for c in (kc, vc):  # no NaN codes in a cache
        c[(c & 0x7F) == 0x7F] = 0x3C
    table = np.array([2, 0, 3, 1], dtype=np.int32)
    length = 11  # block 2 of the table is partial (offsets 0..2 live)
    ks, vs = 0.01, 0.02
    q = r.standard_normal((Hq, Sq, D))
    got = oracle.paged_history_attention(q, kc, vc, ks, vs, table, BS, length, 0.25, 2)
    # brute force: walk logical positions through the table one by one
    out = np.zeros((Hq, Sq, D))
    for h in range(Hq):
        g = h // 2
        for i in range(Sq):
            w, rows = [], []
            for t in range(length):
                blk, off = int(table[t // BS]), t % BS
                kk = [E4M3FN_TABLE[kc[blk, g, off, d]] * ks for d in range(D)]
                vv = [E4M3FN_TABLE[vc[blk, g, off, d]] * vs for d in range(D)]
                w.append(math.exp(0.25 * math.fsum(q[h, i, d] * kk[d] for d in range(D))))
                rows.append(vv)
            den = math.fsum(w)
            for d in range(D):
                out[h, i, d] = math.fsum(w[t] * rows[t][d] for t in range(length)) / den
    assert np.max(np.abs(got - out)) <= 1e-12


# ---------------------------------------------------------- library special case
@pytest.mark.parametrize("groups", [1, 2, 8])
def test_matches_torch_sdpa_float64(groups):
    g = torch.Generator().manual_seed(groups)
    B, Hkv, Sq, L, D = 2, 2, 33, 70, 16
    Hq = Hkv * groups
    q = torch.randn(B, Hq, Sq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, L, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, L, D, generator=g, dtype=torch.float64)
    mask = torch.zeros(B, 1, 1, L, dtype=torch.float64)
    mask[0, ..., 50:] = -math.inf
    mask[1, ..., ::3] = -math.inf
    mask += torch.rand(B, 1, 1, L, generator=g, dtype=torch.float64) * (mask == 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=mask, scale=0.3, enable_gqa=(groups > 1)).numpy()
    got = oracle.softmax_attention(q.numpy(), k.numpy(), v.numpy(), 0.3, groups, mask.numpy())
    assert np.max(np.abs(got - ref)) <= 1e-12


# ---------------------------------------------------------------- invariants
def test_zero_query_gives_mean_of_valid_values():
    r = _rng(3)
    k = r.standard_normal((1, 2, 40, 16))
    v = r.standard_normal((1, 2, 40, 16))
    q = np.zeros((1, 2, 1, 16))
    mask = np.zeros((1, 1, 1, 40))
    mask[..., 29:] = -np.inf
    got = oracle.gqa_decode_attention(q, k, v, mask, 1.0, 1)
    assert np.allclose(got[0, :, 0], v[0, :, :29].mean(axis=1), rtol=0, atol=1e-14)


def test_single_unmasked_key_returns_its_value_row():
    r = _rng(4)
    k = r.standard_normal((2, 1, 64, 8))
    v = r.standard_normal((2, 1, 64, 8))
    q = r.standard_normal((2, 4, 1, 8)) * 10
    mask = np.full((2, 1, 1, 64), -np.inf)
    mask[0, ..., 17] = 0.0
    mask[1, ..., 0] = 3.0
    got = oracle.gqa_decode_attention(q, k, v, mask, 1.0, 4)
    assert np.array_equal(got[0, :, 0], np.broadcast_to(v[0, 0, 17], (4, 8)))
    assert np.array_equal(got[1, :, 0], np.broadcast_to(v[1, 0, 0], (4, 8)))


def test_masked_tail_equals_truncated_problem():
    r = _rng(5)
    q = r.standard_normal((1, 2, 5, 8))
    k = r.standard_normal((1, 2, 50, 8))
    v = r.standard_normal((1, 2, 50, 8))
    kb = np.zeros((1, 50))
    kb[:, 31:] = -np.inf
    full = oracle.encoder_attention(q, k, v, 0.5, key_bias=kb)
    trunc = oracle.encoder_attention(q, k[:, :, :31], v[:, :, :31], 0.5)
    assert np.max(np.abs(full - trunc)) <= 1e-15


def test_gqa_equals_repeated_kv_heads():
    r = _rng(6)
    q = r.standard_normal((2, 8, 3, 8))
    k = r.standard_normal((2, 2, 20, 8))
    v = r.standard_normal((2, 2, 20, 8))
    got = oracle.softmax_attention(q, k, v, 0.7, 4)
    rep = oracle.softmax_attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 0.7, 1)
    assert np.array_equal(got, rep)
    # the wrong mapping (h % Hkv) must give a different answer on these inputs
    alt = oracle.softmax_attention(q, np.tile(k, (1, 4, 1, 1)), np.tile(v, (1, 4, 1, 1)), 0.7, 1)
    assert np.max(np.abs(got - alt)) > 1e-3


def test_mask_shift_and_key_permutation_invariance():
    r = _rng(8)
    q = r.standard_normal((1, 1, 4, 8))
    k = r.standard_normal((1, 1, 30, 8))
    v = r.standard_normal((1, 1, 30, 8))
    mask = r.standard_normal((1, 1, 1, 30))
    base = oracle.softmax_attention(q, k, v, 0.4, 1, mask)
    shifted = oracle.softmax_attention(q, k, v, 0.4, 1, mask + 123.0)
    assert np.max(np.abs(base - shifted)) <= 1e-13
    perm = r.permutation(30)
    permuted = oracle.softmax_attention(q, k[:, :, perm], v[:, :, perm], 0.4, 1, mask[..., perm])
    assert np.max(np.abs(base - permuted)) <= 1e-14


def test_scale_and_large_scores_are_stable():
    # a uniform score offset of 1e3 must not overflow (the max shift handles it)
    r = _rng(9)
    q = np.ones((1, 1, 1, 4))
    k = r.standard_normal((1, 1, 10, 4)) + 250.0
    v = r.standard_normal((1, 1, 10, 4))
    out = oracle.softmax_attention(q, k, v, 1.0)
    assert np.all(np.isfinite(out))
    # scale 0 gives the plain mean
    out0 = oracle.softmax_attention(q, k, v, 0.0)
    assert np.allclose(out0[0, 0, 0], v[0, 0].mean(axis=0), atol=1e-15)


def test_fully_masked_row_is_zero_and_lse_neg_inf():
    q = np.ones((1, 1, 2, 4))
    k = np.ones((1, 1, 3, 4))
    v = np.ones((1, 1, 3, 4))
    mask = np.full((1, 1, 2, 3), -np.inf)
    mask[0, 0, 1, 2] = 0.0
    out, lse = oracle.softmax_attention(q, k, v, 1.0, 1, mask, return_lse=True)
    assert np.array_equal(out[0, 0, 0], np.zeros(4)) and lse[0, 0, 0] == -np.inf
    assert np.array_equal(out[0, 0, 1], np.ones(4)) and abs(lse[0, 0, 1] - 4.0) < 1e-15


def test_removed_keys_ignore_nonfinite_k_and_v_rows():
    # A -inf mask entry removes the key outright: NaN / inf in its K or V row must not reach
    # the result (truncated problem as the pin), while a NaN V row at a kept key does.
    r = _rng(12)
    q = r.standard_normal((2, 4, 1, 8))
    k = r.standard_normal((2, 2, 20, 8))
    v = r.standard_normal((2, 2, 20, 8))
    mask = np.zeros((2, 1, 1, 20))
    mask[0, ..., [3, 7]] = -np.inf
    mask[1, ..., 11:] = -np.inf
    keep0 = [j for j in range(20) if j not in (3, 7)]
    kk, vv = k.copy(), v.copy()
    kk[0, :, 3] = np.nan
    vv[0, :, 3] = np.nan
    vv[0, :, 7] = np.inf
    kk[1, :, 15] = np.inf
    vv[1, :, 12:] = np.nan
    got = oracle.gqa_decode_attention(q, kk, vv, mask, 1.0, 2)
    ref0 = brute_attention(q[:1], k[:1, :, keep0], v[:1, :, keep0], 1.0, 2)
    ref1 = brute_attention(q[1:], k[1:, :, :11], v[1:, :, :11], 1.0, 2)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got[:1] - ref0)) <= 1e-12
    assert np.max(np.abs(got[1:] - ref1)) <= 1e-12
    vv[0, :, 5] = np.nan   # kept key
    assert np.all(np.isnan(oracle.gqa_decode_attention(q, kk, vv, mask, 1.0, 2)[0]))


def test_float32_min_fill_keeps_its_keys():
    # -FLT_MAX (torch.finfo(float32).min, a common mask fill) is finite: a row masked with it
    # everywhere keeps every key with equal scores (q.k is absorbed), i.e. the mean of V;
    # next to 0-masked keys those keys get weight e^(-3.4e38) = 0.
    fmin = float(np.finfo(np.float32).min)
    r = _rng(13)
    q = r.standard_normal((1, 2, 1, 8))
    k = r.standard_normal((1, 1, 12, 8))
    v = r.standard_normal((1, 1, 12, 8))
    mask = np.full((1, 1, 1, 12), fmin)
    got = oracle.gqa_decode_attention(q, k, v, mask, 1.0, 2)
    assert np.allclose(got[0, :, 0], np.broadcast_to(v[0, 0].mean(axis=0), (2, 8)), atol=1e-15)
    mask[..., :5] = 0.0
    got = oracle.gqa_decode_attention(q, k, v, mask, 1.0, 2)
    ref = brute_attention(q, k[:, :, :5], v[:, :, :5], 1.0, 2)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_lse_combine_equals_unsplit_row():
    r = _rng(10)
    D, L = 16, 37
    q = r.standard_normal(D)
    k = r.standard_normal((L, D))
    v = r.standard_normal((L, D))
    keep = np.ones(L, bool)
    keep[12:20] = False          # one split below is entirely masked
    s = np.where(keep, k @ q * 0.5, -np.inf)
    parts_o, parts_m, parts_l = [], [], []
    for lo, hi in [(0, 12), (12, 20), (20, 31), (31, 37)]:
        ss = s[lo:hi]
        m = ss.max()
        p = np.exp(ss - m) if np.isfinite(m) else np.zeros_like(ss)
        parts_o.append(p @ v[lo:hi])
        parts_m.append(m)
        parts_l.append(p.sum())
    got = oracle.lse_combine(np.array(parts_o), np.array(parts_m), np.array(parts_l))
    mask = np.where(keep, 0.0, -np.inf)[None, None, None, :]
    ref = oracle.softmax_attention(q[None, None, None], k[None, None], v[None, None], 0.5, 1, mask)
    assert np.max(np.abs(got - ref[0, 0, 0])) <= 1e-14


# ---------------------------------------------------------------- paged gather
def _small_paged(seed=21, NB=6, BS=8, Hkv=2, D=16, Hq=4, Sq=5):
    return syn.paged_case(Hq, Hkv, Sq, D, NB, BS, actual_history_len=NB * BS - 3, seed=seed,
                          softmax_scale=0.25)


def test_paged_identity_table_equals_dense():
    c = _small_paged()
    NB, Hkv, BS, D = c.k_cache.shape
    ident = np.arange(NB, dtype=np.int32)
    got = oracle.paged_history_attention(c.q.double().numpy(), c.k_cache.numpy(),
                                         c.v_cache.numpy(), c.k_scale, c.v_scale, ident, BS,
                                         c.actual_history_len, c.softmax_scale, c.num_kv_groups)
    # dense layout by plain reshaping of the pool (identity table), decoded by torch's cast
    kd = (c.k_cache.view(torch.float8_e4m3fn).double() * c.k_scale).numpy()
    vd = (c.v_cache.view(torch.float8_e4m3fn).double() * c.v_scale).numpy()
    kd = kd.transpose(1, 0, 2, 3).reshape(Hkv, NB * BS, D)[:, :c.actual_history_len]
    vd = vd.transpose(1, 0, 2, 3).reshape(Hkv, NB * BS, D)[:, :c.actual_history_len]
    ref = torch.nn.functional.scaled_dot_product_attention(
        c.q.double()[None], torch.from_numpy(kd)[None], torch.from_numpy(vd)[None],
        scale=c.softmax_scale, enable_gqa=True)[0].numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_paged_one_hot_probe_hits_table_entry():
    c = _small_paged(seed=22)
    NB, Hkv, BS, D = c.k_cache.shape
    table = c.block_table.numpy()
    q = np.zeros((c.q.shape[0], 1, D))
    q[:, 0, 0] = 1.0
    kc = c.k_cache.numpy().copy()
    kc[..., 0] = 0  # code 0 = +0.0 everywhere in the probe lane
    for t in [0, BS - 1, BS, 2 * BS + 3, c.actual_history_len - 1]:
        k_probe = kc.copy()
        blk, off = int(table[t // BS]), t % BS
        k_probe[blk, :, off, 0] = 0x7E  # 448: dominates every other score
        out = oracle.paged_history_attention(q, k_probe, c.v_cache.numpy(), 1.0, c.v_scale,
                                             table, BS, c.actual_history_len, 1.0, c.num_kv_groups)
        want = e4m3fn_to_float64(c.v_cache.numpy()[blk, :, off, :]) * c.v_scale   # [Hkv, D]
        for h in range(c.q.shape[0]):
            assert np.allclose(out[h, 0], want[h // c.num_kv_groups], rtol=0, atol=1e-12)


def test_paged_relabel_pool_invariance():
    c = _small_paged(seed=23)
    NB = c.k_cache.shape[0]
    BS = c.block_size
    base = oracle.paged_history_attention(c.q.double().numpy(), c.k_cache.numpy(),
                                          c.v_cache.numpy(), c.k_scale, c.v_scale,
                                          c.block_table.numpy(), BS, c.actual_history_len,
                                          c.softmax_scale, c.num_kv_groups)
    perm = np.random.default_rng(0).permutation(NB)       # new physical id of old block b = perm[b]
    k2 = np.empty_like(c.k_cache.numpy())
    v2 = np.empty_like(c.v_cache.numpy())
    k2[perm] = c.k_cache.numpy()
    v2[perm] = c.v_cache.numpy()
    t2 = perm[c.block_table.numpy()].astype(np.int32)
    moved = oracle.paged_history_attention(c.q.double().numpy(), k2, v2, c.k_scale, c.v_scale, t2,
                                           BS, c.actual_history_len, c.softmax_scale,
                                           c.num_kv_groups)
    assert np.array_equal(base, moved)


# ---------------------------------------------------------------- FP8 decoder
def test_e4m3fn_fixed_points():
    t = E4M3FN_TABLE
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and math.copysign(1, t[0x80]) == -1
    assert t[0x01] == 2.0 ** -9                 # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9             # largest subnormal
    assert t[0x08] == 2.0 ** -6                 # smallest normal
    assert t[0x38] == 1.0                       # exponent field 7 = bias
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2             # FN: no infinities, two NaN codes


def test_e4m3fn_matches_torch_cast_for_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = e4m3fn_to_float64(codes.numpy())
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# ---------------------------------------------------------------- FLOP accounting
def test_flop_formula_reproduces_page_mfu(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "pcp_mfu_table.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    assert len(rows) >= 9
    for q_tok, hist, chips, ms, mfu in rows:
        fl = oracle.attention_flops(1, 32, q_tok, hist, 256)
        got = 100.0 * fl / (ms * 1e-3) / (chips * 667e12)
        assert abs(got - mfu) / mfu < 1.5e-3, (q_tok, hist, ms, got, mfu)


# ---------------------------------------------------------------- planted mistakes
def _mutants():
    """Plausible mistakes, planted in a copy of the oracle's row kernel."""
    def no_scale(q_rows, k_head, v_head, scale, mask_rows):
        return oatt._orig_rows(q_rows, k_head, v_head, 1.0, mask_rows)

    def bad_sign(q_rows, k_head, v_head, scale, mask_rows):
        return oatt._orig_rows(q_rows, k_head, v_head, -scale, mask_rows)

    def dropped_mask(q_rows, k_head, v_head, scale, mask_rows):
        return oatt._orig_rows(q_rows, k_head, v_head, scale, None)

    def wrong_value_rows(q_rows, k_head, v_head, scale, mask_rows):
        return oatt._orig_rows(q_rows, k_head, v_head[::-1], scale, mask_rows)

    def no_normalise(q_rows, k_head, v_head, scale, mask_rows):
        o, lse = oatt._orig_rows(q_rows, k_head, v_head, scale, mask_rows)
        return o * 1.5, lse

    return [no_scale, bad_sign, dropped_mask, wrong_value_rows, no_normalise]


@pytest.mark.parametrize("idx", range(5))
def test_planted_mistakes_are_caught(monkeypatch, idx):
    oatt._orig_rows = oatt._rows_attention
    mutant = _mutants()[idx]
    monkeypatch.setattr(oatt, "_rows_attention", mutant)
    failures = 0
    for check in (test_brute_force_with_mask, lambda: test_matches_torch_sdpa_float64(2)):
        try:
            check()
        except AssertionError:
            failures += 1
    assert failures >= 1, mutant.__name__
