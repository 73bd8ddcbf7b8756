"""The paged kernel's precision design, measured on the CPU with the oracle's replay of its
roundings (oracle/precision_model.py) against the exact attention:

* the E4M3FN rounding agrees with torch's saturating round-to-nearest-even cast for a sweep
  of values (an independent implementation), including ties and the saturation point;
* with N(0, 1) inputs and 4096 history keys, splitting both bf16 operands into e4m3 hi + lo
  keeps the result at bf16-level accuracy, while one or no split does not (the reason the
  kernel spends two FP8 MMAs per matmul);
* the encoder's stale running max (refreshed only when a tile exceeds it by 2^8) is as
  accurate as the exact running max, and a replay that drops the O rescale is caught.
"""

import numpy as np
import torch

import oracle
from oracle import precision_model as pm
from online_softmax_attention_flash_b200 import inputs as syn


def test_e4m3_rounding_matches_torch_cast():
    x = np.concatenate([np.linspace(-500, 500, 20001), np.linspace(-0.02, 0.02, 4001),
                        pm._FINITE[1:-1] + np.diff(pm._FINITE)[1:] / 2])   # exact midpoints
    got = pm.e4m3_round(x)
    ref = torch.from_numpy(x.astype(np.float32)).clamp(-448, 448).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(got, ref)


def test_both_splits_are_needed_for_bf16_level_accuracy():
    c = syn.paged_case(1, 1, 64, 256, num_phys_blocks=8, block_size=512,
                       actual_history_len=4096, seed=31, softmax_scale=1 / 16)
    kl, vl = oracle.paged_logical_kv(c.k_cache.numpy(), c.v_cache.numpy(), 1.0, 1.0,
                                     c.block_table.numpy(), 512, 4096)
    q = c.q[0].double().numpy()
    ref = oracle.paged_history_attention(c.q.double().numpy(), c.k_cache.numpy(), c.v_cache.numpy(),
                                         c.k_scale, c.v_scale, c.block_table.numpy(), 512, 4096,
                                         c.softmax_scale, 1)[0]

    def err(sq, sp):
        out = pm.paged_history_emulated(q, kl[0], vl[0], c.k_scale, c.v_scale, c.softmax_scale,
                                        split_q=sq, split_p=sp)
        return np.linalg.norm(out - ref) / np.linalg.norm(ref)

    both, q_only, p_only, none = err(True, True), err(True, False), err(False, True), err(False, False)
    assert both <= 3e-3
    assert min(q_only, p_only) > 4 * both and none > 4 * both
    assert none >= max(q_only, p_only) * 0.9


def test_encoder_stale_max_threshold_costs_no_accuracy():
    """The encoder keeps a row's running max unless a tile exceeds it by more than 2^8:
    P may reach 256 before its bf16 rounding, which is relative, so the result is as
    accurate as with the exact running max (threshold 0)."""
    g = np.random.default_rng(41)
    L, D = 2048, 64
    q = pm.bf16_round(g.standard_normal(D))
    k = pm.bf16_round(g.standard_normal((L, D)))
    v = pm.bf16_round(g.standard_normal((L, D)))
    k[1500:1600] *= 4.0                          # a late block of large scores moves the max
    scale = 0.125
    ref = oracle.encoder_attention(q[None, None, None], k[None, None], v[None, None], scale)[0, 0, 0]
    s_log2 = (k @ q) * scale * np.log2(np.e)
    errs = {}
    for thr in (0.0, 8.0):
        out = pm.encoder_row_emulated(s_log2, v, thr)
        errs[thr] = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert errs[8.0] <= 3e-3 and errs[0.0] <= 3e-3
    assert errs[8.0] <= 2.0 * errs[0.0] + 1e-6


def test_planted_missing_rescale_is_caught():
    """A replay that forgets to rescale O when the max moves is caught by the same check."""
    g = np.random.default_rng(42)
    L, D = 1024, 32
    k, v = g.standard_normal((L, D)), g.standard_normal((L, D))
    q = g.standard_normal(D)
    k[700:] *= 3.0
    s_log2 = (k @ q) * 0.2 * np.log2(np.e)
    ref = oracle.encoder_attention(q[None, None, None], k[None, None], v[None, None], 0.2)[0, 0, 0]
    good = pm.encoder_row_emulated(s_log2, v, 8.0)
    real_exp2 = np.exp2

    def bad_row(s_row, v_, threshold, tile=128):
        m, l, o = -np.inf, 0.0, np.zeros(v_.shape[1])
        for j0 in range(0, s_row.shape[0], tile):
            s = s_row[j0:j0 + tile]
            if s.max() > m + threshold:
                l *= real_exp2(m - s.max()) if np.isfinite(m) else 0.0   # o is not rescaled
                m = s.max()
            p = real_exp2(s - m)
            l += p.sum()
            o += p @ v_[j0:j0 + tile]
        return o / l
    bad = bad_row(s_log2, v, 8.0)
    assert np.linalg.norm(good - ref) / np.linalg.norm(ref) < 3e-3
    assert np.linalg.norm(bad - ref) / np.linalg.norm(ref) > 1e-2
