"""The paged kernel's precision design, measured on the CPU with the oracle's replay of its
roundings (oracle/precision_model.py) against the exact attention:

* the E4M3FN rounding agrees with torch's saturating round-to-nearest-even cast for a sweep
  of values (an independent implementation), including ties and the saturation point;
* with N(0, 1) inputs and 4096 history keys, splitting both bf16 operands into e4m3 hi + lo
  keeps the result at bf16-level accuracy, while one or no split does not (the reason the
  kernel spends two FP8 MMAs per matmul).
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
