"""The allocation-free decode entry point, attn_gqa_decode_noalloc.

Some callers cannot allocate device memory: hosts that own the whole memory
budget and forbid allocations once they are running, and latency-critical
loops that cannot pay for cudaMalloc's possible device-wide synchronisation.
They cannot hand attn_gqa_decode a workspace, so the library offers a variant
whose split-KV partials live in a scratch array reserved statically on the
device. These tests call it through the C ABI and check that it returns what
the workspace-taking entry point returns, twice in a row (the scratch keeps the
previous call's contents, so the second call must not be affected by the first).

This file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn
from parity import BF16_HEAD_COS, BF16_REL_L2, head_cosines, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _device_case(case):
    return tuple(t.to(DEV) for t in (case.q, case.k, case.v, case.attn_mask))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [syn.decode_case(8, 16, 8, 4096, 256, seed=4242, softmax_scale=1.0),
             syn.decode_case(3, 8, 2, 1500, 512, seed=4343, softmax_scale=512 ** -0.5,
                             min_len=1)]
    for i, case in enumerate(cases):   # two calls in a row, different sizes and contents
        q, k, v, m = _device_case(case)
        need = B.attn_gqa_decode_workspace_size(q.shape[0], q.shape[1], k.shape[1], k.shape[2],
                                                q.shape[3])
        assert need <= B.NOALLOC_SCRATCH_BYTES
        ref = B.attn_gqa_decode(q, k, v, m, case.softmax_scale, case.num_kv_groups)
        got = B.attn_gqa_decode_noalloc(q, k, v, m, case.softmax_scale, case.num_kv_groups)
        assert B.attn_check() == 0
        # same kernels and the same deterministic split: identical bits, so an offset or
        # carve error in the scratch would show even if it moved the result only slightly
        assert torch.equal(got, ref)
        g, r = to_f64(got), to_f64(ref)
        assert rel_l2(g, r) <= BF16_REL_L2
        assert head_cosines(g, r, 2).min() >= BF16_HEAD_COS
        if i == 1:   # and the oracle agrees (tolerance of the bf16 paths)
            want = oracle.gqa_decode_attention(to_f64(case.q), to_f64(case.k), to_f64(case.v),
                                               case.attn_mask.double().numpy(),
                                               case.softmax_scale, case.num_kv_groups)
            assert rel_l2(g, want) <= BF16_REL_L2
            assert head_cosines(g, want, 2).min() >= BF16_HEAD_COS


def test_noalloc_call_leaves_free_device_memory_unchanged():
    case = syn.decode_case(4, 8, 4, 2048, 256, seed=4444)
    q, k, v, m = _device_case(case)
    out = torch.empty_like(q)
    B.attn_gqa_decode_noalloc(q, k, v, m, case.softmax_scale, case.num_kv_groups, out=out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        B.attn_gqa_decode_noalloc(q, k, v, m, case.softmax_scale, case.num_kv_groups, out=out)
    assert B.attn_check() == 0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    lib = B.load_library()
    fake = ctypes.c_void_p(4096)   # never dereferenced: the size check comes first
    # 64 batch entries x 8192 sub-tiles of lists alone are beyond the scratch
    st = lib.attn_gqa_decode_noalloc(fake, fake, fake, None, fake, 64, 64, 8, 8, 65536, 512,
                                     1.0, None)
    assert st == -5   # ATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
