"""The kernels' bounded waits: when one runs out, the call reports ATTN_ERR_DEVICE_TIMEOUT
and the GPU context stays usable.

A copy of the library is built with ATTN_WAIT_LIMIT_NS = 1, non-blocking polls and the clock
read after every failed poll (every mbarrier wait of the compute path that is not complete at
once gives up as soon as the global timer moves), while the teardown drains keep
their full one-second limit, so every copy and MMA a CTA started still lands before it
exits and TMEM is freed only once the tensor core is done with it. Each entry point of
that copy must then report the timeout through attn_check; afterwards the product
library, in the same process, must still produce oracle-exact results.
No fault is provoked: the waits simply stop early and the kernels return.
"""

import ctypes

import pytest
import torch

import oracle
from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import build as build_mod
from online_softmax_attention_flash_b200 import inputs as syn
from parity import FP8_REL_L2, assert_bf16_parity, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TIMEOUT = -7   # ATTN_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module")
def short_wait_lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("shortwait") / "libattn_shortwait.so")
    build_mod.build(force=True, out=out,
                    extra_flags=["-DATTN_WAIT_LIMIT_NS=1ull", "-DATTN_WAIT_SPINS_PER_CHECK=1u",
                                 "-DATTN_WAIT_TEST_POLL"])
    lib = ctypes.CDLL(out)
    for name, res, args in B.SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _until_timeout(lib, launch, tries=5):
    """Launch through the short-wait copy until its device status reports the timeout."""
    seen = []
    for _ in range(tries):
        assert launch() == 0
        st = lib.attn_check(_stream())
        seen.append(st)
        if st == TIMEOUT:
            return seen
    return seen


@pytest.mark.parametrize("D,with_bias", [(64, False), (64, True), (128, False), (128, True)],
                         ids=["d64", "d64_key_bias", "d128", "d128_key_bias"])
def test_encoder_wait_timeout_is_reported(short_wait_lib, D, with_bias):
    c = syn.encoder_case(1, 4, 1024, D, seed=501)
    q, k, v = (t.to(DEV) for t in (c.q, c.k, c.v))
    kb = torch.zeros((1, 1024), dtype=torch.float32, device=DEV) if with_bias else None
    if kb is not None:
        kb[0, 900:] = float("-inf")
    out = torch.empty_like(q)
    seen = _until_timeout(short_wait_lib, lambda: short_wait_lib.attn_encoder_fwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), 1, 4, 1024, D, 0.125,
        None if kb is None else kb.data_ptr(), _stream()))
    assert seen[-1] == TIMEOUT, seen
    torch.cuda.synchronize()   # the context is intact
    # the product library, same process, same inputs: exact as ever
    good = B.attn_encoder_fwd(q, k, v, 0.125, key_bias=kb)
    assert B.attn_check() == 0
    ref = oracle.encoder_attention(to_f64(c.q), to_f64(c.k), to_f64(c.v), 0.125,
                                   key_bias=None if kb is None else kb.double().cpu().numpy())
    assert_bf16_parity(good, ref, 2, "encoder after a timed-out call")


def test_decode_wait_timeout_is_reported(short_wait_lib):
    c = syn.decode_case(8, 16, 8, 4096, 256, seed=502)
    q, k, v, m = (t.to(DEV) for t in (c.q, c.k, c.v, c.attn_mask))
    out = torch.empty_like(q)
    ws_bytes = B.attn_gqa_decode_workspace_size(8, 16, 8, 4096, 256)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    seen = _until_timeout(short_wait_lib, lambda: short_wait_lib.attn_gqa_decode(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), m.data_ptr(), out.data_ptr(), 8, 16, 8, 2, 4096,
        256, 1.0, ws.data_ptr(), ws_bytes, _stream()))
    assert seen[-1] == TIMEOUT, seen
    torch.cuda.synchronize()
    good = B.attn_gqa_decode(q, k, v, m, 1.0, 2, workspace=ws)
    assert B.attn_check() == 0
    ref = oracle.gqa_decode_attention(to_f64(c.q), to_f64(c.k), to_f64(c.v),
                                      c.attn_mask.double().numpy(), 1.0, 2)
    assert_bf16_parity(good, ref, 2, "decode after a timed-out call")


def test_paged_wait_timeout_is_reported(short_wait_lib):
    p = syn.paged_case(8, 2, 512, 256, num_phys_blocks=8, block_size=512, actual_history_len=3000,
                       seed=503, softmax_scale=1.0 / 16)
    q, kc, vc, bt = (t.to(DEV) for t in (p.q, p.k_cache, p.v_cache, p.block_table))
    out = torch.empty_like(q)
    seen = _until_timeout(short_wait_lib, lambda: short_wait_lib.attn_paged_history(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), bt.data_ptr(), bt.numel(), 8, 512, 3000,
        p.k_scale, p.v_scale, p.softmax_scale, 8, 2, 4, 512, 256, out.data_ptr(), _stream()))
    assert seen[-1] == TIMEOUT, seen
    torch.cuda.synchronize()
    good = B.attn_paged_history(q, kc, vc, bt, 512, 3000, p.k_scale, p.v_scale, p.softmax_scale, 4)
    assert B.attn_check() == 0
    ref = oracle.paged_history_attention(to_f64(p.q), p.k_cache.numpy(), p.v_cache.numpy(),
                                         p.k_scale, p.v_scale, p.block_table.numpy(), 512, 3000,
                                         p.softmax_scale, 4)
    assert rel_l2(to_f64(good), ref) <= FP8_REL_L2


def test_projection_wait_timeout_is_reported(short_wait_lib):
    c = syn.projection_case(1, 512, 256, 4, 64, seed=504)
    x, w, bq = c.x.to(DEV), c.w_qkv.to(DEV), c.b_qkv.to(DEV)
    q, k, v = (torch.empty((1, 4, 512, 64), dtype=torch.bfloat16, device=DEV) for _ in range(3))
    seen = _until_timeout(short_wait_lib, lambda: short_wait_lib.attn_qkv_rope_proj(
        x.data_ptr(), w.data_ptr(), bq.data_ptr(), None, None, 0, 1, 512, 256, 4, 64,
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _stream()))
    assert seen[-1] == TIMEOUT, seen
    torch.cuda.synchronize()
    gq, gk, gv = B.attn_qkv_rope_proj(x, w, bq, 4, 64)
    assert B.attn_check() == 0
    ref = oracle.qkv_projection(to_f64(c.x), to_f64(c.w_qkv), c.b_qkv.double().numpy(), 4, 64)
    for g, r, n in zip((gq, gk, gv), ref, "qkv"):
        assert_bf16_parity(g, r, 2, f"{n} after a timed-out call")
