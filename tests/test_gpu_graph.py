"""The entry points can be captured in a CUDA graph (after a first eager call on the
device) and replaying the graph gives the eager results bit for bit."""

import pytest
import torch

from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import inputs as syn

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_graph_replay_matches_eager_for_all_entry_points():
    e = syn.encoder_case(2, 4, 300, 64, seed=1)
    d = syn.decode_case(2, 8, 4, 1000, 256, seed=2)
    p = syn.paged_case(4, 2, 200, 256, num_phys_blocks=4, block_size=512,
                       actual_history_len=1800, seed=3, softmax_scale=1 / 16)
    eq, ek, ev = (t.to(DEV) for t in (e.q, e.k, e.v))
    dq, dk, dv, dm = (t.to(DEV) for t in (d.q, d.k, d.v, d.attn_mask))
    pq, pk, pv, pt = (t.to(DEV) for t in (p.q, p.k_cache, p.v_cache, p.block_table))
    f = syn.paged_prefill_case(4, 2, 256, 128, hist_lens=[300, 0], q_lens=[150, 90], seed=4,
                               softmax_scale=1 / 16)
    fq, fk, fv, ft, fs, fh = (t.to(DEV) for t in (f.q, f.k_cache, f.v_cache, f.block_tables,
                                                  f.q_start, f.hist_lens))
    rc, rs = (t.to(DEV) for t in syn.rope_tables(300, 64))
    ws = torch.zeros(B.attn_gqa_decode_workspace_size(2, 8, 4, 1000, 256), dtype=torch.uint8,
                     device=DEV)
    outs = [torch.empty_like(eq), torch.empty_like(dq), torch.empty_like(pq), torch.empty_like(fq),
            torch.empty_like(eq), torch.empty_like(ek)]

    def calls():
        B.attn_encoder_fwd(eq, ek, ev, e.softmax_scale, out=outs[0])
        B.attn_gqa_decode(dq, dk, dv, dm, d.softmax_scale, d.num_kv_groups, out=outs[1],
                          workspace=ws)
        B.attn_paged_history(pq, pk, pv, pt, p.block_size, p.actual_history_len, p.k_scale,
                             p.v_scale, p.softmax_scale, p.num_kv_groups, out=outs[2])
        B.attn_paged_prefill(fq, fk, fv, ft, fs, fh, f.k_scale, f.v_scale, f.softmax_scale,
                             f.num_kv_groups, max_q_len=150, out=outs[3])
        B.attn_rope_qk(eq, ek, rc, rs, interleaved=True, q_out=outs[4], k_out=outs[5])

    calls()   # first calls on the device happen outside the capture
    assert B.attn_check() == 0
    eager = [o.clone() for o in outs]
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert B.attn_check() == 0
    for a, b in zip(eager, outs):
        assert torch.equal(a, b)
