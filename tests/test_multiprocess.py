"""Host-side multi-process paths (world size 2, gloo, CPU only).

bench.py runs one process per GPU; ranks run independent replicas of the
workload, meet at a barrier around the timed region and report the max of
their times. These tests exercise that plumbing with two gloo ranks on the CPU,
and the rank-0-only behaviour of the oracle (reference) arm.
"""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    from online_softmax_attention_flash_b200 import dist as D
    info = D.init("gloo", timeout_s=60)
    D.barrier(info)
    m = D.max_over_ranks(1.5 + rank, info)
    D.barrier(info)
    D.shutdown(info)
    q.put((rank, info.world_size, info.is_main, m))


def test_two_gloo_ranks_barrier_and_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2, True, 2.5), (1, 2, False, 2.5)]


def test_rank_info_defaults_to_single_process(monkeypatch):
    from online_softmax_attention_flash_b200 import dist as D
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    info = D.init("gloo")
    assert (info.rank, info.local_rank, info.world_size, info.is_main) == (0, 0, 1, True)
    assert D.max_over_ranks(3.0, info) == 3.0


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
                         "--workload", "tiny"])
    assert rc == 0 and buf.getvalue() == ""
    monkeypatch.setenv("RANK", "0")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
                         "--workload", "tiny"])
    line = json.loads(buf.getvalue().strip())
    assert rc == 0 and line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["value"] > 0


@pytest.mark.parametrize("workload", ["tiny", "decode"])
def test_reference_arm_units_match_product_arm(workload, monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", workload])
    line = json.loads(buf.getvalue().strip())
    assert line["unit"] == ("GB/s" if workload == "decode" else "TFLOP/s")
    assert line["metric"] == bench.METRIC
