"""Process-group plumbing for multi-GPU runs (one process per GPU).

The attention path shards into independent problems (layers, batch entries,
heads), so N GPUs run N replicas of the workload with no data-path collective.
The only collectives are the timing barrier and the max-over-ranks of the
measured time, both here. Works with the NCCL backend on GPUs and with gloo on
the CPU (used by the tests).
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class RankInfo:
    rank: int
    local_rank: int
    world_size: int

    @property
    def is_main(self) -> bool:
        return self.rank == 0


def rank_info_from_env() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
                    int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0) -> RankInfo:
    """Initialise the default process group when WORLD_SIZE > 1 (env:// rendezvous)."""
    info = rank_info_from_env()
    if info.world_size > 1 and not dist.is_initialized():
        kwargs = dict(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
        if backend == "nccl":
            kwargs["device_id"] = torch.device("cuda", info.local_rank)
        dist.init_process_group(**kwargs)
    return info


def barrier(info: RankInfo) -> None:
    if info.world_size > 1:
        dist.barrier()


def max_over_ranks(value: float, info: RankInfo, device=None) -> float:
    """Max of a per-rank scalar; every rank must call it (same collective order)."""
    if info.world_size == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shutdown(info: RankInfo) -> None:
    if info.world_size > 1 and dist.is_initialized():
        dist.destroy_process_group()
