"""One process per GPU, independent replicas (no data-path collective).

A 10-step chunk is a serial chain of ~900 dependent phases, so it does not
shard across GPUs; independent chunks (robots, requests) do.  Each rank
holds a full copy of the expert and serves its own chunks.  The only
collectives are the host-side barrier and the max-over-ranks reduction of
the measured time.
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass
class RankInfo:
    rank: int = 0
    world: int = 1
    local_rank: int = 0

    @property
    def is_main(self) -> bool:
        return self.rank == 0


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                    int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, timeout_s: float = 120.0) -> RankInfo:
    """Join the process group when launched with WORLD_SIZE > 1."""
    info = rank_info()
    if info.world > 1:
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if not dist.is_initialized():
            kw = {}
            if backend == "nccl":
                import torch
                kw["device_id"] = torch.device("cuda", info.local_rank)
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return info


def barrier(info: RankInfo, device=None):
    if info.world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def max_over_ranks(value: float, info: RankInfo, device=None) -> float:
    """The largest value any rank measured (timings are reported as the max)."""
    if info.world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, info: RankInfo, device=None) -> float:
    if info.world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shutdown(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
