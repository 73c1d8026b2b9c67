"""Host plumbing for running the layer as independent per-GPU replicas.

On one GPU the layer has no exchange step, so N GPUs run N independent
replicas (one process each, launched by torchrun).  The only cross-process
traffic is plumbing: a barrier around the timed region and the max of the
per-rank timings.  Works with NCCL (GPU ranks) and gloo (CPU ranks in tests).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info(env=None) -> RankInfo:
    env = os.environ if env is None else env
    return RankInfo(int(env.get("RANK", 0)), int(env.get("WORLD_SIZE", 1)), int(env.get("LOCAL_RANK", 0)))


def physical_gpu_index(local_rank: int, env=None) -> int:
    """nvidia-smi index of this rank's GPU (honours CUDA_VISIBLE_DEVICES when it lists indices)."""
    env = os.environ if env is None else env
    vis = env.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(parts) and parts[local_rank].isdigit():
            return int(parts[local_rank])
    return local_rank


def init(info: RankInfo, backend: str, timeout_s: float = 120.0, device=None):
    """Join the process group (no-op for a single process)."""
    if info.world <= 1:
        return
    import torch.distributed as dist
    kw = {"backend": backend, "timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(**kw)


def barrier(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, info: RankInfo, device="cpu") -> float:
    """Maximum of a per-rank scalar (e.g. the timed region's milliseconds) over all ranks."""
    if info.world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
