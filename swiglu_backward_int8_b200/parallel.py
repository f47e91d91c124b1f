"""Host-side helpers for running the op on several GPUs (one process per GPU).

The op partitions with no exchange: a row group lies inside one token and a
column group inside one 128-token block ("kernelgen-challenge-9-task3-silu-quant",
outputs section: row-wise 128-channel groups, 128-token groups of y), so a
split of the tokens into 128-aligned ranges gives every rank exactly the
global result restricted to its tokens.  Nothing here moves data between GPUs;
the only collective is the max-over-ranks of a timing.
"""
from __future__ import annotations

from typing import Optional, Tuple

GROUP = 128


def shard_rows(M: int, world: int, rank: int, group: int = GROUP) -> Tuple[int, int]:
    """Token range [m0, m1) of `rank` out of `world`: whole 128-token groups,
    as even as possible (the first M_groups % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of world {world}")
    groups = (M + group - 1) // group
    base, extra = divmod(groups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return min(M, g0 * group), min(M, g1 * group)


def group_range(m0: int, m1: int, group: int = GROUP) -> Tuple[int, int]:
    """Columns [i0, i1) of y_s_t that the token range [m0, m1) owns (m0 must be
    128-aligned unless the range is empty)."""
    if m0 == m1:
        i = (m0 + group - 1) // group
        return i, i
    if m0 % group:
        raise ValueError("shard start must be a multiple of the group size")
    return m0 // group, (m1 + group - 1) // group


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Maximum of a per-rank number over all ranks (identity without a
    process group).  NCCL needs a CUDA device; gloo works on the CPU."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def aggregate_gbs(bytes_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput in GB/s: the bytes of all ranks over the slowest
    rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


def barrier(device=None, group=None) -> None:
    """A barrier that works on NCCL (through a tiny all-reduce on `device`)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return
    t = torch.zeros(1, device=device)
    dist.all_reduce(t, group=group)
    if device is not None and torch.device(device).type == "cuda":
        torch.cuda.synchronize(device)


def init_from_env(backend: str = "nccl", timeout_s: float = 120.0,
                  device: Optional[object] = None) -> Tuple[int, int, int]:
    """(world, rank, local_rank) from the torchrun environment; initialises the
    process group when world > 1."""
    import datetime
    import os
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if (backend == "nccl" and device is not None) else {}
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local
