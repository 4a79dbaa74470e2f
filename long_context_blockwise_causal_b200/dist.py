"""Multi-GPU helpers: one process per GPU, independent shards.

The attention problems of different (batch row, head) pairs are
independent, so a job spreads over G GPUs by giving each rank a contiguous
slice of heads (strong scaling: the whole job is fixed) or a full replica
(weak scaling). Neither needs a collective on the data path; the process
group only synchronises timing (barrier, max over ranks).
"""

from __future__ import annotations

import datetime
import os


def head_shard(H: int, world: int, rank: int) -> tuple[int, int]:
    """[h0, h1) of rank `rank` when H heads are split over `world` ranks:
    the first H % world ranks take one extra head."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def init_from_env(backend: str = "nccl", timeout_s: int = 120):
    """Initialise torch.distributed from torchrun's environment (no-op for
    a single process). Returns (world, rank, local_rank)."""
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(
            backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (the job's time is the slowest
    rank's)."""
    if world == 1:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())
