"""Running the tensor product on several GPUs of one node: one process per GPU,
each working on its own independent problems (graphs, batches, configurations).

The edge-wise tensor product of one graph needs no data from another graph, so
the units of work are split between ranks and no collective touches the data
path. The only communication is host-side bookkeeping: a barrier around a timed
region and the maximum of the ranks' times (a job is as slow as its slowest
rank). These helpers take their backend from the device: NCCL for CUDA tensors,
gloo for CPU (used by the tests).
"""
from __future__ import annotations

import datetime
import os


def rank_env() -> tuple:
    """(rank, world_size, local_rank) from the launcher's environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, device, timeout_s: float = 120.0) -> None:
    """Join the process group when world > 1 (MASTER_ADDR / MASTER_PORT from the env)."""
    import torch.distributed as dist

    if world <= 1 or dist.is_initialized():
        return
    timeout = datetime.timedelta(seconds=timeout_s)
    if getattr(device, "type", "cpu") == "cuda":
        dist.init_process_group("nccl", timeout=timeout, device_id=device)
    else:
        dist.init_process_group("gloo", timeout=timeout)


def barrier(world: int) -> None:
    import torch.distributed as dist

    if world > 1:
        dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous block of the units [0, n_units) owned by `rank`: the blocks are
    disjoint, cover every unit, and differ in size by at most one."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("need 0 <= rank < world and n_units >= 0")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def finalize(world: int) -> None:
    import torch.distributed as dist

    if world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
