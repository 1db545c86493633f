"""Data-parallel plumbing: one process per GPU, sequences sharded over ranks.

Decode over a latent cache has no exchange between sequences, so the data
path carries no collective.  torch.distributed is used only to agree on
timings (max over ranks) and for barriers around timed regions.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as td


def env_world() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str = "nccl", timeout_s: int = 120) -> Tuple[int, int, int]:
    rank, local, world = env_world()
    if world > 1 and not td.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        td.init_process_group(backend=backend, rank=rank, world_size=world,
                              timeout=datetime.timedelta(seconds=timeout_s), **kw)
    elif torch.cuda.is_available() and backend == "nccl":
        torch.cuda.set_device(local)
    return rank, local, world


def shard(num_units: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [begin, end) share of ``num_units`` for ``rank`` (sizes differ by <= 1)."""
    base, extra = divmod(num_units, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Distinct, reproducible data per rank (weak scaling: every rank has its own batch)."""
    return seed + 7919 * rank


def _device_for_collectives() -> torch.device:
    if td.is_initialized() and td.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def max_over_ranks(x: float) -> float:
    if not (td.is_available() and td.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device_for_collectives())
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not (td.is_available() and td.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device_for_collectives())
    td.all_reduce(t, op=td.ReduceOp.SUM)
    return float(t.item())


def barrier() -> None:
    if td.is_available() and td.is_initialized():
        if td.get_backend() == "nccl":
            td.barrier(device_ids=[torch.cuda.current_device()])
        else:
            td.barrier()


def finish() -> None:
    if td.is_available() and td.is_initialized():
        td.destroy_process_group()
