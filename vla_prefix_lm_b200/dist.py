"""Multi-process plumbing for running the attention on several GPUs.

The joint attention is independent per batch element (each element carries its
own tokens, mask and prefix cache), so N GPUs run N replicas over disjoint
batch shards with no collective on the data path.  torch.distributed is used
only to line the ranks up (barrier) and to take the maximum of the per-rank
device times.  One process per GPU; RANK / WORLD_SIZE / LOCAL_RANK come from
the launcher's environment.
"""

from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str | None = None, timeout_s: float = 120.0) -> bool:
    """Initialises the default process group when WORLD_SIZE > 1; returns True if it did."""
    rank, ws, local = world()
    if ws <= 1 or dist.is_initialized():
        return dist.is_initialized()
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return True


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    """Maximum of a per-rank scalar (identity with one process)."""
    if not dist.is_initialized():
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) \
        if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not dist.is_initialized():
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) \
        if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
