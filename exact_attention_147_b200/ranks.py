"""One process per GPU: rank discovery, process-group set-up and the two
collectives the benchmark needs around its timed region.

Exact attention over a batch splits into independent (batch, head) problems
with nothing exchanged between them ("FlashAttention-2" abstract: the work
is spread over thread blocks even within one head, and heads and batches
never interact).  Across GPUs the library therefore shards whole batches:
every rank runs its own batch of the same shape (weak scaling) and no
collective touches the data path.  The only collectives are a barrier on
each side of a timed region and the maximum of the ranks' times, both on
the host's schedule, between kernel launches.

Backends: "nccl" with one CUDA device per rank on a GPU node, "gloo" on the
CPU (used by the tests to run the same logic with two processes).
"""

from __future__ import annotations

import datetime
import os


def rank_env():
    """(rank, world size, local rank) from the launcher's environment; a
    process started without a launcher is rank 0 of 1."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init(backend: str = "nccl", timeout_s: float = 120.0):
    """Join the process group named by the environment (MASTER_ADDR,
    MASTER_PORT, RANK, WORLD_SIZE).  A short timeout turns a rank that never
    arrives into an error on the others instead of a wait without end.
    Returns (rank, world, local); world 1 creates no group."""
    import torch
    import torch.distributed as dist

    rank, world, local = rank_env()
    if world <= 1:
        return rank, world, local
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, world, local


def batch_seed(base: int, rank: int) -> int:
    """Seed of the synthetic batch rank `rank` draws: every rank owns a
    different batch of the same shape."""
    return base + rank


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest x over all ranks (device: "cuda" for NCCL, "cpu" for
    gloo)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Units all ranks processed per second of the slowest rank (weak
    scaling: each rank processes units_per_rank)."""
    return world * units_per_rank / slowest_seconds


def finalize(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
