"""Multi-process plumbing for running the pruning / decode path on several
GPUs of one node.

SparK's work splits into independent (layer, batch row, kv head) units: a
unit's pruning, statistics and decode read nothing from any other unit, so
the path shards with no data-path collective.  Each rank owns a contiguous
range of units (or, for weak scaling, a whole replica of the workload); the
only cross-rank operations are a barrier around the timed region and a max of
the ranks' device times.  One process per GPU, launched by torchrun.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank_world() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> tuple[int, int]:
    """Initialise the default process group (short timeout so that ranks
    waiting on a missing peer fail instead of hanging).  Returns
    (rank, world_size)."""
    rank, local, world = env_rank_world()
    if world == 1:
        return 0, 1
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return dist.get_rank(), dist.get_world_size()


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous block of units [start, stop) owned by `rank`: sizes differ
    by at most one, blocks are disjoint and cover 0..n_units-1 in order."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank scalar (e.g. elapsed device time) over ranks."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finalize() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
