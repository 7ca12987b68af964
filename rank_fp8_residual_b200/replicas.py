"""Multi-GPU execution of the forward as token-sharded replicas.

The forward shards by tokens with no exchange step: every output row y[m]
depends only on x[m] and the layer's factors.  So N GPUs run N independent
replicas, one process per GPU: each holds the whole layer, draws (or is
given) its own tokens and calls the library on them; nothing crosses
between GPUs on the data path.  The only collectives are the host-side
timing ones: a barrier around the timed region and the maximum of the
ranks' device times, so that the reported rate is the whole job's (all
ranks' units over the slowest rank's time).

Process-group plumbing goes through torch.distributed (nccl on GPUs, gloo
for the CPU tests); nothing here touches the compute path.
"""
from __future__ import annotations

import datetime
import os


def rank_env():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def token_seed(rank: int, base: int = 1000) -> int:
    """Seed of a rank's synthetic tokens: rank 0 uses the workload's own
    tokens (seed 0), rank k > 0 draws from seed base + k, so no two ranks
    process the same tokens."""
    return 0 if rank == 0 else base + rank


def init(backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Join the process group (MASTER_ADDR / MASTER_PORT from the
    environment) with a short timeout, so that ranks waiting for a rank
    that left end with an error instead of waiting for good."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def world_size() -> int:
    import torch.distributed as dist
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def barrier() -> None:
    import torch.distributed as dist
    if world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world_size() == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, steps: int, max_time_s: float, world: int) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time."""
    return world * steps * units_per_rank / max_time_s


def finalize() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
