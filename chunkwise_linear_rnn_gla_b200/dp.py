"""Host-side logic of the data-parallel run: one process per GPU, every rank
runs the whole layer on its own batch shard (weak scaling: the layer has no
exchange between independent sequences, so the data path needs no
collective). The only cross-rank steps are the barriers around the timed
region and the reduction of the per-rank device time to its maximum.

Nothing here touches the GPU; the functions take the process group (NCCL
on GPUs, gloo in the CPU tests) and plain numbers.
"""
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankEnv:
    rank: int
    world: int
    local_rank: int


def rank_env(environ=None) -> RankEnv:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (1 process if unset)."""
    env = os.environ if environ is None else environ
    world = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if world < 1 or not (0 <= rank < world) or local < 0:
        raise ValueError("bad rank environment: RANK=%d WORLD_SIZE=%d LOCAL_RANK=%d" % (rank, world, local))
    return RankEnv(rank, world, local)


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of the synthetic batch shard of `rank` (distinct per rank)."""
    return int(base_seed) * 1000003 + int(rank)


def global_batch(per_rank_batch: int, world: int) -> int:
    return int(per_rank_batch) * int(world)


def max_over_ranks(value: float, group=None) -> float:
    """Maximum of a per-rank scalar (e.g. the device time of the timed region) over all ranks."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_throughput(units_per_rank_step: float, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: the units all ranks processed per step over the slowest rank's step time."""
    if max_ms_per_step <= 0:
        raise ValueError("step time must be positive")
    return float(units_per_rank_step) * int(world) / (max_ms_per_step / 1e3)
