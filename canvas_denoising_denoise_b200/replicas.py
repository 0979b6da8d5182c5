"""Host plumbing for running the denoising path as independent replicas.

The block-autoregressive denoiser has no data-path exchange: every sequence
is denoised against its own KV cache, so N GPUs run N independent replicas,
one process per GPU, each with its own prompts and sampler seed.  The only
inter-process traffic is timing: a barrier on both sides of the timed region
and the maximum of the per-rank device times, so that the whole-job rate is
the work of all ranks divided by the slowest rank's time.

Everything here is backend-agnostic (NCCL on GPUs, gloo on CPU) so that the
N>1 host path can be exercised without GPUs.
"""
import datetime
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankEnv:
    rank: int
    world: int
    local: int


def rank_env(environ=None) -> RankEnv:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (1 rank if unset)."""
    e = os.environ if environ is None else environ
    rank = int(e.get("RANK", "0"))
    world = int(e.get("WORLD_SIZE", "1"))
    local = int(e.get("LOCAL_RANK", str(rank)))
    if world < 1 or not 0 <= rank < world or local < 0:
        raise ValueError(f"inconsistent rank environment: rank={rank} world={world} local={local}")
    return RankEnv(rank, world, local)


@dataclass(frozen=True)
class ReplicaSeeds:
    prompt: int   # seed of the synthetic prompt generator
    sampler: int  # Philox key word 0 of the sampler draws


def replica_seeds(rank: int) -> ReplicaSeeds:
    """Per-rank seeds: distinct prompts and distinct sampler streams per replica."""
    if rank < 0:
        raise ValueError("rank must be non-negative")
    return ReplicaSeeds(prompt=1 + rank, sampler=1000 + rank)


def init(backend: str, timeout_s: float = 120.0) -> None:
    """Join the process group (rendezvous from MASTER_ADDR / MASTER_PORT)."""
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def _device():
    import torch
    import torch.distributed as dist
    if dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """The maximum of `value` over all ranks (the identity for one rank)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, max_elapsed_s: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    if max_elapsed_s <= 0:
        raise ValueError("elapsed time must be positive")
    return world * units_per_rank / max_elapsed_s


def finish(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
