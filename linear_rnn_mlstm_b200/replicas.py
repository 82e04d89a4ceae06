"""Host-side plumbing for running the forward/decode as independent replicas,
one process per GPU (heads are independent in the mLSTM cell -- "xLSTM:
Extended Long Short-Term Memory" section 2.3: no memory mixing between heads --
so the batch shards across GPUs with no data-path collective).

Everything here is device-agnostic: with the NCCL backend the timing tensor
lives on the rank's GPU, with gloo on the CPU.  The only collectives are the
barriers around a timed region and the max over ranks of its duration.
"""
import datetime
import os
from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankEnv:
    world: int
    rank: int
    local_rank: int

    @property
    def distributed(self) -> bool:
        return self.world > 1

    @property
    def reports(self) -> bool:
        """Only rank 0 prints the result line."""
        return self.rank == 0


def rank_env(env: Optional[dict] = None) -> RankEnv:
    """WORLD_SIZE / RANK / LOCAL_RANK as set by torch.distributed.run (defaults:
    a single process)."""
    env = os.environ if env is None else env
    world = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local_rank = int(env.get("LOCAL_RANK", str(rank)))
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank environment: WORLD_SIZE={world} RANK={rank}")
    return RankEnv(world, rank, local_rank)


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own synthetic batch (a different shard of heads)."""
    return base_seed + rank


def init(env: RankEnv, backend: str, device: Optional[torch.device] = None, timeout_s: float = 300.0):
    """Join the process group (a no-op for one process).  A short timeout makes a
    rank that never arrives end the others' next collective with an error."""
    if not env.distributed:
        return
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def barrier(env: RankEnv):
    if env.distributed:
        dist.barrier()


def max_over_ranks(value: float, env: RankEnv, device: Optional[torch.device] = None) -> float:
    """The largest of the ranks' values (every rank gets it): the duration of a
    timed region is the slowest replica's."""
    if not env.distributed:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, env: RankEnv, seconds: float) -> float:
    """Whole-job throughput: the units all replicas processed over the slowest
    replica's time (weak scaling: per-replica work is fixed)."""
    return units_per_rank * env.world / seconds


def shutdown(env: RankEnv):
    if env.distributed and dist.is_initialized():
        dist.destroy_process_group()
