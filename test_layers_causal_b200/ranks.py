"""Host-side plumbing for running the layer on several GPUs of one node.

The layer shards naturally over independent sequences: every (b, h) pair has
its own fast weight, so a global batch splits along B with no exchange on the
data path ("replicas": each rank runs the layer on its own slice; weak scaling
gives every rank a full batch).  The only collectives here are for timing:
a barrier around the timed region and a max over ranks of the elapsed time.
NCCL is used on GPUs, gloo on CPU (tests).
"""
from __future__ import annotations

import dataclasses
import datetime
import os

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local: int
    backend: str | None


def init(backend: str | None = None, timeout_s: int = 120) -> RankInfo:
    """Reads WORLD_SIZE / RANK / LOCAL_RANK (torchrun); joins a process group
    when the world has more than one rank.  Backend: nccl when CUDA is
    available, else gloo."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world <= 1:
        return RankInfo(1, 0, local, None)
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, **kw)
    return RankInfo(world, rank, local, backend)


def _device(info: RankInfo):
    return torch.device("cuda", info.local) if info.backend == "nccl" else torch.device("cpu")


def barrier(info: RankInfo):
    if info.world > 1:
        dist.barrier()


def max_over_ranks(x: float, info: RankInfo) -> float:
    """The slowest rank's value (timing is reported as the max over ranks)."""
    if info.world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device(info))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finalize(info: RankInfo):
    if info.world > 1 and dist.is_initialized():
        dist.destroy_process_group()


def local_slice(B: int, rank: int, world: int) -> slice:
    """Contiguous share of the batch axis owned by `rank` (sizes differ by at
    most one); empty when there are more ranks than sequences."""
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def weak_scaling_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)
