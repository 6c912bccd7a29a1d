"""Process-group plumbing for running the hot path on several GPUs of one node.

The SP-KV path has no exchange step between batch rows or key heads: they are
independent, so N GPUs serve disjoint batch shards and only the timing is combined
(max over ranks).  The one exchange is that of a sequence split by position across
GPUs (``seqsplit``): every rank's decode partial is all-gathered before the merge.
Backend "nccl" on GPUs, "gloo" for CPU tests.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch


def env() -> Tuple[int, int, int]:
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 600) -> Tuple[int, int, int]:
    """Join the process group described by the torchrun environment (no-op for one
    process).  Returns (world, rank, local_rank)."""
    import torch.distributed as dist
    world, rank, local = env()
    if world > 1 and not dist.is_initialized():
        kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kwargs["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kwargs)
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """Largest value of x over all ranks (the job's elapsed time is its slowest rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous share [start, start+count) of n independent units for this rank."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def all_gather_partials(o_part: torch.Tensor, lse_part: torch.Tensor, o_all: torch.Tensor,
                        lse_all: torch.Tensor) -> None:
    """Every rank's decode partial, in rank order: o_all[r] = rank r's o_part, lse_all[r] =
    rank r's lse_part (fp32; o_all [world][...], lse_all [world][...]).  One collective:
    both are packed into one buffer per rank."""
    import torch.distributed as dist
    world = o_all.shape[0]
    n_o, n_l = o_part.numel(), lse_part.numel()
    send = torch.cat([o_part.reshape(-1), lse_part.reshape(-1)])
    recv = torch.empty((world, n_o + n_l), dtype=send.dtype, device=send.device)
    dist.all_gather_into_tensor(recv.view(-1), send)
    o_all.copy_(recv[:, :n_o].reshape(o_all.shape))
    lse_all.copy_(recv[:, n_o:].reshape(lse_all.shape))


def job_throughput(units_per_rank: float, world: int, elapsed_max_s: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / elapsed_max_s


def finalize(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
