"""Data-parallel plumbing of the LTE hot path.

"Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention and
Contextualized Learnable Token Eviction", Fig. 2 and Fig. 3 captions: LTE
scores, evicts and attends per (sequence, KV head); sequences never exchange
data.  Data parallelism therefore shards whole sequences over ranks (one
process per GPU) and the forward data path has no collective: the host needs
only a barrier around the timed region and a max over ranks of each
device-timed interval, which is how the job's time is defined (the slowest
rank finishes the job).  Training adds one exchange: the gradients of the
scoring CNN's weights, shared by all sequences, are summed over ranks
(all_reduce_sum_).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as tdist


def env_ranks() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, backend: str, device: torch.device | None = None,
         timeout_s: float = 120.0) -> None:
    """Join the process group (no-op for a single rank).  A short timeout makes
    ranks that wait for a rank that died end with an error instead of hanging."""
    if world <= 1:
        return
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    tdist.init_process_group(backend, **kw)


def shutdown(world: int) -> None:
    if world > 1 and tdist.is_initialized():
        tdist.destroy_process_group()


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic sequences: every rank draws its own."""
    return base_seed + 1000 * rank


def barrier(world: int) -> None:
    if world > 1:
        tdist.barrier()


def max_over_ranks(x: float, world: int, device: torch.device | None = None) -> float:
    """Max of a host scalar over all ranks (the job's time for an interval)."""
    if world <= 1:
        return float(x)
    on_gpu = device is not None and device.type == "cuda" and tdist.get_backend() == "nccl"
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if on_gpu else torch.device("cpu"))
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes
    `units_per_rank` and the job takes the slowest rank's `seconds`."""
    return units_per_rank * world / seconds


def all_reduce_sum_(tensors, world: int) -> None:
    """Sum each tensor over all ranks, in place.  Used for the scoring CNN's
    weight gradients, which lte_score_backward sums over a rank's own sequences
    only.  The tensors (one dtype and device) are coalesced into one buffer,
    so the exchange is a single all-reduce (NCCL on GPUs, gloo on the CPU)."""
    if world <= 1 or not tensors:
        return
    flat = torch.cat([t.reshape(-1) for t in tensors])
    tdist.all_reduce(flat, op=tdist.ReduceOp.SUM)
    off = 0
    for t in tensors:
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t))
        off += n
