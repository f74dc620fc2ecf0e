"""Multi-process plumbing for running the path on several GPUs of one node.

The attention path partitions into independent problems (a batch, a layer,
a sequence), so N GPUs run as N ranks that each process their own batch with
no collective on the data path (weak scaling).  The cross-rank steps are a
barrier around the timed region and the maximum of the ranks' device times,
from which the whole-job throughput is computed; and, for data-parallel
training over batch shards, the sum of the ranks' sink gradients
(allreduce_dsinks: attn_sink_bwd sums dsinks over its own batch only).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank():
    """(rank, world, local_rank) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 300.0) -> None:
    """Initialises the default process group from the environment (torchrun sets it)."""
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s own batch: distinct per rank, rank 0 = the single-GPU seed."""
    return base + 7919 * rank


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity for one process)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def allreduce_dsinks(dsinks: torch.Tensor) -> torch.Tensor:
    """Sum the per-rank sink gradients in place (one all-reduce of Hq floats).

    Each rank's attn_sink_bwd returns dsinks summed over that rank's batch
    shard; the sink logits are shared by all ranks, so their gradient is the
    sum over ranks.  Identity for one process."""
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dsinks, op=dist.ReduceOp.SUM)
    return dsinks
