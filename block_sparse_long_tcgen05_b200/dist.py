"""Multi-GPU plumbing for running the MSA hot path data-parallel.

The path shards without any exchange, two ways: each rank owns whole independent sequences
(prefill) or whole sequences of a decode batch; or every rank works on the same sequence
and owns a contiguous range of GQA groups with their query heads (groups never interact:
each has its own index head and its own block selection, zhichai.net section 2). Either
way the data path has no collective. The only cross-rank traffic is timing: a barrier
around timed regions and the max of the per-rank times (a job is as fast as its slowest
rank). One process per GPU; torchrun sets RANK, LOCAL_RANK and WORLD_SIZE.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_ranks() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300) -> tuple[int, int, int]:
    """Join the process group when launched with more than one rank."""
    world, rank, local = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s independent sequence (distinct per rank, stable across runs)."""
    return seed + 7 * rank


def shard(n_units: int, world: int, rank: int) -> range:
    """Contiguous share of n_units whole units (sequences) for `rank`; sizes differ by <= 1."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def group_slice(G: int, R: int, world: int, rank: int) -> tuple[range, slice, slice]:
    """Group sharding of one sequence: (groups, query-head slice, group slice) of `rank`.
    Query head h belongs to group h // R, so a contiguous range of groups owns a contiguous
    range of heads; requires world <= G."""
    if world > G:
        raise ValueError(f"{world} ranks for {G} groups")
    groups = shard(G, world, rank)
    return groups, slice(groups.start * R, groups.stop * R), slice(groups.start, groups.stop)


def shard_inputs_by_group(inp: dict, G: int, world: int, rank: int) -> dict:
    """This rank's contiguous copies of a prefill input dict (q [N,Hq,d]; k, v, q_idx,
    k_idx [N,G,*]) for its groups."""
    R = inp["q"].shape[1] // G
    _, hs, gs = group_slice(G, R, world, rank)
    return {n: (t[:, hs] if n == "q" else t[:, gs]).contiguous() for n, t in inp.items()}


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. the timed milliseconds) across all ranks."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def job_throughput(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
