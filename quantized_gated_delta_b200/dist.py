"""Multi-GPU plumbing for the decode step: one process per GPU, one pool per GPU.

The (request, head) updates are independent and the step has no exchange, so the GPUs
share nothing on the data path: each rank owns a pool and the requests resident in it
(weak scaling), and collectives appear only around the timing (max over ranks) and, for
callers that want every output on every rank, an optional gather of y.  Works with the
"nccl" backend on GPUs and "gloo" on CPU (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def init_from_env(backend: str | None = None, timeout_s: float = 120.0):
    """Join the process group described by RANK / WORLD_SIZE / MASTER_* (torchrun).

    Returns (rank, world, local_rank).  A single process without those variables runs
    alone (rank 0 of 1) and creates no group."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, world, local


def shard_seed(seed: int, rank: int) -> int:
    """Seed of the requests served by `rank` (each rank serves requests of its own)."""
    return seed + 1000 * rank


def shard_requests(n: int, world: int, rank: int) -> range:
    """Contiguous block of request indices for `rank` when one batch of n requests is split
    across `world` GPUs (sizes differ by at most one)."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def _reduce(value: float, op, device) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device="cpu") -> float:
    """Maximum over ranks (the elapsed time of a step is the slowest rank's)."""
    return _reduce(value, dist.ReduceOp.MAX, device)


def sum_over_ranks(value: float, device="cpu") -> float:
    return _reduce(value, dist.ReduceOp.SUM, device)


def gather_outputs(y_local: torch.Tensor, counts: list[int]) -> torch.Tensor:
    """All ranks' outputs [sum(counts), ...] on every rank, in rank order (outside the hot
    path; ranks may hold different request counts)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return y_local
    world = dist.get_world_size()
    width = max(counts)
    pad = torch.zeros((width,) + tuple(y_local.shape[1:]), dtype=y_local.dtype, device=y_local.device)
    pad[: y_local.shape[0]] = y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def finalize():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
