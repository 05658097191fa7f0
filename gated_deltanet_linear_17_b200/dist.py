"""Multi-GPU plumbing for the forward pass: the operator has no exchange step.

Sequences (and v-head groups) are independent problems, so a multi-GPU run
gives each rank its own units and needs no collective on the data path.  The
only collectives are timing ones (a barrier and a max over ranks).
"""
from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str = "nccl", timeout_s: int = 120):
    """Initialise the default process group from torchrun's environment (no-op for one rank)."""
    rank, local, world = env_rank()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=timeout_s), **kw)
    return rank, local, world


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """Maximum of a per-rank scalar over all ranks (the rank itself for one process)."""
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device="cpu") -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard_sequences(seqlens, world: int, rank: int):
    """Contiguous split of a batch's sequences over ranks, balanced by tokens.

    Returns (first, last) sequence indices (half-open) of ``rank``.  Every
    sequence goes to exactly one rank; sequence order is kept."""
    n = len(seqlens)
    total = sum(seqlens)
    bounds = [0]
    acc = 0
    b = 0
    for r in range(1, world):
        target = total * r / world
        while b < n and acc + seqlens[b] / 2 <= target:
            acc += seqlens[b]
            b += 1
        bounds.append(b)
    bounds.append(n)
    for r in range(1, world + 1):  # keep monotone
        bounds[r] = max(bounds[r], bounds[r - 1])
    return bounds[rank], bounds[rank + 1]


def shard_heads(Nqk: int, Nv: int, world: int, rank: int):
    """Contiguous split of the qk-head groups (with their Nv/Nqk v-heads) over ranks.

    Returns (qk_first, qk_last, v_first, v_last), half-open."""
    G = Nv // Nqk
    per = [Nqk // world + (1 if r < Nqk % world else 0) for r in range(world)]
    a = sum(per[:rank])
    b = a + per[rank]
    return a, b, a * G, b * G
