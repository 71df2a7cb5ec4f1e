"""Host-side logic for running the recurrence on several GPUs (one process per GPU).

The prefill and decode partition into independent (sequence, head) chains: no chain ever needs
another chain's state, so ranks share no data and the data path has no collective. This module
decides which documents or heads a rank takes, and reduces timings over ranks (the only
collectives: a barrier and max/sum all-reduces of scalars).

Used by bench.py under torchrun and tested with world-size-2 gloo groups on CPU.
"""

from __future__ import annotations

import heapq

import torch


def partition_documents(lengths, world: int) -> list[list[int]]:
    """Assign packed documents to `world` ranks, balancing tokens (longest processing time first).

    Every document goes to exactly one rank; documents are placed longest first on the rank
    with the fewest tokens so far (ties: lowest rank). Returns, per rank, the document indices
    in their original packed order. The result is a pure function of (lengths, world), so every
    rank computes the same partition without communicating.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    heap = [(0, r) for r in range(world)]
    heapq.heapify(heap)
    owned: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        owned[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [sorted(d) for d in owned]


def shard_lengths(lengths, docs) -> list[int]:
    """Lengths of the documents a rank owns, in packed order (its own cu_seqlens follow)."""
    return [int(lengths[i]) for i in docs]


def split_heads(H: int, world: int) -> list[range]:
    """Contiguous head ranges, sizes differing by at most one, covering [0, H)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    base, extra = divmod(H, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append(range(start, start + n))
        start += n
    return out


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, reproducible."""
    return int(base) + 7919 * int(rank)


def _reduce(x: float, op, device) -> float:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, device="cpu") -> float:
    """Maximum of a scalar over all ranks (the job's time is its slowest rank's time)."""
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.MAX if dist.is_available() else None, device)


def sum_over_ranks(x: float, device="cpu") -> float:
    """Sum of a scalar over all ranks (e.g. tokens processed by the whole job)."""
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.SUM if dist.is_available() else None, device)


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
