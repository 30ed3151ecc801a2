"""Batch sharding over GPUs, one process per GPU.

The rows of a batch are independent problems: each sequence drafts its own
block, verifies it against its own target rows and emits its own tokens (the
draft-then-verify step of "DeepSeek prezentuje DSpark", section "Jak działa
spekulatywne dekodowanie", applies to one sequence at a time, and nothing in
it reads another sequence).  A job over several GPUs
therefore splits the batch into contiguous blocks of rows, one per rank, and
runs the whole fused cycle on each block with no collective on the data path.
Each rank passes its block's first global row as ``row_offset``, so its random
draws are the ones an unsharded call over the whole batch would make: the
emitted tokens do not depend on how many GPUs the batch was spread over.

The host side needs only three collective steps, none inside a cycle: a barrier
around a timed region, the max over ranks of a measured time, and, when a
caller wants the whole batch's output on one rank, a gather of the row blocks.
They run on whatever process group ``torch.distributed`` holds (NCCL on GPUs,
gloo on CPU).
"""
from __future__ import annotations

import datetime
import os

import torch


def env_rank() -> tuple[int, int, int]:
    """(rank, world size, local rank) as the launcher exported them; a plain
    single-process run is rank 0 of 1."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Join the process group when the launcher started more than one rank.
    A short timeout makes a rank that never arrives end the others' next
    collective with an error instead of a wait without end.  Returns whether a
    group is active."""
    import torch.distributed as dist
    _, world, _ = env_rank()
    if world <= 1:
        return False
    if not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def shard_range(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [start, stop) of rank ``rank`` when ``rows`` rows are split into
    ``world`` contiguous blocks whose sizes differ by at most one (the first
    rows % world blocks take the extra row)."""
    if rows < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split: rows={rows} world={world} rank={rank}")
    q, rem = divmod(rows, world)
    start = rank * q + min(rank, rem)
    return start, start + q + (1 if rank < rem else 0)


def shard_counts(rows: int, world: int) -> list[int]:
    """Rows per rank, in rank order."""
    return [b - a for a, b in (shard_range(rows, world, r) for r in range(world))]


def _device():
    import torch.distributed as dist
    return torch.device("cuda", torch.cuda.current_device()) \
        if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    """The largest value of ``x`` over all ranks (``x`` itself on one rank):
    a multi-GPU time is the slowest rank's."""
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: int) -> int:
    """The sum of ``x`` over all ranks (units processed by the whole job)."""
    import torch.distributed as dist
    if not dist.is_initialized():
        return int(x)
    t = torch.tensor([int(x)], dtype=torch.int64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def gather_rows(block: torch.Tensor, rows: int) -> torch.Tensor | None:
    """Concatenate every rank's block of rows (first dimension) in rank order
    on rank 0; other ranks get None.  Blocks may differ in length by one row
    (``shard_range``): they are padded to the longest for the collective and
    trimmed after it."""
    import torch.distributed as dist
    if not dist.is_initialized():
        return block
    world, rank = dist.get_world_size(), dist.get_rank()
    counts = shard_counts(rows, world)
    if block.shape[0] != counts[rank]:
        raise ValueError(f"rank {rank} holds {block.shape[0]} rows, its share is {counts[rank]}")
    dev = _device()
    most = max(counts)
    pad = torch.zeros((most,) + tuple(block.shape[1:]), dtype=block.dtype, device=dev)
    pad[: block.shape[0]] = block.to(dev)
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad)
    if rank != 0:
        return None
    return torch.cat([b[:c] for b, c in zip(bufs, counts)], dim=0).to(block.device)
