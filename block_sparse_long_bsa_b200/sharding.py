"""Host-side plan for running the forward on several GPUs, one process each.

The work of block-sparse attention splits into independent problems: every
(batch element, head, query block) item reads only its own query rows and the
key/value blocks its layout row keeps ("Block Sparse Attention in LLMs",
section 6: the loop over query blocks and their allowed key blocks has no
dependence between query blocks).  A global batch is therefore sharded by
batch element across ranks with no collective on the data path; the only
collectives are the timing reduction (max over ranks) and barriers around
the timed region.

This module holds no attention arithmetic: it plans shards, derives each
batch element's input seeds, and reduces per-rank timings.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    """The batch elements one rank owns: ``range(start, stop)``."""

    rank: int
    world: int
    start: int
    stop: int

    @property
    def elements(self) -> range:
        return range(self.start, self.stop)

    def __len__(self) -> int:
        return self.stop - self.start


def shard(global_batch: int, world: int, rank: int) -> Shard:
    """Contiguous, balanced split of ``global_batch`` elements over ``world``
    ranks: the first ``global_batch % world`` ranks take one extra element.
    Raises ValueError on a non-positive world, a rank outside it, or a
    negative batch."""
    if world < 1:
        raise ValueError(f"world must be >= 1, got {world}")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if global_batch < 0:
        raise ValueError(f"global_batch must be >= 0, got {global_batch}")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return Shard(rank, world, start, stop)


def element_seeds(element: int) -> tuple[int, int, int]:
    """Seeds of (q, k, v) for batch element ``element``.  Element 0 uses
    (0, 1, 2), the seeds of a single-problem run, so a one-rank run and rank 0
    of a sharded run draw the same inputs."""
    if element < 0:
        raise ValueError(f"element must be >= 0, got {element}")
    return (3 * element, 3 * element + 1, 3 * element + 2)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of ``value`` over all ranks of the default process group
    (identity when ``world == 1``).  ``device`` is where the reduction tensor
    lives: a CUDA device for NCCL, None (CPU) for gloo."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(work_per_rank: list[float] | float, world: int, time_s: float) -> float:
    """Whole-job throughput: the work all ranks did divided by the slowest
    rank's time.  ``work_per_rank`` is one figure per rank, or a single figure
    when every rank did the same work."""
    if time_s <= 0:
        raise ValueError("time must be positive")
    if isinstance(work_per_rank, (int, float)):
        total = float(work_per_rank) * world
    else:
        if len(work_per_rank) != world:
            raise ValueError("one work figure per rank")
        total = float(sum(work_per_rank))
    return total / time_s
