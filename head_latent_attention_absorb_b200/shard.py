"""Host-side plumbing of the batch-sharded multi-GPU decode: which sequences a rank owns and the
max-over-ranks reduction of device times.  The attention itself needs no exchange between ranks
(each sequence reads only its own cache rows), so there is no data-path collective."""

from __future__ import annotations

from typing import List, Sequence, Tuple

import torch


def shard_range(global_batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced share [start, start + count) of `global_batch` sequences for `rank`."""
    if world <= 0 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise maximum of `values` over all ranks of the default process group (identity when
    torch.distributed is not initialised)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()
