"""Host-side helpers for running the hot path on several GPUs of one node.

The GEMV of one layer is independent per output row, so it partitions by
rows with no exchange on the data path: a rank that owns rows [r0, r1) of W
needs only those rows' records and the (replicated) activations, and writes
y[r0:r1].  ``bench.py`` runs independent layer stacks per GPU (weak
scaling) and combines the ranks' timings with ``max_over_ranks``; tensor
parallel callers use ``row_shard``/``shard_view`` to give each rank its rows
and an all-gather of y if every rank needs the whole output.
"""
from __future__ import annotations


def row_shard(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) owned by `rank`: contiguous, sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    return rows * rank // world, rows * (rank + 1) // world


def shard_view(fmt: dict, rec, eplane, r0: int, r1: int):
    """(fmt, rec, eplane) of rows [r0, r1): same pitches, first row moved."""
    sub = dict(fmt)
    sub["rows"] = r1 - r0
    rec_s = rec[r0:r1]
    ep_s = eplane[r0:r1] if (eplane is not None and fmt["P"] == 4) else eplane
    return sub, rec_s, ep_s


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks of the default process group (or the
    value itself when no group is initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
