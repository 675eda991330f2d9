"""Data-parallel plumbing for row-sharded calibration activations (one process per GPU).

h_j = E_r[x_rj^2] over all ranks' rows: each rank reduces its own rows to column sums
(float64 [K], ``mxq_act_sqsum``), the sums are gathered in rank order (one all-gather of
K doubles per rank; NCCL over NVLink on GPUs, gloo in the CPU tests), and every rank
finishes h with the same fixed-order combine (``mxq_act_sqmean_finalize``), so all ranks
quantize their own weight rows with the identical global h. The quantization itself needs
no communication: blocks are independent.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def shard_rows(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced row range [r0, r1) of ``rank`` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(int(total), world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def gather_in_rank_order(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's ``t``, stacked by rank."""
    world = dist.get_world_size(group)
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t.contiguous(), group=group)
    return torch.stack(out)


def total_rows(local_rows: int, device, group=None) -> int:
    n = torch.tensor([int(local_rows)], dtype=torch.int64, device=device)
    dist.all_reduce(n, group=group)
    return int(n.item())


def distributed_h(X_local: torch.Tensor, colsum_fn: Callable, finalize_fn: Callable,
                  rows_total: int | None = None, group=None) -> torch.Tensor:
    """Global h from this rank's rows: local column sums, rank-ordered gather, finalize.

    ``colsum_fn(X_local) -> float64 [K]`` and ``finalize_fn(parts [world, K], rows_total)
    -> float32 [K]`` are the library's ``mxq_act_sqsum`` and ``mxq_act_sqmean_finalize``
    on GPUs.
    """
    if rows_total is None:
        rows_total = total_rows(X_local.shape[0], X_local.device, group)
    parts = gather_in_rank_order(colsum_fn(X_local), group)
    return finalize_fn(parts, rows_total)
