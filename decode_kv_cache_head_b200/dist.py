"""Multi-GPU plumbing for the compression step: one process per GPU.

Every (sequence, layer, KV head) unit of the step is independent, so ranks
shard sequences and never exchange data on the compute path.  What they share
is bookkeeping: which sequences a rank owns, a distinct input seed per rank
(for synthetic runs), and the step time taken as the maximum over ranks.

The one exchange is the shared selection of tensor-parallel ranks (each rank
holds some KV heads and all ranks must evict the same tokens): the ranks'
eviction scores are summed by an all-reduce between the scoring call and the
select-and-compact call.
"""
from __future__ import annotations

from typing import Tuple

import torch


def world() -> Tuple[int, int]:
    """(world_size, rank), (1, 0) without an initialised process group."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        return torch.distributed.get_world_size(), torch.distributed.get_rank()
    return 1, 0


def shard_range(n: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) share of n sequences for `rank`; the first
    n % world_size ranks take one more."""
    base, extra = divmod(n, world_size)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct sequences on every rank."""
    return base_seed + 1000 * rank


def max_over_ranks(values, device) -> list:
    """Element-wise max of a list of floats across ranks (identity on one rank)."""
    ws, _ = world()
    if ws == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def barrier(device=None) -> None:
    ws, _ = world()
    if ws > 1:
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def head_range(n_kv_heads: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Tensor parallelism: the contiguous KV heads [start, stop) of `rank`."""
    if n_kv_heads % world_size:
        raise ValueError(f"{n_kv_heads} KV heads do not split over {world_size} ranks")
    per = n_kv_heads // world_size
    return rank * per, (rank + 1) * per


def allreduce_eviction_scores(z_sum: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of the ranks' eviction scores, in place (identity on one rank)."""
    ws, _ = world()
    if ws > 1:
        torch.distributed.all_reduce(z_sum, op=torch.distributed.ReduceOp.SUM, group=group)
    return z_sum


def compress_step_shared(rkv, cfg, k_layers, v_layers, q_layers, cur_len, z_sum, workspace,
                         budgets=None, lambdas=None, kept_out=None, group=None, stream=None):
    """The tensor-parallel step: this rank's heads scored, the scores summed over
    the ranks, and one kept set per (layer, sequence) applied to this rank's heads."""
    rkv.rkv_score_shared(cfg, k_layers, q_layers, cur_len, z_sum, workspace, budgets=budgets,
                         lambdas=lambdas, stream=stream)
    allreduce_eviction_scores(z_sum, group)
    return rkv.rkv_select_compact_shared(cfg, k_layers, v_layers, cur_len, z_sum, workspace,
                                         budgets=budgets, kept_out=kept_out, stream=stream)
