"""Query-row sharding of the DSA path over ranks (one process per GPU), and the one collective
the path has.

Every step of the path is per query row t: the indexer scores of row t, its top-k set S_t and
its attention over S_t ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (1)-(2)), so ranks take
disjoint rows and exchange no data on the way.  The sparse-stage indexer loss is a sum over all
rows ("DSA Continued Pre-Training" page, Stage 2; analysis page eq. (4)), so a batch sharded
over ranks needs one sum of the per-rank partial losses.  Host-side plumbing only
(torch.distributed: NCCL between GPUs, gloo in the CPU tests); no arithmetic of the method
lives here.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist


def shard_rows(n_rows: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous rows [start, stop) of rank `rank`; shard sizes differ by at most one."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(n_rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


# Work of one selected latent entry in the attention relative to one indexer key: 128 heads x
# (576 + 512) = 139264 bf16 MACs against 64 x 128 = 8192 FP8 MACs, which run at twice the bf16
# rate ("DeepSeek-V3.2" analysis page, sec. 1.1: the indexer costs about 1/34 of the attention
# per (t, s) pair).
MLA_WEIGHT = 128 * (576 + 512) / (64 * 128 / 2)


def causal_row_cost(Lq: int, Lk: int, k: int, mla_weight: float = 1.0) -> np.ndarray:
    """Relative work of each query row i of a causal sequence (position t = i + Lk - Lq): the
    indexer scores t + 1 keys and the attention reads min(k, t + 1) latents, each weighted by
    mla_weight (MLA_WEIGHT for the full DSA dimensions)."""
    t = np.arange(Lq, dtype=np.float64) + (Lk - Lq)
    return (t + 1.0) + mla_weight * np.minimum(float(k), t + 1.0)


def shard_causal_rows(Lq: int, Lk: int, k: int, rank: int, world: int,
                      mla_weight: float = 1.0) -> tuple[int, int]:
    """Contiguous query rows [start, stop) of one causal sequence for rank `rank`, cut where the
    running work crosses rank/world of the total, so that late (long) rows are not all on the
    last rank.

    How a rank calls the C ABI for its shard: the ABI places query i at t = i + Lk - Lq, so the
    rank passes Lq' = stop - start and Lk' = stop + (Lk - Lq), with q_I, w and q sliced to the
    query rows [start, stop) and k_I and kv truncated to the keys [0, Lk').  Query i of the shard
    then sits at t = start + i + (Lk - Lq), as in the whole sequence.  Passing the full Lk
    instead would shift every position."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    cum = np.concatenate([[0.0], np.cumsum(causal_row_cost(Lq, Lk, k, mla_weight))])

    def cut(r: int) -> int:
        if r <= 0:
            return 0
        if r >= world:
            return Lq
        return int(np.searchsorted(cum, cum[-1] * r / world, side="left"))

    return cut(rank), cut(rank + 1)


def _active() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def sum_over_ranks(x: torch.Tensor) -> torch.Tensor:
    """In-place sum of `x` over all ranks (the sharded indexer loss); a no-op on one rank."""
    if _active():
        dist.all_reduce(x, op=dist.ReduceOp.SUM)
    return x


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The largest `value` over all ranks (a step time is the slowest rank's)."""
    if not _active():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()
