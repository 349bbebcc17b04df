"""Host-side helpers for running LiteLA on several GPUs of one node.

The forward pass shards without any data exchange: calls (layers), batches and heads are
independent units, so each rank runs its own share and the only cross-rank step is the
max-over-ranks of the measured time in the benchmark.  These helpers hold that host logic so
that it can be tested with the gloo backend on CPU.
"""
from __future__ import annotations

import os

__all__ = ["world_info", "rank_seeds", "shard_heads", "pack_head_shard", "max_over_ranks", "aggregate_rate"]


def world_info():
    """(world_size, rank, local_rank) from the torch.distributed.run environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seeds(base_seeds, rank: int, stride: int = 100000):
    """Seeds of a rank's own inputs for weak scaling: every rank gets a distinct, reproducible
    copy of the per-GPU workload (rank 0 keeps the single-GPU seeds)."""
    return [int(s) + stride * int(rank) for s in base_seeds]


def shard_heads(H: int, world: int, rank: int):
    """Contiguous head range [h0, h1) of a rank when one problem's heads are split over ranks
    (heads are independent; ranges differ in size by at most one head)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d out of range for world %d" % (rank, world))
    h0 = H * rank // world
    h1 = H * (rank + 1) // world
    return h0, h1


def pack_head_shard(qkv, H: int, h0: int, h1: int, d: int = 32):
    """The packed qkv [B, N, 3*(h1-h0)*d] of heads [h0, h1) of a packed qkv [B, N, 3*H*d] (q, k
    and v of those heads, each head-major): the input a rank gets when a tensor-parallel qkv
    projection produces only its own heads.  Data movement only (a strided copy)."""
    B, N = qkv.shape[0], qkv.shape[1]
    if not 0 <= h0 < h1 <= H or qkv.shape[2] != 3 * H * d:
        raise ValueError("bad head range or qkv shape")
    return qkv.view(B, N, 3, H, d)[:, :, :, h0:h1].reshape(B, N, 3 * (h1 - h0) * d).contiguous()


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without an initialised group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed divided by the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / (max_ms / 1e3)
