"""Host-side helpers for running independent decode steps on several GPUs.

The decode step shards with no data-path collective: every (sequence, KV head)
slice is independent (its top-p set, its attention and its output).  With one
process per GPU, each rank owns whole sequences; the only cross-rank traffic is
the timing reduction (max over ranks) and result gathering in tests.
"""
from __future__ import annotations

import os
from typing import List, Tuple

import numpy as np


def dist_env() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return rank, local, world


def shard_sequences(n_seq: int, world: int, rank: int) -> np.ndarray:
    """Contiguous block of sequence indices owned by ``rank`` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} / world {world}")
    base, extra = divmod(n_seq, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return np.arange(start, stop, dtype=np.int64)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's synthetic batch under weak scaling (each rank draws its own batch)."""
    return int(seed) * 1000003 + int(rank)


def reduce_max(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_rows(local: np.ndarray, n_total: int, device=None) -> List[np.ndarray]:
    """all_gather of per-rank row blocks (same trailing shape; blocks may differ in length)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [local]
    world = dist.get_world_size()
    n_max = -(-n_total // world)
    pad = np.zeros((n_max,) + local.shape[1:], dtype=local.dtype)
    pad[:len(local)] = local
    t = torch.from_numpy(pad).to(device) if device is not None else torch.from_numpy(pad)
    bufs = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(bufs, t)
    sizes = [len(shard_sequences(n_total, world, r)) for r in range(world)]
    return [b.cpu().numpy()[:s] for b, s in zip(bufs, sizes)]
