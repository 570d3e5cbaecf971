"""Data-parallel sharding of the TTT layer forward over GPUs.

Every (batch, head) unit is independent, so ranks split the batch: rank r of N
processes the global batch rows [r B, (r + 1) B) of a workload whose per-rank
batch is B (weak scaling).  No collective touches the data; timing is reduced
with a max over ranks.
"""
from __future__ import annotations

from .inputs import TTTConfig


def shard(cfg: TTTConfig, world: int, rank: int) -> tuple[TTTConfig, int]:
    """(per-rank config, global batch offset of this rank's first row)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    return cfg, rank * cfg.B


def global_config(cfg: TTTConfig, world: int) -> TTTConfig:
    """The workload all ranks process together."""
    return cfg.replace(B=cfg.B * world)


def max_over_ranks(values, dist, device=None):
    """Elementwise max of a list of floats over all ranks (identity without a group)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]
