"""Head partition of one PBSA layer across ranks (one process per GPU).

Sparse Forcing's persistent memory, the local selections and the fine attention are all
per (layer, head): a head's persistent set, EMA scores and selections depend on that
head's queries and keys only (gist.science English explainer, 2.B "Structured Memory
Decomposition" and 2.C "Persistent Block-Sparse Attention"; the per-head reading of the
method).  So a layer shards over G GPUs by heads with no exchange inside the step: rank g
owns the heads ``head_range(H, G, g)``, holds their pools and slot tables (a
``PBSALayerCache`` built with ``local_config``) and takes their Q, K, V slices.  The only
collective is the one the surrounding model already performs on the attention output
(an all-gather of O over heads, or the out-projection's reduction under head-sharded
tensor parallelism); it is not part of this path.

This module is host logic only: ranges and slices.  Every number of the path is still
computed by the library's kernels on each rank.
"""
from __future__ import annotations

import dataclasses

import torch


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of ``rank``: contiguous, sizes differing by at most one, lower ranks
    taking the larger shares (12 heads over 8 ranks: 2, 2, 2, 2, 1, 1, 1, 1)."""
    if not (world > 0 and 0 <= rank < world and heads > 0):
        raise ValueError(f"bad partition: heads={heads} world={world} rank={rank}")
    if world > heads:
        raise ValueError(f"{world} ranks cannot each own one of {heads} heads")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def local_config(cfg, world: int, rank: int):
    """The ``LayerConfig`` of rank ``rank``'s heads (every other field unchanged)."""
    h0, h1 = head_range(cfg.heads, world, rank)
    return dataclasses.replace(cfg, heads=h1 - h0)


def head_slice(x: torch.Tensor, heads: int, world: int, rank: int) -> torch.Tensor:
    """Rank ``rank``'s heads of a raster token tensor ``[T, H, d]``, contiguous (in a
    head-sharded model each rank's projections produce this slice directly)."""
    if x.dim() != 3 or x.shape[1] != heads:
        raise ValueError(f"expected [T, {heads}, d], got {tuple(x.shape)}")
    h0, h1 = head_range(heads, world, rank)
    return x[:, h0:h1].contiguous()
