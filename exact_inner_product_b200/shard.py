"""Exact top-k over a corpus split into row shards, one shard per rank.

Each rank holds rows [start, start + count) of the corpus as its own index,
scores the (replicated) query batch against it with ``tt_score_topk``,
exchanges only its [b, k] list with the other ranks (an all-gather over
``torch.distributed``: NCCL for CUDA tensors, gloo for CPU tensors), and
merges the lists with ``tt_merge_topk``. The merged result equals the
single-corpus result: each member of the global top-k is in its own shard's
top-k, and scores do not depend on where a row sits.

(recsys_two_tower_model.py `forward` shards the corpus over devices on the
`expert` axis; there every device's [B/E, N] scores cross devices in an
all_to_all before `top_k_by_key`. Here only b * k (id, score) pairs per rank
do.)
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import tt_merge_topk, tt_score_topk

ALIGN = 32  # shard starts fall on exclusion-bitmask word boundaries


def shard_bounds(n: int, world: int, align: int = ALIGN) -> list[tuple[int, int]]:
    """(start, count) of every rank's rows: contiguous, disjoint, covering
    [0, n), starts multiples of `align`, counts within `align` of each other
    (the last shard may be shorter or empty when n is small)."""
    if world < 1 or n < 0 or align < 1:
        raise ValueError("need world >= 1, n >= 0, align >= 1")
    blocks = -(-n // align)
    out = []
    for r in range(world):
        b0 = blocks * r // world
        b1 = blocks * (r + 1) // world
        start = min(n, b0 * align)
        stop = min(n, b1 * align)
        out.append((start, stop - start))
    return out


def exclude_slice(exclude: torch.Tensor | None, start: int, count: int) -> torch.Tensor | None:
    """The words of a packed exclusion bitmask that cover rows [start, start + count)
    (start must be a multiple of 32), as a contiguous tensor for the shard."""
    if exclude is None:
        return None
    if start % 32:
        raise ValueError("shard start must be a multiple of 32")
    return exclude[start // 32:(start + count + 31) // 32].contiguous()


def gather_lists(ids: torch.Tensor, scores: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's [b, k] (ids, scores) into [world, b, k] tensors
    (rank r's list at index r)."""
    world = dist.get_world_size(group)
    b, k = ids.shape
    # the output is the ranks' inputs concatenated along dim 0 (the form every
    # backend accepts), viewed as [world, b, k]
    all_ids = torch.empty((world * b, k), dtype=ids.dtype, device=ids.device)
    all_scores = torch.empty((world * b, k), dtype=scores.dtype, device=scores.device)
    dist.all_gather_into_tensor(all_ids, ids.contiguous(), group=group)
    dist.all_gather_into_tensor(all_scores, scores.contiguous(), group=group)
    return all_ids.view(world, b, k), all_scores.view(world, b, k)


def sharded_score_topk(local_index, queries: torch.Tensor, k: int, bounds: list[tuple[int, int]],
                       tau: float = 1.0, exclude_local: torch.Tensor | None = None, group=None,
                       **options) -> tuple[torch.Tensor, torch.Tensor]:
    """Exact top-k of the whole corpus on every rank: local scoring of this
    rank's shard (`local_index`, rows bounds[rank]), all-gather of the lists,
    merge with global ids (start of each shard). Returns (ids, scores) [b, k]."""
    ids, scores = tt_score_topk(local_index, queries, k, tau=tau, exclude=exclude_local, **options)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        all_ids, all_scores = gather_lists(ids, scores, group)
    else:  # a single shard: nothing to exchange
        all_ids, all_scores = ids[None], scores[None]
    return tt_merge_topk(all_ids, all_scores, [start for start, _ in bounds], k)
