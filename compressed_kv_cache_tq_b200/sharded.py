"""Vector search over a database sharded by rows across the ranks of a
process group (one process per GPU).

Each rank holds a contiguous block of rows, searches it with ``tq_topk``
(shard-local ids), the per-rank (score, id) lists of every query are
all-gathered over the process group (NCCL on GPUs), and ``tq_topk_merge``
keeps the k best by score descending and global id ascending.  The exchange
is one all-gather of nq x k x (4 + 8) bytes per rank; every computing step
runs in libtq's kernels.
"""

from __future__ import annotations

import torch

from compressed_kv_cache_tq_b200 import tq


def shard_rows(n: int, world: int, rank: int) -> tuple[int, int]:
    """First row and row count of `rank`'s contiguous block of an n-row database."""
    first = n * rank // world
    return first, n * (rank + 1) // world - first


def _world(group) -> int:
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group)
    return 1


def gather_topk(ids: torch.Tensor, scores: torch.Tensor, first_rows, k: int, group=None, merge=None):
    """All-gather every rank's (nq, k) top-k lists (shard-local ids) and merge
    them.  first_rows: the first global row of every rank's shard, in rank
    order.  merge(scores [P, nq, k], ids [P, nq, k], first_rows, k) defaults to
    tq.tq_topk_merge.  Returns (ids (nq, k) global, scores (nq, k))."""
    import torch.distributed as dist

    merge = tq.tq_topk_merge if merge is None else merge
    world = _world(group)
    if len(first_rows) != world:
        raise ValueError("first_rows must hold one entry per rank")
    if world == 1:
        return merge(scores[None], ids[None], first_rows, k)
    nq = scores.shape[0]
    gs = torch.empty((world * nq, k), dtype=scores.dtype, device=scores.device)
    gi = torch.empty((world * nq, k), dtype=ids.dtype, device=ids.device)
    dist.all_gather_into_tensor(gs, scores.contiguous(), group=group)
    dist.all_gather_into_tensor(gi, ids.contiguous(), group=group)
    return merge(gs.view(world, nq, k), gi.view(world, nq, k), first_rows, k)


def sharded_topk(ctx, q: torch.Tensor, payload: torch.Tensor, norms: torch.Tensor, first_rows, k: int, group=None,
                 workspace: torch.Tensor | None = None):
    """Top-k of queries q (nq, d) over the database whose rows this rank holds
    in payload / norms (its shard, rows first_rows[rank] ..); every rank calls
    it with the same queries.  Returns the global (ids, scores) on every rank."""
    ids, scores = tq.tq_topk(ctx, q, payload, norms, k, workspace=workspace)
    return gather_topk(ids, scores, first_rows, k, group)
