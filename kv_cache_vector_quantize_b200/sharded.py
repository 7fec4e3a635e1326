"""Multi-GPU data paths: one process per GPU (torch.distributed, NCCL), the work split over ranks.

The decode path splits with no exchange over (sequence, KV head): quantize, logits and softmax.V
of a head never read another head's cache, so ranks that own disjoint heads just run the library's
calls on their own caches. Two splits need one exchange each, and this module holds their
plumbing; every compute step runs in the library's kernels:

- a KV cache whose *tokens* are split over ranks (a long context): each rank turns its tokens'
  softmax.V into one mergeable partial per query head (``tq_attend_v_partial``: M, L and the
  unrotated weighted sum A, d + 2 floats), the ranks all-gather the partials, and each merges them
  (``tq_attend_merge``: log-sum-exp weights, one Pi^T) into the same output a single GPU would give;
- a nearest-neighbour database whose *rows* are split over ranks: each rank searches its shard
  (``tq_nn_search``), makes the ids global, the ranks all-gather the top-k lists (k score/id pairs
  per query) and each merges them (``tq_nn_merge``, the search's own ordering: score descending,
  then id ascending).

Exchanged bytes: (d + 2) * 4 per query head and rank for softmax.V, 12 k per query and rank for the
search. The collective is an all-gather of a small tensor (NCCL over NVLink on GPUs; gloo works for
CPU tensors). ``merge`` arguments default to the library's kernels.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as B


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of rank's contiguous share of n items (the first n % world ranks get one more)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"shard_range(n={n}, world={world}, rank={rank})")
    q, r = divmod(n, world)
    begin = rank * q + min(rank, r)
    return begin, begin + q + (1 if rank < r else 0)


def gather_parts(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's tensor, in rank order (all ranks get the same)."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def globalize_ids(ids: torch.Tensor, offset: int) -> torch.Tensor:
    """Shard-local database ids -> global ids (empty places, id -1, stay -1)."""
    return torch.where(ids >= 0, ids + offset, ids)


def merge_topk_sharded(local_scores: torch.Tensor, local_ids: torch.Tensor, id_offset: int, group=None,
                       merge=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k of every rank's shard lists ([n_q, k] each, shard-local ids) -> ([n_q, k], [n_q, k])."""
    ids = globalize_ids(local_ids, id_offset)
    ps, pi = gather_parts(local_scores, group), gather_parts(ids, group)
    return (merge or B.tq_nn_merge)(ps, pi)


def nn_search_sharded(db: "B.PackedCache", queries: torch.Tensor, n_db_local: int, id_offset: int,
                      Pi: torch.Tensor, S: torch.Tensor, codebook: torch.Tensor, k: int, group=None,
                      workspace: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k search of the queries over a database split by rows: this rank's shard is ``db``
    (rows [id_offset, id_offset + n_db_local) of the whole); every rank returns the global top-k."""
    s, i = B.tq_nn_search(db, queries, n_db_local, Pi, S, codebook, k, workspace=workspace)
    return merge_topk_sharded(s, i, id_offset, group)


def merge_attend_sharded(local_partial: torch.Tensor, Pi: torch.Tensor, group=None, merge=None) -> torch.Tensor:
    """Every rank's partial [rows, d + 2] -> the merged softmax.V [rows, d]."""
    parts = gather_parts(local_partial, group)            # [world, rows, d + 2]
    return (merge or B.tq_attend_merge)(parts.transpose(0, 1).contiguous(), Pi)


def attend_v_sharded(v: "B.PackedCache", logits: torch.Tensor, scale: float, n_tokens_local: int, Pi: torch.Tensor,
                     codebook: torch.Tensor, group=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """softmax.V over a cache whose tokens are split over ranks: ``v`` and ``logits`` hold this
    rank's tokens. Returns [n_seq, H_q, d] on every rank."""
    part = B.tq_attend_v_partial(v, logits, scale, n_tokens_local, codebook, workspace=workspace)
    out = merge_attend_sharded(part, Pi, group)
    return out.view(v.n_seq, logits.shape[1], v.d)
