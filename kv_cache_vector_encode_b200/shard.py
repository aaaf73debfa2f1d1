"""Multi-GPU plumbing of the hot path: one process per GPU, torch.distributed for the exchanges.

The path partitions without a data-path collective:
  * encode / decode: every rank owns a contiguous range of vector rows (``shard_rows``);
  * decode attention: every rank owns whole (batch, KV head) slices of the cache (``shard_slices``),
    so no softmax state crosses ranks;
  * vector search: every rank scores its own rows of the database, keeps a local top-k, and the
    per-query lists are gathered and merged once (``merge_topk`` / ``distributed_topk``).
Timing is the maximum over ranks of each rank's device time (``max_over_ranks``).

Everything here works with the gloo backend on CPU tensors (the tests run two processes that way)
and with NCCL on CUDA tensors.
"""
from __future__ import annotations


def shard_rows(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous split of n rows over `world` ranks: (first row, row count) of `rank`. The first
    n % world ranks get one row more; every row belongs to exactly one rank."""
    if world <= 0 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def shard_slices(B: int, Hkv: int, rank: int, world: int) -> list[tuple[int, int]]:
    """The (batch, KV head) slices of a decode-attention cache owned by `rank`: a contiguous range
    of the B * Hkv slices in (b, h) order (whole slices, so a rank attends its slices alone)."""
    start, count = shard_rows(B * Hkv, rank, world)
    return [divmod(s, Hkv) for s in range(start, start + count)]


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank scalar (a device time) over the ranks of the default group; the
    value itself when torch.distributed is not initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def merge_topk(ids, scores, k: int):
    """Merge candidate lists per query into the top-k: `ids` and `scores` are [Q, m] (m >= k,
    global ids, -1 / -inf for missing entries). The result is ordered by descending score, ties
    to the lower id (the rule of tq_scores' own top-k); missing entries stay -1 / -inf at the end."""
    import torch
    ids = torch.as_tensor(ids)
    scores = torch.as_tensor(scores)
    Q, m = ids.shape
    out_ids = torch.full((Q, k), -1, dtype=ids.dtype)
    out_sc = torch.full((Q, k), float("-inf"), dtype=scores.dtype)
    for q in range(Q):
        valid = ids[q] >= 0
        cand = sorted(zip(scores[q][valid].tolist(), ids[q][valid].tolist()), key=lambda t: (-t[0], t[1]))
        for j, (s, i) in enumerate(cand[:k]):
            out_ids[q, j] = i
            out_sc[q, j] = s
    return out_ids, out_sc


def distributed_topk(local_ids, local_scores, k: int):
    """Global top-k of a row-sharded search: every rank passes its local top-k ([Q, k], ids already
    global) and every rank returns the merged [Q, k] lists (one all-gather of Q x k ids and scores
    per rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return merge_topk(local_ids, local_scores, k)
    world = dist.get_world_size()
    ids_all = [torch.empty_like(local_ids) for _ in range(world)]
    sc_all = [torch.empty_like(local_scores) for _ in range(world)]
    dist.all_gather(ids_all, local_ids.contiguous())
    dist.all_gather(sc_all, local_scores.contiguous())
    return merge_topk(torch.cat([t.cpu() for t in ids_all], dim=1), torch.cat([t.cpu() for t in sc_all], dim=1), k)
