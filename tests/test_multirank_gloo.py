"""The multi-GPU host logic with two processes on CPU (gloo backend): row and slice sharding, the
max-over-ranks timing, and the sharded-search top-k merge. Every collective the path uses runs here
on CPU tensors; the same calls take CUDA tensors with NCCL in bench.py.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from kv_cache_vector_encode_b200 import shard  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # max over ranks of a per-rank time
        assert shard.max_over_ranks(1.0 + rank) == float(world)

        # row shards: disjoint, in order, covering every row (gathered from all ranks)
        for n in (0, 1, 7, 1000, 1_000_001):
            mine = torch.tensor(shard.shard_rows(n, rank, world), dtype=torch.int64)
            allr = [torch.empty_like(mine) for _ in range(world)]
            dist.all_gather(allr, mine)
            pos = 0
            for r in allr:
                assert int(r[0]) == pos
                pos += int(r[1])
            assert pos == n

        # attention slices: every (b, h) exactly once
        B, Hkv = 3, 5
        mine = torch.tensor([b * Hkv + h for b, h in shard.shard_slices(B, Hkv, rank, world)] + [-1] * (B * Hkv),
                            dtype=torch.int64)[: B * Hkv]
        allr = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(allr, mine)
        got = sorted(int(x) for r in allr for x in r if x >= 0)
        assert got == list(range(B * Hkv))

        # sharded search: local top-k of this rank's rows, then the distributed merge equals the
        # top-k over all rows (scores rounded to make ties across ranks)
        Q, N, k = 5, 301, 10
        g = np.random.default_rng(11)
        scores = np.round(g.standard_normal((Q, N)), 1)
        start, count = shard.shard_rows(N, rank, world)
        loc = scores[:, start:start + count]
        loc_ids = np.tile(np.arange(start, start + count), (Q, 1))
        li, ls = shard.merge_topk(torch.from_numpy(loc_ids), torch.from_numpy(loc), k)
        gi, gs = shard.distributed_topk(li, ls, k)
        wi, ws = shard.merge_topk(torch.from_numpy(np.tile(np.arange(N), (Q, 1))), torch.from_numpy(scores), k)
        assert torch.equal(gi, wi) and torch.equal(gs, ws)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    mp.spawn(_worker, args=(WORLD, _free_port()), nprocs=WORLD, join=True)


def test_merge_topk_rules():
    # descending scores, ties to the lower id, missing entries (-1 / -inf) last
    ids = torch.tensor([[7, 3, 5, -1, 9], [4, -1, -1, -1, -1]])
    sc = torch.tensor([[1.0, 2.0, 2.0, float("-inf"), 0.5], [0.3, float("-inf"), float("-inf"), float("-inf"),
                                                                float("-inf")]], dtype=torch.float64)
    i, s = shard.merge_topk(ids, sc, 3)
    assert i.tolist() == [[3, 5, 7], [4, -1, -1]]
    assert s[0].tolist() == [2.0, 2.0, 1.0] and s[1, 0] == 0.3 and torch.isinf(s[1, 1:]).all()


def test_shard_rows_single_process():
    assert shard.shard_rows(10, 0, 3) == (0, 4)
    assert shard.shard_rows(10, 1, 3) == (4, 3)
    assert shard.shard_rows(10, 2, 3) == (7, 3)
    with pytest.raises(ValueError):
        shard.shard_rows(10, 3, 3)
