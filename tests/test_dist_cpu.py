"""Host logic of the multi-GPU benchmark on CPU: sharding of sequences and the
max-over-ranks timing, with world_size 2 over gloo."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from hierarchical_tree_indexed_b200 import dist as D


@pytest.mark.parametrize("total,world", [(4, 1), (4, 2), (5, 2), (3, 4), (8, 8)])
def test_shards_cover_every_sequence_once(total, world):
    seen = []
    for r in range(world):
        seen.extend(D.shard(total, D.Rank(r, world, r)))
    assert sorted(seen) == list(range(total))
    sizes = [len(D.shard(total, D.Rank(r, world, r))) for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r = D.Rank(rank, world, rank)
    D.init(r, backend="gloo", timeout_s=60)
    D.barrier(r)
    t = D.max_over_ranks(1.5 + rank, r)
    s = D.sum_over_ranks(float(len(D.shard(4, r))), r)
    q.put((rank, t, s))
    D.finish(r)


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [2.5, 2.5]     # both ranks see the max
    assert [o[2] for o in out] == [4.0, 4.0]     # the shards add up to the whole batch
