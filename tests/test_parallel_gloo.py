"""The multi-GPU plumbing on CPU: world_size-2 gloo ranks check that the batch
shards cover every volume exactly once and that the step time reported is the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dimensional_long_convolution_b200.parallel import max_over_ranks, shard_range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, total, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        lo, hi = shard_range(total, rank, world)
        mine = torch.zeros(total, dtype=torch.int64)
        mine[lo:hi] = 1
        dist.all_reduce(mine)
        t = max_over_ranks(1.0 + rank * 0.5, dist)
        q.put((rank, mine.tolist(), t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("total", [7, 256])
def test_two_rank_shards_cover_batch_and_time_is_max(total):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, total, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, cover, t in out:
        assert cover == [1] * total
        assert t == 1.5


def test_shard_range_edges():
    assert shard_range(5, 0, 2) == (0, 3) and shard_range(5, 1, 2) == (3, 5)
    assert shard_range(0, 0, 3) == (0, 0)
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)
