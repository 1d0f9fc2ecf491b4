"""Multi-process host logic of shape sharding (gloo, world size 2, CPU):
shapes split without overlap, max/sum reductions of the timing scalars."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from neural_sdf_volume_b200 import shard


def test_shapes_for_rank_partition():
    for n in (1, 4, 7, 16):
        for world in (1, 2, 3, 8):
            parts = [shard.shapes_for_rank(n, r, world) for r in range(world)]
            flat = [s for p in parts for s in p]
            assert flat == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    with pytest.raises(ValueError):
        shard.shapes_for_rank(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = shard.shapes_for_rank(5, rank, world)
        ms = 10.0 + rank            # this rank's step time
        shard.barrier()
        q.put((rank, mine, shard.max_over_ranks(ms), shard.sum_over_ranks(len(mine))))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == [0, 1, 2] and res[1][1] == [3, 4]
    assert res[0][2] == res[1][2] == 11.0      # max over ranks
    assert res[0][3] == res[1][3] == 5.0       # every shape counted once
