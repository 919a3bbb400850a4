"""Host-side multi-rank logic of bench.py on CPU: 2 gloo ranks on 127.0.0.1.
The layer's (b,h) sequences are independent, so ranks shard work with no
data-path collective; only the timing uses a max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        got_max = bench.max_over_ranks(10.0 * (rank + 1))
        bench.barrier()
        lo, hi = bench.shard_units(13, rank, world)
        q.put((rank, got_max, lo, hi, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [20.0, 20.0]
    spans = [(r[2], r[3]) for r in res]
    assert spans == [(0, 7), (7, 13)]
    assert res[1][4] == (1, 2, 1)


@pytest.mark.parametrize("n,world", [(1, 4), (96, 8), (7, 3)])
def test_shards_cover_exactly(n, world):
    import bench
    spans = [bench.shard_units(n, r, world) for r in range(world)]
    covered = [i for lo, hi in spans for i in range(lo, hi)]
    assert covered == list(range(n))
