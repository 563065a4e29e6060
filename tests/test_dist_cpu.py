"""The multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each rank takes its share of independent work units (sequences or QK-head groups: the
mixer has no exchange step between them), and the timing reduction takes the maximum over
ranks and the total of processed units."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.dist_env()
        units = list(bench.shard_units(16, r, w))
        t_max = bench.max_over_ranks(1.0 + r)
        total = bench.sum_over_ranks(float(len(units)))
        bench.barrier()
        q.put((r, units, t_max, total))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_rank_shard_and_reduce(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    covered = sorted(u for _, units, _, _ in res for u in units)
    assert covered == list(range(16))
    assert all(t == float(world) for _, _, t, _ in res)
    assert all(tot == 16.0 for _, _, _, tot in res)


def test_shard_units_balanced():
    import bench

    for n in (0, 1, 5, 16, 17, 1000):
        for w in (1, 2, 3, 8):
            shares = [bench.shard_units(n, r, w) for r in range(w)]
            assert sorted(i for s in shares for i in s) == list(range(n))
            sizes = [len(s) for s in shares]
            assert max(sizes) - min(sizes) <= 1
