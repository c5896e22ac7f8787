"""Host logic of the multi-GPU run on CPU: two gloo ranks, each with its own
sequences, the slowest rank's time decides, tokens of all ranks count."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        wl = workloads.make("tiny_4k", seed=bench.layer_seed(rank, 0), seq_len=1024)
        mine = float(wl.q.float().sum())
        ms = 1.0 + rank                       # rank 1 is the slower one
        ms_max = bench.max_over_ranks(ms, world)
        total = bench.shard_summary(wl.batch, world, ms_max, 64)
        sums = [None] * world
        dist.all_gather_object(sums, mine)
        q.put((rank, ms_max, total, sums))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, total, sums in res:
        assert ms_max == 2.0                      # the max over ranks
        assert total == pytest.approx(1 * 2 / (2.0e-3 * 64))
        assert sums[0] != sums[1]                 # each rank has its own data
