"""Host logic of the multi-GPU run on CPU: two gloo ranks, each with its own
sequences, the slowest rank's time decides, tokens of all ranks count; and
the data-parallel split itself: ranks that each run the fp64 oracle on their
share of a seeded batch reproduce the unsharded run bit for bit."""
import os
import socket

import numpy as np
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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        from harness import oracle_args, run_oracle
        wl = workloads.make("ragged_hybrid", seed=4, batch=5, ragged_range=(640, 4096))
        mine = bench.rank_sequences(wl.batch, world, rank)
        sub = workloads.gather_units(wl, mine)
        res = run_oracle(sub, "mxfp4", args=oracle_args(sub, "mxfp4"))
        parts = [None] * world
        dist.all_gather_object(parts, (mine, {k: res[k] for k in
                                              ("sel_idx", "sel_cnt", "out", "lse")}))
        q.put((rank, parts))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_batch_like_unsharded_oracle():
    import bench
    import workloads
    from harness import oracle_args, run_oracle
    assert bench.rank_sequences(5, 2, 0) == [0, 1, 2] and bench.rank_sequences(5, 2, 1) == [3, 4]
    assert bench.rank_sequences(1, 2, 1) == []
    wl = workloads.make("ragged_hybrid", seed=4, batch=5, ragged_range=(640, 4096))
    full = run_oracle(wl, "mxfp4", args=oracle_args(wl, "mxfp4"))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, parts in res:
        seen = []
        for seqs, r in parts:
            seen += seqs
            for i, b in enumerate(seqs):
                n = int(r["sel_cnt"][i].max()) if r["sel_cnt"].size else 0
                assert np.array_equal(r["sel_cnt"][i], full["sel_cnt"][b])
                for g in range(wl.num_kv_heads):
                    c = int(full["sel_cnt"][b, g])
                    assert np.array_equal(r["sel_idx"][i, g, :c], full["sel_idx"][b, g, :c])
                assert n <= wl.max_blocks
                assert np.array_equal(r["out"][i], full["out"][b])
                assert np.array_equal(r["lse"][i], full["lse"][b])
        assert seen == list(range(wl.batch))
