"""The N>1 bench path on CPU: two gloo ranks, each with its own independent
layer seed, agree on the max-over-ranks time and the whole-job rate.  No GPU
and no data-path collective are involved (the path shards without exchange)."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [12.5, 20.0][rank]
        mx = bench.max_over_ranks(ms, world)
        rate = bench.whole_job_rate(1e12, world, mx)
        q.put((rank, bench.rank_seed(rank), mx, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [0, 1]              # independent layers per rank
    assert all(r[2] == 20.0 for r in res)             # max over ranks
    assert all(abs(r[3] - 2 * 1e12 / 0.02) < 1 for r in res)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_rate(10.0, 1, 1000.0) == 10.0
