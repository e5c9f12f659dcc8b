"""The N>1 bench path on CPU: two gloo ranks, each with its own independent
layer seed, agree on the max-over-ranks time and the whole-job rate.  No GPU
and no data-path collective are involved (the path shards without exchange)."""
import os
import socket

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


def _heads_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        h0, h1 = bench.head_range(rank, world, 24)
        pairs = 1000.0 * (h1 - h0)                  # this rank's computed pairs
        total = bench.sum_over_ranks(pairs, world)
        q.put((rank, h0, h1, total))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharding_splits_a_layer_and_sums_its_work():
    """--shard heads: the ranks' head ranges tile the layer's heads exactly,
    and the whole-job work is the sum of the ranks' own work."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_heads_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(o[1], o[2]) for o in out] == [(0, 12), (12, 24)]
    assert all(o[3] == 24000.0 for o in out)


def test_heads_are_independent_in_the_oracle():
    """The reason head sharding needs no exchange: planning and selection of a
    subset of heads equal the same heads of the full layer (the A2V map is per
    token and shared)."""
    import numpy as np
    from oracle import prism_oracle as O
    rng = np.random.default_rng(0)
    T, H, W = 8, 16, 16
    N = T * H * W
    V = rng.normal(size=(N, 4, 8)) * rng.uniform(0.3, 3, size=(N, 4, 1))
    Q, K = rng.normal(size=(N, 4, 8)), rng.normal(size=(N, 4, 8))
    a = np.abs(rng.normal(size=N))
    full = O.plan(V, a, T, H, W)
    part = O.plan(V[:, 2:4], a, T, H, W)
    for k in range(2):
        assert np.array_equal(full.heads[2 + k].perm, part.heads[k].perm)
        assert np.array_equal(full.heads[2 + k].g, part.heads[k].g)
    s_full = O.select(Q, K, full, 0.1, 0, 0.9, heads=[2, 3])
    s_part = O.select(Q[:, 2:4], K[:, 2:4], part, 0.1, 0, 0.9)
    for a_, b_ in zip(s_full, s_part):
        assert all(np.array_equal(x[1], y[1]) for x, y in zip(a_, b_))


def test_head_ranges_tile_the_heads_with_a_remainder():
    """Contiguous, balanced, disjoint ranges covering every head, also when
    the ranks do not divide the heads (the first `heads % world` ranks take
    one more)."""
    import bench
    for heads in (1, 5, 7, 24, 25):
        for world in range(1, min(heads, 8) + 1):
            ranges = [bench.head_range(r, world, heads) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == heads
            assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    assert [bench.head_range(r, 3, 5) for r in range(3)] == [(0, 2), (2, 4), (4, 5)]
