"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each timing its
own replica, must agree on the max-over-ranks time and the whole-job value."""
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


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    r, w, local = bench.dist_env()
    dist = bench.init_dist(w, "gloo", timeout_s=60)
    # each rank "measures" a different time; every rank must see the max
    t = bench.reduce_max(10.0 + rank, w)
    bench.barrier(w)
    q.put((r, w, local, t))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 0, 11.0), (1, 2, 1, 11.0)]


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.algorithmic_map_bytes(10, 100) == 16 * 10 + 108 * 10 + 800
    assert bench.pair_flops(5, 64, 32) == 2 * 5 * 64 * 32
