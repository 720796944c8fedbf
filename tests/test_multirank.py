"""Multi-rank host logic on CPU: two gloo ranks of bench.py, each timing its
own replica, must agree on the max-over-ranks time and the whole-job value;
and one item split into z-slabs over gloo ranks, with a halo exchange before
every layer, must give the unsharded result."""
import os
import socket

import numpy as np
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


# ------------------------------------------------------------------ z-slab sharding of one item
def test_slab_bounds_cover_and_balance():
    from submanifold_sparse_convolution_packed_b200.shard import slab_bounds
    counts = np.array([0, 5, 9, 1, 0, 0, 7, 3, 12, 2])
    for world in range(1, 11):
        b = slab_bounds(counts, world)
        assert b[0] == 0 and b[-1] == len(counts) and len(b) == world + 1
        assert all(b[i] < b[i + 1] for i in range(world))  # every slab holds a plane
        per = [int(counts[b[i]:b[i + 1]].sum()) for i in range(world)]
        assert sum(per) == counts.sum()
        if world <= 3:  # balanced to within one plane's count
            assert max(per) - min(per) <= 2 * counts.max()
    with pytest.raises(ValueError):
        slab_bounds(counts, 11)


@pytest.mark.parametrize("world", [2, 3, 5])
def test_slab_plans_agree_between_neighbours(world):
    """Every row is owned by exactly one rank; a rank's halo below is exactly
    the plane its lower neighbour sends up, row for row, and likewise above."""
    from submanifold_sparse_convolution_packed_b200 import synth as S
    from submanifold_sparse_convolution_packed_b200.shard import plan_slabs
    w = S.workload("shell2")
    plans = [plan_slabs(w.coords, w.grid, world, r) for r in range(world)]
    owned = np.sort(np.concatenate([p.owned for p in plans]))
    np.testing.assert_array_equal(owned, np.arange(w.n))
    for r in range(world):
        p = plans[r]
        z = w.coords[p.local_rows, 1]
        lo, hi = p.bounds[r], p.bounds[r + 1]
        assert (z[:p.n_owned] >= lo).all() and (z[:p.n_owned] < hi).all()
        if r > 0:
            below = plans[r - 1]
            np.testing.assert_array_equal(p.halo_lo, below.owned[below.send_hi])
            np.testing.assert_array_equal(p.owned[p.send_lo], below.halo_hi)
            assert (w.coords[p.halo_lo, 1] == lo - 1).all()
        else:
            assert p.halo_lo.size == 0 and p.send_lo.size == 0
        if r == world - 1:
            assert p.halo_hi.size == 0 and p.send_hi.size == 0


def _slab_rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from oracle import oracle
    from submanifold_sparse_convolution_packed_b200 import synth as S
    from submanifold_sparse_convolution_packed_b200.shard import exchange_halos, plan_slabs
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w = S.workload("shell2")
    plan = plan_slabs(w.coords, w.grid, world, rank)
    local_coords = w.coords[plan.local_rows]
    f0, w1, b1 = S.layer_tensors(w, "f32", 0, 3, 8, 6)
    _, w2, b2 = S.layer_tensors(w, "f32", 1, 3, 6, 5)
    x = torch.from_numpy(f0[plan.local_rows].astype(np.float64))
    x[plan.n_owned:] = float("nan")  # halo rows only ever come from the exchange
    for wt, b in ((w1, b1), (w2, b2)):
        exchange_halos(plan, x)
        assert not torch.isnan(x).any()
        y = oracle.conv(local_coords, w.grid, x.numpy(), wt, b, 3, 1)  # the per-rank conv, here the oracle
        x = torch.from_numpy(y)
        x[plan.n_owned:] = float("nan")
    q.put((rank, plan.owned, x[:plan.n_owned].numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_slab_sharded_layers_equal_unsharded(world):
    """Two stacked k=3 layers on the two-item shell workload split into z-slabs
    over gloo ranks, with one halo exchange before each layer, give exactly
    the unsharded result (the per-rank conv is the oracle, in fp64)."""
    from oracle import oracle
    from submanifold_sparse_convolution_packed_b200 import synth as S
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_slab_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = S.workload("shell2")
    f0, w1, b1 = S.layer_tensors(w, "f32", 0, 3, 8, 6)
    _, w2, b2 = S.layer_tensors(w, "f32", 1, 3, 6, 5)
    ref = oracle.conv(w.coords, w.grid, oracle.conv(w.coords, w.grid, f0, w1, b1, 3, 1), w2, b2, 3, 1)
    got = np.full_like(ref, np.nan)
    for _, owned, y in parts:
        got[owned] = y
    np.testing.assert_array_equal(got, ref)
