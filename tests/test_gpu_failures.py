"""Failure paths on the GPU, with every failure made on the host.

* Allocation failure: the library's test hook makes its k-th pool allocation
  report failure.  Every allocating entry point must return SMC_E_OOM, leave
  its handle output NULL, release what it had allocated (device memory stays
  flat over many failed calls) and leave the library usable.
* A device-side wait that runs out: a test hook makes one segment of every
  look-back scan publish nothing, with the wait bound cut to a few
  milliseconds, so the later segments give up.  The call must report
  SMC_E_TIMEOUT, every map entry must still be -1 or a valid row, and the next
  build (hooks off) must be exact again.

Nothing here faults, traps or hangs a GPU: the held scan waits are bounded
and no conv kernel with loads in flight is made to time out.
"""
import ctypes

import numpy as np
import pytest
import torch

import submanifold_sparse_convolution_packed_b200 as smc
from submanifold_sparse_convolution_packed_b200 import synth as S

pytestmark = pytest.mark.gpu

SMC_E_OOM, SMC_E_TIMEOUT = -8, -10


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    smc.lib()
    yield
    smc.set_alloc_fail_after(0)
    smc.set_scan_hold(-1)
    smc.set_wait_limit_ns(0)


@pytest.fixture(autouse=True)
def _hooks_off():
    yield
    smc.set_alloc_fail_after(0)
    smc.set_scan_hold(-1)
    smc.set_wait_limit_ns(0)


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _shell2():
    w = S.workload("shell2")
    return w, torch.from_numpy(w.coords).cuda()


def test_build_allocation_failure(oracle_mod):
    w, coords = _shell2()
    lib = smc.lib()
    g = (ctypes.c_int32 * 3)(*w.grid)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    smc.build_map(coords, w.grid, batch=2).free()  # the pool now holds a build's buffers
    free0 = _free_bytes()
    for k in (1, 2):  # the map's own buffers, then the build's scratch
        for fn in (lib.smc_build_map, lib.smc_build_map_async):
            for _ in range(10):
                smc.set_alloc_fail_after(k)
                h = ctypes.c_void_p(0x1234)
                rc = fn(_p(coords), w.n, 2, g, stream, ctypes.byref(h))
                assert rc == SMC_E_OOM, (k, rc)
                assert h.value is None
    smc.set_alloc_fail_after(0)
    assert _free_bytes() >= free0 - (32 << 20)
    m = smc.build_map(coords, w.grid, batch=2)
    np.testing.assert_array_equal(m.nbr().cpu().numpy(), oracle_mod.neighbour_map(w.coords, w.grid))
    m.free()


def test_subdivide_allocation_failure(oracle_mod):
    w = S.workload("tiny")
    coords = torch.from_numpy(w.coords).cuda()
    parent = smc.build_map(coords, w.grid, batch=1)
    for k in (1, 2, 3):  # the children's scratch, then the child map's two allocations
        smc.set_alloc_fail_after(k)
        with pytest.raises(smc.SmcError) as e:
            smc.subdivide(parent, coords)
        assert e.value.code == SMC_E_OOM
    smc.set_alloc_fail_after(0)
    child_coords, child = smc.subdivide(parent, coords)
    ref = oracle_mod.subdivide(w.coords)
    np.testing.assert_array_equal(child_coords.cpu().numpy(), ref)
    grid2 = [2 * g for g in w.grid]
    np.testing.assert_array_equal(child.nbr().cpu().numpy(), oracle_mod.neighbour_map(ref, grid2))
    child.free()
    parent.free()


def test_resample_allocation_failure():
    w, coords = _shell2()
    feats = torch.randn(w.n, 64, device="cuda").bfloat16()
    smc.set_alloc_fail_after(1)
    with pytest.raises(smc.SmcError) as e:
        smc.downsample(coords, w.grid, feats, mode="max", batch=2)
    assert e.value.code == SMC_E_OOM
    pc, pooled, mask, _ = smc.downsample(coords, w.grid, feats, mode="max", batch=2)
    smc.set_alloc_fail_after(1)
    with pytest.raises(smc.SmcError) as e:
        smc.upsample(pc, mask, pooled)
    assert e.value.code == SMC_E_OOM
    cc, cf, _ = smc.upsample(pc, mask, pooled)
    assert cc.shape[0] == w.n


def test_per_offset_conv_and_stats_allocation_failure():
    w, coords = _shell2()
    m = smc.build_map(coords, w.grid, batch=2)
    x = torch.randn(w.n, 64, device="cuda").bfloat16()
    wt = (torch.randn(64, 3, 3, 3, 64, device="cuda") * 0.02).bfloat16()
    ref = smc.conv(m, x, wt)
    smc.set_conv_variant(3)
    try:
        smc.set_alloc_fail_after(1)  # the per-offset kernel's fp32 accumulator
        with pytest.raises(smc.SmcError) as e:
            smc.conv(m, x, wt)
        assert e.value.code == SMC_E_OOM
        got = smc.conv(m, x, wt)
    finally:
        smc.set_conv_variant(0)
    assert float((got.float() - ref.float()).abs().max()) <= 5e-3 * float(ref.float().abs().max())
    stats = torch.zeros((2, 32, 3), dtype=torch.float64, device="cuda")
    smc.set_alloc_fail_after(1)  # the striped statistics copies
    with pytest.raises(smc.SmcError) as e:
        smc.group_stats(ref, coords, 2, 32, stats=stats)
    assert e.value.code == SMC_E_OOM
    m.free()


def test_scan_wait_runs_out(oracle_mod):
    # a map large enough for several scan segments in each of its scans
    w = S.workload("decoder2")
    coords = torch.from_numpy(w.coords).cuda()
    ref_nbr = oracle_mod.neighbour_map(w.coords, w.grid)
    smc.set_wait_limit_ns(2_000_000)  # 2 ms
    smc.set_scan_hold(1)
    m = smc.build_map(coords, w.grid, batch=1, sync=False)
    with pytest.raises(smc.SmcError) as e:
        m.wait()
    assert e.value.code == SMC_E_TIMEOUT
    # the lookups ran before any scan: the map itself is whole and in bounds
    np.testing.assert_array_equal(m.nbr().cpu().numpy(), ref_nbr)
    # a conv on the failed map is refused
    x = torch.zeros((w.n, 64), dtype=torch.bfloat16, device="cuda")
    wt = torch.zeros((64, 3, 3, 3, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(smc.SmcError) as e:
        smc.conv(m, x, wt)
    assert e.value.code == SMC_E_TIMEOUT
    m.free()
    # the downsample's scan of its flags runs out the same way
    ws, cs = _shell2()
    feats = torch.randn(ws.n, 64, device="cuda").bfloat16()
    with pytest.raises(smc.SmcError) as e:
        smc.downsample(cs, ws.grid, feats, mode="mean", batch=2)
    assert e.value.code == SMC_E_TIMEOUT
    # hooks off: the device is usable and the next build is exact
    smc.set_scan_hold(-1)
    smc.set_wait_limit_ns(0)
    m = smc.build_map(coords, w.grid, batch=1)
    np.testing.assert_array_equal(m.nbr().cpu().numpy(), ref_nbr)
    _, _, in_idx, out_idx = oracle_mod.pair_lists(ref_nbr)
    got_in, got_out, _ = m.pairs()
    np.testing.assert_array_equal(got_in.cpu().numpy(), in_idx)
    np.testing.assert_array_equal(got_out.cpu().numpy(), out_idx)
    smc.status()
    m.free()


def test_hook_arguments():
    lib = smc.lib()
    assert lib.smc_set_alloc_fail_after(-1) == -1
    assert lib.smc_set_wait_limit_ns(-5) == -1
    assert lib.smc_set_scan_hold(-2) == -1
