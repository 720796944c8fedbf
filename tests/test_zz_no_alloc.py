"""The neighbour map computed without device allocation.

smc_neighbour_map_noalloc serves callers that may not allocate device memory
while they run (a fixed device-memory budget reserved up front, or a host
framework that owns the allocator): its scratch is a fixed static device
array.  Here it is called through the C ABI into a preallocated buffer and its
output must equal the map of the ordinary entry point, on two calls in a row
with different coordinate sets (the shared scratch keeps the previous call's
contents, so a stale table would show up on the second call).

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import submanifold_sparse_convolution_packed_b200 as smc
from submanifold_sparse_convolution_packed_b200 import synth as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    smc.lib()


def _noalloc_via_cabi(coords_np, grid, batch):
    coords = torch.from_numpy(coords_np).cuda()
    out = torch.full((coords.shape[0], 27), -7, dtype=torch.int32, device="cuda")
    g = (ctypes.c_int32 * 3)(*grid)
    stream = torch.cuda.current_stream()
    rc = smc.lib().smc_neighbour_map_noalloc(ctypes.c_void_p(coords.data_ptr()), coords.shape[0], batch, g,
                                             ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, smc.lib().smc_strerror(rc)
    return out.cpu().numpy()


def _reference(coords_np, grid, batch):
    m = smc.build_map(torch.from_numpy(coords_np).cuda(), grid, batch=batch)
    nbr = m.nbr().cpu().numpy()
    m.free()
    return nbr


def test_noalloc_matches_build_map_twice():
    cases = [S.workload("shell2"), S.workload("tiny")]
    for w in cases:  # two calls in a row on the shared scratch
        batch = int(w.coords[:, 0].max()) + 1
        got = _noalloc_via_cabi(w.coords, list(w.grid), batch)
        np.testing.assert_array_equal(got, _reference(w.coords, w.grid, batch))
    # and the first case again, after the smaller one
    w = cases[0]
    batch = int(w.coords[:, 0].max()) + 1
    np.testing.assert_array_equal(_noalloc_via_cabi(w.coords, list(w.grid), batch),
                                  _reference(w.coords, w.grid, batch))


def test_noalloc_matches_oracle(oracle_mod):
    """Bit for bit against the CPU oracle's neighbour map, not only against
    the other GPU entry point."""
    for name in ("tiny", "shell2"):
        w = S.workload(name)
        batch = int(w.coords[:, 0].max()) + 1
        got = _noalloc_via_cabi(w.coords, list(w.grid), batch)
        np.testing.assert_array_equal(got, oracle_mod.neighbour_map(w.coords, w.grid))


def test_noalloc_out_of_range_row():
    """A coordinate outside the box is reported as SMC_E_RANGE and its row of
    the map is left all -1 (it is never a neighbour of anything)."""
    w = S.workload("tiny")
    coords = w.coords.copy()
    bad = 7
    coords[bad, 3] = w.grid[2]  # x one past the last plane
    c = torch.from_numpy(coords).cuda()
    out = torch.full((coords.shape[0], 27), -7, dtype=torch.int32, device="cuda")
    g = (ctypes.c_int32 * 3)(*w.grid)
    rc = smc.lib().smc_neighbour_map_noalloc(ctypes.c_void_p(c.data_ptr()), coords.shape[0], 1, g,
                                             ctypes.c_void_p(out.data_ptr()), None)
    assert rc == -2  # SMC_E_RANGE
    got = out.cpu().numpy()
    assert (got[bad] == -1).all()
    assert not (got == bad).any()
    assert ((got >= -1) & (got < coords.shape[0])).all()


def test_noalloc_limits_and_errors():
    lib = smc.lib()
    g = (ctypes.c_int32 * 3)(8, 8, 8)
    buf = torch.zeros((16, 27), dtype=torch.int32, device="cuda")
    c = torch.zeros((16, 4), dtype=torch.int32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    # above the fixed scratch size: rejected before any device work
    assert lib.smc_neighbour_map_noalloc(p(c), smc.NOALLOC_MAX_N + 1, 1, g, p(buf), None) == -5
    # duplicate coordinates are reported like smc_build_map does
    dup = torch.tensor([[0, 1, 1, 1], [0, 1, 1, 1]], dtype=torch.int32, device="cuda")
    out = torch.zeros((2, 27), dtype=torch.int32, device="cuda")
    assert lib.smc_neighbour_map_noalloc(p(dup), 2, 1, g, p(out), None) == -3
    # the binding wrapper
    w = S.workload("tiny")
    got = smc.neighbour_map_noalloc(torch.from_numpy(w.coords).cuda(), w.grid, batch=1)
    np.testing.assert_array_equal(got.cpu().numpy(), _reference(w.coords, w.grid, 1))
