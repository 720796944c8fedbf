"""CPU checks of the C ABI: the library loads and exports exactly the entry
points include/smc.h declares (no compute call is made without a GPU)."""
import os
import re
import subprocess

import submanifold_sparse_convolution_packed_b200 as smc
from submanifold_sparse_convolution_packed_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    src = open(os.path.join(ROOT, "include", "smc.h")).read()
    return sorted(set(re.findall(r"SMC_API\s+[\w\s\*]+?\b(smc_\w+)\s*\(", src)))


def test_header_declares_binding_exports():
    assert declared() == sorted(smc.EXPORTS)


def test_library_exports_every_declared_symbol():
    B.build()
    lib = smc.lib()
    for name in declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == declared()


def test_strerror_without_gpu():
    lib = smc.lib()
    assert lib.smc_strerror(0) == b"ok"
    assert lib.smc_strerror(-3) == b"duplicate coordinate"
    assert lib.smc_set_hash_capacity(-1) == -1
    assert lib.smc_set_hash_capacity(0) == 0
    assert lib.smc_set_conv_variant(5) == -1
    assert lib.smc_set_conv_variant(4) == 0
    assert lib.smc_set_conv_variant(-1) == -1
    assert lib.smc_set_conv_variant(0) == 0
    assert lib.smc_set_conv_epilogue(2) == -1
    assert lib.smc_set_conv_epilogue(0) == 0
    assert lib.smc_set_conv_priority(2) == -1
    assert lib.smc_set_conv_priority(1) == 0
    assert lib.smc_set_map_lookup(4) == -1
    assert lib.smc_set_map_lookup(3) == 0
    assert lib.smc_set_map_lookup(0) == 0


def test_argument_errors_without_gpu():
    """Validation happens before any device work, so these run on a CPU machine."""
    import ctypes
    lib = smc.lib()
    h = ctypes.c_void_p()
    grid = (ctypes.c_int32 * 3)(4, 4, 4)
    assert lib.smc_build_map(None, 5, 1, grid, None, ctypes.byref(h)) == -1   # null coords
    assert lib.smc_build_map(None, -1, 1, grid, None, ctypes.byref(h)) == -1  # n < 0
    assert lib.smc_build_map(None, 0, 0, grid, None, ctypes.byref(h)) == -1   # batch 0
    assert lib.smc_build_map(ctypes.c_void_p(8), 3, 1, grid, None, ctypes.byref(h)) == -11  # misaligned
    assert h.value is None
    assert lib.smc_conv(None, None, 1, None, None, None, 1, 3, 1, 0, None) == -1
    assert lib.smc_free_map(None) == 0


def test_resample_argument_errors_without_gpu():
    import ctypes
    lib = smc.lib()
    m = ctypes.c_int64(7)
    grid = (ctypes.c_int32 * 3)(4, 4, 4)
    P = ctypes.c_void_p
    a16 = P(16)
    # downsample: no m, bad mode, feats without an output, bad dtype, misaligned coords
    assert lib.smc_downsample(None, 1, 1, grid, None, 0, 0, 0, None, None, None, None, None, None) == -1
    assert lib.smc_downsample(a16, 1, 1, grid, None, 0, 0, 2, a16, None, a16, None, ctypes.byref(m), None) == -1
    assert m.value == 0
    assert lib.smc_downsample(a16, 1, 1, grid, a16, 4, 0, 0, a16, None, a16, None, ctypes.byref(m), None) == -1
    assert lib.smc_downsample(a16, 1, 1, grid, a16, 4, 7, 0, a16, P(4096), a16, None, ctypes.byref(m), None) == -4
    assert lib.smc_downsample(P(8), 1, 1, grid, None, 0, 0, 0, a16, None, a16, None, ctypes.byref(m), None) == -11
    assert lib.smc_downsample(a16, 1, 0, grid, None, 0, 0, 0, a16, None, a16, None, ctypes.byref(m), None) == -1
    assert lib.smc_downsample(None, 0, 1, grid, None, 0, 0, 1, None, None, None, None, ctypes.byref(m), None) == 0
    # pooled output overlapping the input
    assert lib.smc_downsample(a16, 4, 1, grid, P(4096), 8, 0, 0, a16, P(4096 + 64), a16, None,
                              ctypes.byref(m), None) == -6
    # upsample: no m, a map without somewhere to put the child map, bad dtype, misaligned coords
    assert lib.smc_upsample(a16, 1, None, None, 0, 0, None, a16, None, None, None, None) == -1
    assert lib.smc_upsample(a16, 1, None, None, 0, 0, P(64), a16, None, ctypes.byref(m), None, None) == -1
    assert lib.smc_upsample(a16, 1, None, a16, 4, 9, None, a16, P(4096), ctypes.byref(m), None, None) == -4
    assert lib.smc_upsample(P(4), 1, None, None, 0, 0, None, a16, None, ctypes.byref(m), None, None) == -11
    assert lib.smc_upsample(None, 0, None, None, 0, 0, None, None, None, ctypes.byref(m), None, None) == 0


def test_binding_rejects_bad_tensors_without_gpu():
    """The Python binding checks dtypes, shapes and devices before any call
    into the library, so these raise on a CPU machine."""
    import pytest
    import torch
    c = torch.zeros((4, 4), dtype=torch.int32)  # a CPU tensor
    with pytest.raises(ValueError):
        smc.downsample(c, (4, 4, 4))                      # not on a CUDA device
    with pytest.raises(ValueError):
        smc.downsample(c.float(), (4, 4, 4))              # not int32
    with pytest.raises(ValueError):
        smc.downsample(c, (4, 4, 4), mode="median")       # unknown pooling
    with pytest.raises(ValueError):
        smc.upsample(c[:, :3], None)                      # not [N, 4]
    with pytest.raises(ValueError):
        smc.neighbour_map_noalloc(c, (4, 4, 4))           # not on a CUDA device
    assert set(smc.POOL_MODES) == {"max", "mean"}
