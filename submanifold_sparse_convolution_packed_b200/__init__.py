"""B200-native submanifold sparse convolution (SubMConv3d, stride 1).

The computation lives in libsmc.so (hand-written sm_100a CUDA kernels behind
the C ABI of include/smc.h); this package is its thin Python binding plus the
seeded synthetic-workload generators (``synth``).

    from submanifold_sparse_convolution_packed_b200 import build_map, conv
    m = build_map(coords_int32_Nx4_cuda, grid=(Z, Y, X), key="level0")
    out = conv(m, feats, weight_krsc, bias, ksize=3, orientation=+1)
"""
from ._binding import (  # noqa: F401
    EXPORTS, LIB_PATH, Map, SmcError, build_map, clear_cache, conv, kernel_launches, lib,
    NOALLOC_MAX_N, neighbour_map_noalloc, set_conv_variant, set_hash_capacity, set_map_lookup, set_profiling, status, subdivide, group_stats, group_norm,
    downsample, upsample, POOL_MODES, set_conv_epilogue, set_alloc_fail_after, set_wait_limit_ns, set_scan_hold,
    set_schedule_segment, set_conv_priority,
)
