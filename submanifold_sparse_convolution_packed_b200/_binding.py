"""ctypes binding of libsmc.so (include/smc.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
checks tensor dtypes and shapes, passes raw device pointers and the current
CUDA stream, and turns negative return codes into ``SmcError``.  If the
library has not been built, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Hashable, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmc.so")

SMC_F32, SMC_BF16, SMC_F16 = 0, 1, 2
_DTYPES = {torch.float32: SMC_F32, torch.bfloat16: SMC_BF16, torch.float16: SMC_F16}

ERROR_NAMES = {
    -1: "SMC_E_ARG", -2: "SMC_E_RANGE", -3: "SMC_E_DUPLICATE", -4: "SMC_E_DTYPE",
    -5: "SMC_E_SHAPE", -6: "SMC_E_ALIAS", -7: "SMC_E_CAPACITY", -8: "SMC_E_OOM",
    -9: "SMC_E_CUDA", -10: "SMC_E_TIMEOUT", -11: "SMC_E_ALIGN",
}

EXPORTS = [
    "smc_build_map", "smc_conv", "smc_map_info", "smc_map_nbr", "smc_map_pairs",
    "smc_map_schedule", "smc_free_map", "smc_status", "smc_strerror",
    "smc_set_hash_capacity", "smc_set_profiling", "smc_map_timing", "smc_kernel_launches",
    "smc_build_map_async", "smc_map_wait", "smc_neighbour_map_noalloc", "smc_set_conv_variant",
    "smc_set_map_lookup", "smc_map_stream_wait", "smc_subdivide", "smc_conv_ex", "smc_group_stats",
    "smc_group_norm", "smc_downsample", "smc_upsample", "smc_set_conv_epilogue",
    "smc_set_alloc_fail_after", "smc_set_wait_limit_ns", "smc_set_scan_hold", "smc_set_schedule_segment",
    "smc_set_conv_priority",
]


class SmcError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        msg = lib().smc_strerror(code).decode() if _lib is not None else "error"
        super().__init__(f"{what}: {ERROR_NAMES.get(code, code)} ({msg})")
        self.code = code
        self.name = ERROR_NAMES.get(code, str(code))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libsmc.so.  Raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m submanifold_sparse_convolution_packed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.smc_build_map.argtypes = [P, i64, i32, P, P, ctypes.POINTER(P)]
        L.smc_build_map_async.argtypes = [P, i64, i32, P, P, ctypes.POINTER(P)]
        L.smc_map_wait.argtypes = [P]
        L.smc_map_stream_wait.argtypes = [P, P]
        L.smc_subdivide.argtypes = [P, P, P, P, P, P, P]
        L.smc_downsample.argtypes = [P, i64, i32, P, P, i64, i32, i32, P, P, P, P, P, P]
        L.smc_upsample.argtypes = [P, i64, P, P, i64, i32, P, P, P, P, P, P]
        L.smc_conv_ex.argtypes = [P, P, i64, P, P, P, P, i64, i32, i32, i32, i32, P, P, i32, P]
        L.smc_group_stats.argtypes = [P, i64, i64, P, i32, i32, P, i32, P]
        L.smc_group_norm.argtypes = [P, i64, i64, P, i32, i32, P, P, P, ctypes.c_float, i32, P, i32, P]
        L.smc_neighbour_map_noalloc.argtypes = [P, i64, i32, P, P, P]
        L.smc_conv.argtypes = [P, P, i64, P, P, P, i64, i32, i32, i32, P]
        L.smc_map_info.argtypes = [P, P, P]
        L.smc_map_nbr.argtypes = [P, ctypes.POINTER(P)]
        L.smc_map_pairs.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(P), P]
        L.smc_map_schedule.argtypes = [P, ctypes.POINTER(P)]
        L.smc_free_map.argtypes = [P]
        L.smc_status.argtypes = [P]
        L.smc_strerror.argtypes = [ctypes.c_int]
        L.smc_strerror.restype = ctypes.c_char_p
        L.smc_set_hash_capacity.argtypes = [i64]
        L.smc_set_profiling.argtypes = [i32]
        L.smc_map_timing.argtypes = [P, P]
        L.smc_kernel_launches.argtypes = [P]
        L.smc_set_conv_variant.argtypes = [i32]
        L.smc_set_conv_epilogue.argtypes = [i32]
        L.smc_set_map_lookup.argtypes = [i32]
        L.smc_set_alloc_fail_after.argtypes = [i64]
        L.smc_set_wait_limit_ns.argtypes = [i64]
        L.smc_set_scan_hold.argtypes = [i64]
        L.smc_set_schedule_segment.argtypes = [i64]
        L.smc_set_conv_priority.argtypes = [i32]
        for name in EXPORTS:
            if name != "smc_strerror":
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(code: int, what: str) -> None:
    if code != 0:
        raise SmcError(code, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[ctypes.c_void_p]:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class _DeviceView:
    """__cuda_array_interface__ over library-owned memory (kept alive by `owner`)."""

    def __init__(self, ptr: int, shape, typestr: str, owner):
        self.owner = owner
        self.__cuda_array_interface__ = {
            "shape": tuple(shape), "typestr": typestr, "data": (ptr, False), "version": 3,
            "strides": None, "stream": None,
        }


class Map:
    """A built neighbour map (library-owned device buffers)."""

    def __init__(self, handle: ctypes.c_void_p, n: int, batch: int, grid: Sequence[int], device):
        self._h = handle
        self.n = n
        self.batch = batch
        self.grid = tuple(int(g) for g in grid)
        self.device = device
        self._counts = None
        self._offsets = None

    def wait(self) -> "Map":
        """Block until the build has finished; raise SmcError if it failed."""
        _check(lib().smc_map_wait(self.handle), "smc_build_map")
        return self

    def stream_wait(self, stream=None) -> "Map":
        """Make `stream` wait on the device for the whole build, pair lists
        included (no host synchronisation)."""
        _check(lib().smc_map_stream_wait(self.handle, _stream(stream)), "smc_map_stream_wait")
        return self

    @property
    def counts(self):
        if self._counts is None:
            c = (ctypes.c_int64 * 27)()
            _check(lib().smc_map_info(self.handle, None, c), "smc_map_info")
            self._counts = [int(x) for x in c]
        return self._counts

    @property
    def offsets(self):
        if self._offsets is None:
            o = (ctypes.c_int64 * 28)()
            _check(lib().smc_map_pairs(self.handle, None, None, o), "smc_map_pairs")
            self._offsets = [int(x) for x in o]
        return self._offsets

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise RuntimeError("map already freed")
        return self._h

    @property
    def pairs_total(self) -> int:
        return self.offsets[-1]

    def _view(self, ptr: int, shape, typestr="<i4") -> torch.Tensor:
        if self.n == 0 or ptr is None:
            return torch.empty(shape, dtype=torch.int32, device=self.device)
        return torch.as_tensor(_DeviceView(ptr, shape, typestr, self), device=self.device)

    def nbr(self) -> torch.Tensor:
        """int32 [n, 27] device view of the neighbour map (-1 = absent)."""
        p = ctypes.c_void_p()
        _check(lib().smc_map_nbr(self.handle, ctypes.byref(p)), "smc_map_nbr")
        return self._view(p.value, (self.n, 27))

    def pairs(self):
        """(in_idx, out_idx, offsets): int32 [P] device views and the 28 offsets."""
        pi, po = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().smc_map_pairs(self.handle, ctypes.byref(pi), ctypes.byref(po), None), "smc_map_pairs")
        P = self.pairs_total
        return self._view(pi.value, (P,)), self._view(po.value, (P,)), list(self.offsets)

    def schedule(self) -> torch.Tensor:
        """int32 [n] device view of the tile order of the tensor-core conv."""
        p = ctypes.c_void_p()
        _check(lib().smc_map_schedule(self.handle, ctypes.byref(p)), "smc_map_schedule")
        return self._view(p.value, (self.n,))

    def timing(self):
        """(lookups, tile schedule, pair lists) device times in ms of a build
        made with profiling on; the pair lists run concurrently with the
        schedule."""
        ms = (ctypes.c_float * 3)()
        _check(lib().smc_map_timing(self.handle, ms), "smc_map_timing")
        return float(ms[0]), float(ms[1]), float(ms[2])

    def free(self) -> None:
        if self._h is not None:
            _check(lib().smc_free_map(self._h), "smc_free_map")
            self._h = None

    def __del__(self):
        try:
            if self._h is not None and _lib is not None:
                _lib.smc_free_map(self._h)
                self._h = None
        except Exception:
            pass


_cache: Dict[Hashable, Map] = {}


def build_map(coords: torch.Tensor, grid: Sequence[int], batch: Optional[int] = None,
              key: Optional[Hashable] = None, stream=None, sync: bool = True) -> Map:
    """Build (or fetch from the cache under `key`) the map of int32 [N, 4]
    (b, z, y, x) coordinates on a (Z, Y, X) grid.  Like spconv's indice_key,
    `key` names a coordinate set so every conv on it reuses one map.  With
    sync=False the build is only enqueued (smc_build_map_async); device-side
    input errors then surface at Map.wait() or the first query."""
    if key is not None and key in _cache:
        return _cache[key]
    if coords.dtype != torch.int32 or coords.dim() != 2 or coords.shape[1] != 4:
        raise ValueError("coords must be int32 [N, 4]")
    if not coords.is_cuda:
        raise ValueError("coords must be a CUDA tensor")
    coords = coords.contiguous()
    n = coords.shape[0]
    if batch is None:
        batch = int(coords[:, 0].max().item()) + 1 if n else 1
    g = (ctypes.c_int32 * 3)(*[int(x) for x in grid])
    h = ctypes.c_void_p()
    fn = lib().smc_build_map if sync else lib().smc_build_map_async
    with torch.cuda.device(coords.device):
        _check(fn(_ptr(coords), n, int(batch), g, _stream(stream), ctypes.byref(h)), "smc_build_map")
    m = Map(h, n, int(batch), grid, coords.device)
    if key is not None:
        _cache[key] = m
    return m


def subdivide(parent: "Map", parent_coords: torch.Tensor, keep: Optional[torch.Tensor] = None, stream=None):
    """Children of every voxel of `parent` (x2 per axis, 8 per voxel in C
    order), optionally pruned by a uint8 [N, 8] `keep` mask; returns
    (child_coords int32 [M, 4], child Map on the doubled grid).  The child map
    is built from the parent map (smc_subdivide in include/smc.h)."""
    n = parent.n
    if parent_coords.dtype != torch.int32 or parent_coords.shape != (n, 4) or not parent_coords.is_cuda:
        raise ValueError("parent_coords must be the parent's int32 [N, 4] CUDA tensor")
    parent_coords = parent_coords.contiguous()
    if keep is not None:
        if keep.dtype not in (torch.uint8, torch.bool) or keep.numel() != 8 * n or not keep.is_cuda:
            raise ValueError("keep must be a uint8/bool CUDA tensor of N * 8 entries")
        keep = keep.contiguous().view(torch.uint8)
    out = torch.empty((max(8 * n, 1), 4), dtype=torch.int32, device=parent_coords.device)
    m = ctypes.c_int64()
    h = ctypes.c_void_p()
    with torch.cuda.device(parent_coords.device):
        _check(lib().smc_subdivide(parent.handle, _ptr(parent_coords), _ptr(keep) if keep is not None else None,
                                   _ptr(out), ctypes.byref(m), _stream(stream), ctypes.byref(h)), "smc_subdivide")
    grid = tuple(2 * int(g) for g in parent.grid)
    return out[: m.value], Map(h, int(m.value), parent.batch, grid, parent_coords.device)


POOL_MODES = {"max": 0, "mean": 1}


def _feats_arg(feats: Optional[torch.Tensor], n: int, device) -> int:
    if feats is None:
        return 0
    if feats.dtype not in _DTYPES or feats.dim() != 2 or feats.shape[0] != n or not feats.is_cuda:
        raise ValueError("feats must be a float32/bfloat16/float16 [N, C] CUDA tensor")
    if feats.device != device:
        raise ValueError("feats must be on the coordinates' device")
    return _DTYPES[feats.dtype]


def downsample(coords: torch.Tensor, grid: Sequence[int], feats: Optional[torch.Tensor] = None,
               mode: str = "mean", batch: Optional[int] = None, stream=None):
    """Pool by 2 into parent voxels (smc_downsample in include/smc.h; mode
    "max" or "mean").  Returns (parent_coords int32 [M, 4], pooled [M, C] or
    None, subdivision mask uint8 [M, 8], parent of each row int32 [N]);
    parents are numbered in order of first appearance.  Synchronises the
    stream once."""
    if mode not in POOL_MODES:
        raise ValueError("mode must be 'max' or 'mean'")
    if coords.dtype != torch.int32 or coords.dim() != 2 or coords.shape[1] != 4 or not coords.is_cuda:
        raise ValueError("coords must be an int32 [N, 4] CUDA tensor")
    coords = coords.contiguous()
    n = coords.shape[0]
    if batch is None:
        batch = int(coords[:, 0].max().item()) + 1 if n else 1
    dt = _feats_arg(feats, n, coords.device)
    if feats is not None:
        feats = feats.contiguous()
    dev = coords.device
    pc = torch.empty((max(n, 1), 4), dtype=torch.int32, device=dev)
    mask = torch.empty((max(n, 1), 8), dtype=torch.uint8, device=dev)
    parent = torch.empty((n,), dtype=torch.int32, device=dev)
    pooled = None if feats is None else torch.empty((max(n, 1), feats.shape[1]), dtype=feats.dtype, device=dev)
    m = ctypes.c_int64()
    g = (ctypes.c_int32 * 3)(*[int(x) for x in grid])
    with torch.cuda.device(dev):
        _check(lib().smc_downsample(_ptr(coords), n, int(batch), g, _ptr(feats),
                                    0 if feats is None else feats.shape[1], dt, POOL_MODES[mode], _ptr(pc),
                                    _ptr(pooled), _ptr(mask), _ptr(parent), ctypes.byref(m), _stream(stream)),
               "smc_downsample")
    k = int(m.value)
    return pc[:k], None if pooled is None else pooled[:k], mask[:k], parent


def upsample(coords: torch.Tensor, mask: Optional[torch.Tensor], feats: Optional[torch.Tensor] = None,
             parent: Optional["Map"] = None, stream=None):
    """Masked expansion by 2 (smc_upsample in include/smc.h): child j of
    voxel p, at offset (j % 2, j // 2 % 2, j // 4) along (z, y, x), where
    mask[p, j] != 0 (every child when mask is None), carrying p's features.
    Returns (child_coords int32 [M, 4], child feats [M, C] or None, child Map
    or None); the child map is built from `parent`, the map of `coords`, when
    it is given."""
    if coords.dtype != torch.int32 or coords.dim() != 2 or coords.shape[1] != 4 or not coords.is_cuda:
        raise ValueError("coords must be an int32 [N, 4] CUDA tensor")
    coords = coords.contiguous()
    n = coords.shape[0]
    if mask is not None:
        if mask.dtype not in (torch.uint8, torch.bool) or mask.numel() != 8 * n or not mask.is_cuda:
            raise ValueError("mask must be a uint8/bool CUDA tensor of N * 8 entries")
        mask = mask.contiguous().view(torch.uint8)
    dt = _feats_arg(feats, n, coords.device)
    if feats is not None:
        feats = feats.contiguous()
    if parent is not None and parent.n != n:
        raise ValueError("parent map must be the map of coords")
    dev = coords.device
    out = torch.empty((max(8 * n, 1), 4), dtype=torch.int32, device=dev)
    kf = None if feats is None else torch.empty((max(8 * n, 1), feats.shape[1]), dtype=feats.dtype, device=dev)
    m = ctypes.c_int64()
    h = ctypes.c_void_p()
    with torch.cuda.device(dev):
        _check(lib().smc_upsample(_ptr(coords), n, _ptr(mask), _ptr(feats), 0 if feats is None else feats.shape[1],
                                  dt, None if parent is None else parent.handle, _ptr(out), _ptr(kf),
                                  ctypes.byref(m), _stream(stream), ctypes.byref(h) if parent is not None else None),
               "smc_upsample")
    k = int(m.value)
    cm = None
    if parent is not None:
        cm = Map(h, k, parent.batch, tuple(2 * int(x) for x in parent.grid), dev)
    return out[:k], None if kf is None else kf[:k], cm


NOALLOC_MAX_N = 1 << 18


def neighbour_map_noalloc(coords: torch.Tensor, grid: Sequence[int], batch: Optional[int] = None,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """int32 [N, 27] neighbour map computed without any device allocation by
    the library (its scratch is a fixed static device array; see
    smc_neighbour_map_noalloc in include/smc.h).  For callers that reserve
    device memory up front and may not allocate while they run: pass `out`
    preallocated.  N is limited to NOALLOC_MAX_N."""
    if coords.dtype != torch.int32 or coords.dim() != 2 or coords.shape[1] != 4 or not coords.is_cuda:
        raise ValueError("coords must be an int32 [N, 4] CUDA tensor")
    if not coords.is_contiguous():
        raise ValueError("coords must be contiguous")
    n = coords.shape[0]
    if batch is None:
        batch = int(coords[:, 0].max().item()) + 1 if n else 1
    if out is None:
        out = torch.empty((n, 27), dtype=torch.int32, device=coords.device)
    elif out.shape != (n, 27) or out.dtype != torch.int32 or not out.is_contiguous():
        raise ValueError("out must be a contiguous int32 [N, 27] tensor")
    g = (ctypes.c_int32 * 3)(*[int(x) for x in grid])
    with torch.cuda.device(coords.device):
        _check(lib().smc_neighbour_map_noalloc(_ptr(coords), n, int(batch), g, _ptr(out), _stream(stream)),
               "smc_neighbour_map_noalloc")
    return out


def clear_cache() -> None:
    for m in _cache.values():
        m.free()
    _cache.clear()


ACTS = {None: 0, "none": 0, "relu": 1, "silu": 2}


def conv(m: Map, feats: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
         ksize: int = 3, orientation: int = 1, out: Optional[torch.Tensor] = None,
         stream=None, residual: Optional[torch.Tensor] = None, act: Optional[str] = None,
         coords: Optional[torch.Tensor] = None, stats: Optional[torch.Tensor] = None,
         groups: int = 1) -> torch.Tensor:
    """Submanifold conv over map `m`: feats [N, Cin], KRSC weight [Cout, k, k, k, Cin].
    Fused epilogue (smc_conv_ex): out = act(conv + bias) + residual, act in
    {None, "relu", "silu"}; with `stats` (fp64 [batch, groups, 3], zeroed by
    the caller) and `coords` (the map's int32 [N, 4]) the GroupNorm
    statistics of the output are added into `stats`."""
    if feats.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {feats.dtype}")
    if weight.dtype != feats.dtype or (bias is not None and bias.dtype != feats.dtype):
        raise TypeError("feats, weight and bias must share one dtype")
    if feats.dim() != 2 or feats.shape[0] != m.n:
        raise ValueError(f"feats must be [N={m.n}, Cin]")
    if act not in ACTS:
        raise ValueError(f"act must be one of {list(ACTS)}")
    cin = feats.shape[1]
    cout = weight.shape[0]
    if tuple(weight.shape) != (cout, ksize, ksize, ksize, cin):
        raise ValueError(f"weight must be KRSC [Cout, {ksize}, {ksize}, {ksize}, {cin}]")
    if bias is not None and tuple(bias.shape) != (cout,):
        raise ValueError("bias must be [Cout]")
    feats = feats.contiguous()
    weight = weight.contiguous()
    bias = None if bias is None else bias.contiguous()
    if out is None:
        out = torch.empty((m.n, cout), dtype=feats.dtype, device=feats.device)
    elif out.shape != (m.n, cout) or out.dtype != feats.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous [N, Cout] tensor of the feats dtype")
    if residual is not None and (residual.shape != (m.n, cout) or residual.dtype != feats.dtype
                                 or not residual.is_contiguous()):
        raise ValueError("residual must be a contiguous [N, Cout] tensor of the feats dtype")
    if stats is not None:
        if coords is None or coords.dtype != torch.int32 or coords.shape != (m.n, 4):
            raise ValueError("stats need the map's int32 [N, 4] coords")
        if stats.dtype != torch.float64 or stats.shape != (m.batch, groups, 3) or not stats.is_contiguous():
            raise ValueError(f"stats must be a contiguous float64 [{m.batch}, {groups}, 3] tensor")
        coords = coords.contiguous()
    with torch.cuda.device(feats.device):
        if residual is None and act is None and stats is None:
            _check(lib().smc_conv(m.handle, _ptr(feats), cin, _ptr(weight), _ptr(bias), _ptr(out), cout,
                                  ksize, orientation, _DTYPES[feats.dtype], _stream(stream)), "smc_conv")
        else:
            _check(lib().smc_conv_ex(m.handle, _ptr(feats), cin, _ptr(weight), _ptr(bias), _ptr(residual),
                                     _ptr(out), cout, ksize, orientation, _DTYPES[feats.dtype], ACTS[act],
                                     _ptr(coords) if stats is not None else None, _ptr(stats), int(groups),
                                     _stream(stream)), "smc_conv_ex")
    return out


def group_stats(x: torch.Tensor, coords: torch.Tensor, batch: int, groups: int,
                stats: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fp64 [batch, groups, 3]: (sum, sum of squares, count) of x [N, C] per
    batch item (coords[:, 0]) and group of C / groups channels, added into
    `stats` if given (smc_group_stats)."""
    if x.dtype not in _DTYPES or x.dim() != 2:
        raise TypeError("x must be a 2-D float32 / bfloat16 / float16 tensor")
    n, c = x.shape
    if coords.dtype != torch.int32 or coords.shape != (n, 4):
        raise ValueError("coords must be int32 [N, 4]")
    if stats is None:
        stats = torch.zeros((batch, groups, 3), dtype=torch.float64, device=x.device)
    x, coords = x.contiguous(), coords.contiguous()
    with torch.cuda.device(x.device):
        _check(lib().smc_group_stats(_ptr(x), n, c, _ptr(coords), int(batch), int(groups), _ptr(stats),
                                     _DTYPES[x.dtype], _stream(stream)), "smc_group_stats")
    return stats


def group_norm(x: torch.Tensor, coords: torch.Tensor, batch: int, groups: int, stats: torch.Tensor,
               gamma: Optional[torch.Tensor] = None, beta: Optional[torch.Tensor] = None, eps: float = 1e-5,
               act: Optional[str] = None, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """GroupNorm over a sparse tensor then `act` (smc_group_norm), with the
    statistics of `stats` (from group_stats or conv(..., stats=...))."""
    if x.dtype not in _DTYPES or x.dim() != 2:
        raise TypeError("x must be a 2-D float32 / bfloat16 / float16 tensor")
    if act not in ACTS:
        raise ValueError(f"act must be one of {list(ACTS)}")
    n, c = x.shape
    x, coords = x.contiguous(), coords.contiguous()
    if out is None:
        out = torch.empty_like(x)
    for t in (gamma, beta):
        if t is not None and (t.dtype != x.dtype or t.shape != (c,)):
            raise ValueError("gamma and beta must be [C] of the x dtype")
    with torch.cuda.device(x.device):
        _check(lib().smc_group_norm(_ptr(x), n, c, _ptr(coords), int(batch), int(groups), _ptr(stats.contiguous()),
                                    _ptr(gamma), _ptr(beta), float(eps), ACTS[act], _ptr(out), _DTYPES[x.dtype],
                                    _stream(stream)), "smc_group_norm")
    return out


def status(stream=None) -> None:
    """Synchronise the stream and raise if a conv kernel reported a timeout."""
    _check(lib().smc_status(_stream(stream)), "smc_status")


def set_conv_epilogue(where: int) -> None:
    """Where conv(..., act=, residual=) applies them on the tensor-core
    kernel: 0 = a row pass behind the conv (default), 1 = the conv's own
    epilogue (smc_set_conv_epilogue)."""
    _check(lib().smc_set_conv_epilogue(int(where)), "smc_set_conv_epilogue")


def set_conv_variant(variant: int) -> None:
    """Tensor-core conv: 0 default, 1 fused (one CTA per tile), 2 fused with CTA
    pairs, 3 per-offset gather-GEMM-scatter."""
    _check(lib().smc_set_conv_variant(int(variant)), "smc_set_conv_variant")


def set_map_lookup(mode: int) -> None:
    """Lookup structure of later builds: 0 by size, 1 hash table, 2 dense grid."""
    _check(lib().smc_set_map_lookup(int(mode)), "smc_set_map_lookup")


def set_alloc_fail_after(k: int) -> None:
    """Test hook: the k-th device allocation of the library from now on
    reports failure, once (0 disarms it; smc_set_alloc_fail_after)."""
    _check(lib().smc_set_alloc_fail_after(int(k)), "smc_set_alloc_fail_after")


def set_wait_limit_ns(ns: int) -> None:
    """Bound of the scans' device-side waits, in ns (0 = the default 2 s)."""
    _check(lib().smc_set_wait_limit_ns(int(ns)), "smc_set_wait_limit_ns")


def set_conv_priority(on: bool) -> None:
    """Run convs on the library's high-priority streams, forked from and
    joined back to the caller's stream (default), or on the caller's stream
    itself (smc_set_conv_priority)."""
    _check(lib().smc_set_conv_priority(1 if on else 0), "smc_set_conv_priority")


def set_schedule_segment(rows: int) -> None:
    """Sort the tile schedule within segments of `rows` consecutive input rows
    (0 = the whole map, the default; -1 = the default; else a multiple of 2048;
    smc_set_schedule_segment).  Applies to maps built afterwards."""
    _check(lib().smc_set_schedule_segment(int(rows)), "smc_set_schedule_segment")


def set_scan_hold(ticket: int) -> None:
    """Test hook: the scan segment with this ticket publishes nothing, so the
    later segments' waits run out (-1 turns it off; smc_set_scan_hold)."""
    _check(lib().smc_set_scan_hold(int(ticket)), "smc_set_scan_hold")


def set_hash_capacity(slots: int) -> None:
    _check(lib().smc_set_hash_capacity(int(slots)), "smc_set_hash_capacity")


def kernel_launches() -> int:
    """Kernels launched by libsmc in this process so far."""
    c = ctypes.c_int64()
    _check(lib().smc_kernel_launches(ctypes.byref(c)), "smc_kernel_launches")
    return int(c.value)


def set_profiling(on: bool) -> None:
    _check(lib().smc_set_profiling(1 if on else 0), "smc_set_profiling")
