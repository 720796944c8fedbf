"""Python face of the CPU oracle (smc_oracle.cpp).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.  It shares nothing
with the CUDA library: it compiles and loads its own C++ file with g++, takes
numpy arrays, and computes in fp64.

Functions
---------
neighbour_map(coords, grid, k=3)          -> int32 [N, k^3]
pair_lists(nbr)                           -> (counts int64[T], offsets int64[T+1], in_idx, out_idx)
conv(coords, grid, feats, weight, bias, k=3, orientation=+1, rows=None, threads=1) -> fp64 [rows, Cout]
subdivide(coords, keep=None)              -> int32 [M, 4] children, (parent row, octant) order
activation(y, act)                        -> fp64, act 0 none / 1 ReLU / 2 SiLU
group_stats(x, coords, batch, groups)     -> fp64 [batch, groups, 3] (sum, sum of squares, count)
group_norm(x, coords, batch, groups, gamma, beta, eps, act) -> fp64 [N, C]
downsample(coords, grid, feats=None, mode=POOL_MEAN, batch=None)
                                          -> (parent coords [M, 4], pooled fp64 [M, C] or None,
                                              subdivision mask uint8 [M, 8], parent row int32 [N])
upsample(coords, mask, feats=None)        -> (child coords [K, 4], child feats fp64 [K, C] or None)

The definition each follows is cited in smc_oracle.cpp.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "smc_oracle.cpp")
_LIB = os.path.join(_HERE, "libsmc_oracle.so")

ERRORS = {-1: "bad argument", -2: "coordinate out of range", -3: "duplicate coordinate"}


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle error {code}: {ERRORS.get(code, 'unknown')}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libsmc_oracle.so (g++, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-shared", "-fPIC",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_neighbour_map.argtypes = [P, i64, P, i32, P]
        lib.oracle_pair_lists.argtypes = [P, i64, i32, P, P, P]
        lib.oracle_conv.argtypes = [P, i64, P, P, i64, P, P, i64, i32, i32, P, i64, P, i32]
        for f in (lib.oracle_neighbour_map, lib.oracle_pair_lists, lib.oracle_conv):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _coords(coords) -> np.ndarray:
    c = np.ascontiguousarray(coords, dtype=np.int32)
    if c.ndim != 2 or c.shape[1] != 4:
        raise ValueError("coords must be int32 [N, 4] (b, z, y, x)")
    return c


def _grid(grid: Sequence[int]) -> np.ndarray:
    g = np.ascontiguousarray(grid, dtype=np.int32)
    if g.shape != (3,):
        raise ValueError("grid must be (Z, Y, X)")
    return g


def neighbour_map(coords, grid, k: int = 3) -> np.ndarray:
    c, g = _coords(coords), _grid(grid)
    n = c.shape[0]
    nbr = np.empty((n, k ** 3), dtype=np.int32)
    rc = _load().oracle_neighbour_map(_ptr(c), n, _ptr(g), k, _ptr(nbr))
    if rc:
        raise OracleError(rc)
    return nbr


def pair_lists(nbr: np.ndarray):
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    n, taps = nbr.shape
    counts = np.zeros(taps, dtype=np.int64)
    lib = _load()
    rc = lib.oracle_pair_lists(_ptr(nbr), n, taps, _ptr(counts), None, None)
    if rc:
        raise OracleError(rc)
    total = int(counts.sum())
    in_idx = np.empty(total, dtype=np.int32)
    out_idx = np.empty(total, dtype=np.int32)
    rc = lib.oracle_pair_lists(_ptr(nbr), n, taps, _ptr(counts), _ptr(in_idx), _ptr(out_idx))
    if rc:
        raise OracleError(rc)
    offsets = np.zeros(taps + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    return counts, offsets, in_idx, out_idx


def conv(coords, grid, feats, weight, bias=None, k: int = 3, orientation: int = 1,
         rows=None, threads: int = 1) -> np.ndarray:
    c, g = _coords(coords), _grid(grid)
    n = c.shape[0]
    f = np.ascontiguousarray(feats, dtype=np.float64)
    w = np.ascontiguousarray(weight, dtype=np.float64)
    if f.shape[0] != n:
        raise ValueError("feats must have one row per coordinate")
    cin = f.shape[1]
    cout = w.shape[0]
    if w.shape != (cout, k, k, k, cin):
        raise ValueError(f"weight must be KRSC [Cout, {k}, {k}, {k}, Cin={cin}], got {w.shape}")
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = n if r is None else r.shape[0]
    out = np.empty((nrows, cout), dtype=np.float64)
    rc = _load().oracle_conv(_ptr(c), n, _ptr(g), _ptr(f), cin, _ptr(w), _ptr(b), cout, k,
                             orientation, _ptr(r), nrows, _ptr(out), threads)
    if rc:
        raise OracleError(rc)
    return out


def subdivide(coords, keep=None) -> np.ndarray:
    """Children of every voxel, the decoders' x2 upsampling: voxel (b, z, y, x)
    splits into (b, 2z+a, 2y+c, 2x+e) for a, c, e in {0, 1}, octant
    o = 4a + 2c + e in C order (LATO.2 MLX port README, "The scope, once
    measured" table; shared sparse-core commit log).  `keep` [N, 8] (nonzero =
    keep) prunes children; the result lists the kept children parent by
    parent, octants ascending.  Plain definition, one loop per octant."""
    c = _coords(coords).astype(np.int64)
    n = c.shape[0]
    kept = np.ones((n, 8), dtype=bool) if keep is None else (np.asarray(keep).reshape(n, 8) != 0)
    children = np.empty((n, 8, 4), dtype=np.int64)
    for o in range(8):
        a, cc, e = o >> 2, (o >> 1) & 1, o & 1
        children[:, o, 0] = c[:, 0]
        children[:, o, 1] = 2 * c[:, 1] + a
        children[:, o, 2] = 2 * c[:, 2] + cc
        children[:, o, 3] = 2 * c[:, 3] + e
    return children[kept].astype(np.int32)


ACT_NONE, ACT_RELU, ACT_SILU = 0, 1, 2


def activation(y, act: int) -> np.ndarray:
    """The activations around the decoders' convs (Pixal3D MLX README
    "Status": norms, activations, ResBlock; LATO.2 MLX port README "Status":
    remaining sparse ops SparseGroupNorm32, activations): ReLU max(y, 0) and
    SiLU y * sigmoid(y) = y / (1 + exp(-y)), in fp64."""
    y = np.asarray(y, dtype=np.float64)
    if act == ACT_NONE:
        return y.copy()
    if act == ACT_RELU:
        return np.maximum(y, 0.0)
    if act == ACT_SILU:
        return y / (1.0 + np.exp(-y))
    raise ValueError("act must be 0, 1 or 2")


def group_stats(x, coords, batch: int, groups: int) -> np.ndarray:
    """Per batch item b and channel group g (channels g*C/groups .. (g+1)*C/groups - 1):
    the sum, the sum of squares and the number of values of x over the item's
    rows, in fp64 -- what GroupNorm over a sparse tensor normalises with."""
    x = np.asarray(x, dtype=np.float64)
    n, c = x.shape
    assert c % groups == 0
    b = _coords(coords)[:, 0].astype(np.int64)
    xg = x.reshape(n, groups, c // groups)
    out = np.zeros((batch, groups, 3))
    for item in range(batch):
        rows = xg[b == item]
        out[item, :, 0] = rows.sum(axis=(0, 2))
        out[item, :, 1] = (rows * rows).sum(axis=(0, 2))
        out[item, :, 2] = rows.shape[0] * (c // groups)
    return out


def group_norm(x, coords, batch: int, groups: int, gamma=None, beta=None, eps: float = 1e-5, act: int = 0):
    """GroupNorm over a sparse tensor followed by an activation: for every
    batch item and channel group, (x - mean) / sqrt(var + eps) with the
    item's rows and the group's channels as the population (biased
    variance), then gamma * . + beta per channel, then `act`."""
    x = np.asarray(x, dtype=np.float64)
    n, c = x.shape
    st = group_stats(x, coords, batch, groups)
    b = _coords(coords)[:, 0].astype(np.int64)
    cnt = np.maximum(st[:, :, 2], 1.0)
    mean = st[:, :, 0] / cnt
    var = st[:, :, 1] / cnt - mean * mean
    g_of_c = np.arange(c) // (c // groups)
    y = (x - mean[b][:, g_of_c]) / np.sqrt(var[b][:, g_of_c] + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)[None, :]
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)[None, :]
    return activation(y, act)


POOL_MAX, POOL_MEAN = 0, 1


def subidx(dz, dy, dx) -> int:
    """Child index inside a factor-2 parent as the subdivision mask numbers
    it: the offset along spatial axis i is subidx // 2**i % 2, axis 0 (z)
    varying fastest -- the reverse of the C order subdivide() uses (shared
    sparse-core commit log, the masked-upsample entry)."""
    return dz + 2 * dy + 4 * dx


def downsample(coords, grid, feats=None, mode: int = POOL_MEAN, batch: Optional[int] = None):
    """Pooling by 2 into parent voxels, SparseDownsample(2) (shared
    sparse-core commit log: modes 'max' and 'mean'; Pixal3D MLX README
    "Status").  Row i of (b, z, y, x) pools into the parent
    (b, z // 2, y // 2, x // 2).  Parents are numbered in order of first
    appearance: walking the rows in order, a parent not seen before takes the
    next index.  Returns the parents' coordinates, their pooled features
    (elementwise max, or the mean over the children present, in fp64), the
    subdivision mask (mask[p, subidx] = 1 for every child present) and each
    row's parent.  Coordinates outside (batch, grid) and repeated sites are
    errors, as in the map build."""
    c = _coords(coords).astype(np.int64)
    g = _grid(grid)
    n = c.shape[0]
    nb = (int(c[:, 0].max()) + 1 if n else 1) if batch is None else batch
    lo_ok = (c >= 0).all(axis=1)
    hi_ok = (c[:, 0] < nb) & (c[:, 1] < g[0]) & (c[:, 2] < g[1]) & (c[:, 3] < g[2])
    if n and not (lo_ok & hi_ok).all():
        raise OracleError(-2)
    index = {}
    parent_coords = []
    parent = np.empty(n, dtype=np.int32)
    for i in range(n):
        b, z, y, x = (int(v) for v in c[i])
        key = (b, z // 2, y // 2, x // 2)
        if key not in index:
            index[key] = len(parent_coords)
            parent_coords.append(key)
        parent[i] = index[key]
    m = len(parent_coords)
    mask = np.zeros((m, 8), dtype=np.uint8)
    for i in range(n):
        j = subidx(int(c[i, 1]) % 2, int(c[i, 2]) % 2, int(c[i, 3]) % 2)
        if mask[parent[i], j]:
            raise OracleError(-3)
        mask[parent[i], j] = 1
    pc = np.array(parent_coords, dtype=np.int32).reshape(m, 4)
    pooled = None
    if feats is not None:
        f = np.asarray(feats, dtype=np.float64)
        if f.shape[0] != n:
            raise ValueError("feats must have one row per coordinate")
        if mode == POOL_MAX:
            pooled = np.full((m, f.shape[1]), -np.inf)
            np.maximum.at(pooled, parent, f)
        elif mode == POOL_MEAN:
            pooled = np.zeros((m, f.shape[1]))
            np.add.at(pooled, parent, f)
            pooled /= mask.sum(axis=1, dtype=np.float64)[:, None]
        else:
            raise ValueError("mode must be POOL_MAX (0) or POOL_MEAN (1)")
    return pc, pooled, mask, parent


def upsample(coords, mask, feats=None):
    """Masked expansion by 2, SparseUpsample(2) (shared sparse-core commit
    log, the masked-upsample entry; Pixal3D MLX README, remaining ops): parent
    p emits the child at subidx j wherever mask[p, j] != 0 -- 0 to 8
    children, unlike subdivide(), which always emits 8 -- at
    (b, 2z + j % 2, 2y + j // 2 % 2, 2x + j // 4 % 2), listed parent by
    parent, j ascending.  Each child carries its parent's features."""
    c = _coords(coords).astype(np.int64)
    n = c.shape[0]
    mk = np.asarray(mask).reshape(n, 8) != 0
    children, src = [], []
    for p in range(n):
        b, z, y, x = (int(v) for v in c[p])
        for j in range(8):
            if mk[p, j]:
                children.append((b, 2 * z + j % 2, 2 * y + j // 2 % 2, 2 * x + j // 4 % 2))
                src.append(p)
    kids = np.array(children, dtype=np.int32).reshape(len(children), 4)
    out = None
    if feats is not None:
        f = np.asarray(feats, dtype=np.float64)
        out = f[np.array(src, dtype=np.int64)] if src else np.zeros((0, f.shape[1]))
    return kids, out
