"""Seeded synthetic workloads for submanifold sparse convolution.

This module only draws inputs: voxel coordinate sets with the structure of the
workloads the sparse-voxel decoders run on (random occupancy, thin sphere
shells, thin planes, x8 subdivision chains), and feature / weight / bias
tensors.  It holds none of the convolution's arithmetic, so both the GPU path
and the CPU oracle can be fed from it without sharing any of the method.

Recipe (every draw comes from ``numpy.random.Generator(PCG64(seed))`` with
``seed = 1000 * config + item``):

* features  ~ N(0, 1)
* weights   ~ N(0, 1 / (k^3 * Cin)) in KRSC layout [Cout, k, k, k, Cin]
* bias      ~ N(0, 0.1)            (second parameter is the variance)
* bf16 / fp16 values are the fp32 draws rounded to nearest-even.

A *shell* of radius r and centre c is the set of integer points p with
| ||p - c||_2 - r | < 1 (two voxels thick).  A *plane* with unit normal n and
offset delta is the set of p with |n . p - delta| < 0.5 (one voxel thick).
Coordinates are returned as int32 [N, 4] rows (b, z, y, x) in lexicographic
order, the order ``numpy.argwhere`` gives.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

__all__ = [
    "rng_for", "round_to", "to_bf16_bits", "bf16_bits_to_f32",
    "random_occupancy", "shell_points", "plane_points", "union_of_shells",
    "full_grid", "varlen_item", "subdivide_shell", "subdivision_keep_mask", "Workload", "workload",
    "features", "weights", "bias", "WORKLOADS", "small_integer_values",
]


def rng_for(config: int, item: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.PCG64(1000 * int(config) + int(item)))


# ----------------------------------------------------------------------------
# rounding of fp32 draws to the storage dtype (round to nearest, ties to even)
# ----------------------------------------------------------------------------
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to ``dtype`` and return them as fp32 (exact)."""
    x = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x.copy()
    if dtype == "bf16":
        return bf16_bits_to_f32(to_bf16_bits(x)).reshape(x.shape)
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------
# coordinate sets
# ----------------------------------------------------------------------------
def _with_batch(zyx: np.ndarray, b: int) -> np.ndarray:
    out = np.empty((zyx.shape[0], 4), dtype=np.int32)
    out[:, 0] = b
    out[:, 1:] = zyx
    return out


def random_occupancy(G: int, p: float, rng: np.random.Generator) -> np.ndarray:
    """Sites of a G^3 grid kept independently with probability p -> int32 [n,3]."""
    mask = rng.random((G, G, G)) < p
    return np.argwhere(mask).astype(np.int32)


def _shell_into(mask: np.ndarray, c: np.ndarray, r: float) -> None:
    G = mask.shape[0]
    lo = np.maximum(np.floor(c - r - 2).astype(int), 0)
    hi = np.minimum(np.ceil(c + r + 3).astype(int), G)
    ys = np.arange(lo[1], hi[1], dtype=np.float64)[:, None]
    xs = np.arange(lo[2], hi[2], dtype=np.float64)[None, :]
    dyx2 = (ys - c[1]) ** 2 + (xs - c[2]) ** 2
    for z in range(lo[0], hi[0]):
        d = np.sqrt((z - c[0]) ** 2 + dyx2)
        mask[z, lo[1]:hi[1], lo[2]:hi[2]] |= np.abs(d - r) < 1.0


def _plane_into(mask: np.ndarray, n: np.ndarray, delta: float) -> None:
    G = mask.shape[0]
    ys = np.arange(G, dtype=np.float64)[:, None]
    xs = np.arange(G, dtype=np.float64)[None, :]
    nyx = n[1] * ys + n[2] * xs
    for z in range(G):
        mask[z] |= np.abs(n[0] * z + nyx - delta) < 0.5


def shell_points(G: int, c, r: float) -> np.ndarray:
    mask = np.zeros((G, G, G), dtype=bool)
    _shell_into(mask, np.asarray(c, dtype=np.float64), float(r))
    return np.argwhere(mask).astype(np.int32)


def plane_points(G: int, n, delta: float) -> np.ndarray:
    mask = np.zeros((G, G, G), dtype=bool)
    _plane_into(mask, np.asarray(n, dtype=np.float64), float(delta))
    return np.argwhere(mask).astype(np.int32)


def _random_centre(G: int, r: float, rng: np.random.Generator) -> np.ndarray:
    return rng.uniform(r + 1, G - r - 2, size=3)


def union_of_shells(G: int, count: int, rmin: float, rmax: float,
                    rng: np.random.Generator) -> np.ndarray:
    mask = np.zeros((G, G, G), dtype=bool)
    for _ in range(count):
        r = rng.uniform(rmin, rmax)
        _shell_into(mask, _random_centre(G, r, rng), r)
    return np.argwhere(mask).astype(np.int32)


def full_grid(G: int) -> np.ndarray:
    return np.argwhere(np.ones((G, G, G), dtype=bool)).astype(np.int32)


def varlen_item(G: int, target: int, rmin: float, rmax: float,
                rng: np.random.Generator) -> np.ndarray:
    """Alternately add random shells and random planes until >= target sites."""
    mask = np.zeros((G, G, G), dtype=bool)
    k = 0
    while int(mask.sum()) < target:
        if k % 2 == 0:
            r = rng.uniform(rmin, rmax)
            _shell_into(mask, _random_centre(G, r, rng), r)
        else:
            n = rng.normal(size=3)
            n /= np.linalg.norm(n)
            q = rng.uniform(0.25 * G, 0.75 * G, size=3)
            _plane_into(mask, n, float(n @ q))
        k += 1
    return np.argwhere(mask).astype(np.int32)


def subdivide_shell(zyx: np.ndarray, c: np.ndarray, r: float) -> Tuple[np.ndarray, np.ndarray, float]:
    """x8 subdivision: every site p emits children 2p + (a, b, c) in C order
    (a slowest); children are kept when they lie in the same analytic shell at
    the doubled resolution (centre 2c + 0.5, radius 2r, two voxels thick).
    Returns (children [m,3] in lexicographic order, new centre, new radius)."""
    off = np.argwhere(np.ones((2, 2, 2), dtype=bool)).astype(np.int32)  # C order
    kids = (2 * zyx[:, None, :] + off[None, :, :]).reshape(-1, 3)
    c2 = 2.0 * np.asarray(c, dtype=np.float64) + 0.5
    r2 = 2.0 * r
    d = np.sqrt(((kids.astype(np.float64) - c2) ** 2).sum(axis=1))
    kids = kids[np.abs(d - r2) < 1.0]
    order = np.lexsort((kids[:, 2], kids[:, 1], kids[:, 0]))
    return kids[order].astype(np.int32), c2, r2


def subdivision_keep_mask(parent_coords: np.ndarray, child_coords: np.ndarray,
                          child_grid: Tuple[int, int, int]) -> np.ndarray:
    """uint8 [N, 8]: which of each parent's 8 children (octant o = 4a + 2b + c,
    the child 2p + (a, b, c)) appear in `child_coords` -- the pruning decision
    of a decoder step, as input data for a subdivision."""
    off = np.argwhere(np.ones((2, 2, 2), dtype=bool)).astype(np.int64)  # C order
    p = parent_coords.astype(np.int64)
    kids = 2 * p[:, None, 1:] + off[None, :, :]
    G = np.asarray(child_grid, dtype=np.int64)

    def key(b, zyx):
        return ((b * G[0] + zyx[..., 0]) * G[1] + zyx[..., 1]) * G[2] + zyx[..., 2]

    c = child_coords.astype(np.int64)
    have = np.isin(key(p[:, None, 0], kids), key(c[:, 0], c[:, 1:]))
    return have.astype(np.uint8)


# ----------------------------------------------------------------------------
# dense tensors
# ----------------------------------------------------------------------------
def features(N: int, C: int, rng: np.random.Generator, dtype: str) -> np.ndarray:
    return round_to(rng.standard_normal((N, C), dtype=np.float32), dtype)


def weights(Cout: int, Cin: int, k: int, rng: np.random.Generator, dtype: str) -> np.ndarray:
    std = np.sqrt(1.0 / (k ** 3 * Cin))
    w = rng.standard_normal((Cout, k, k, k, Cin), dtype=np.float32) * np.float32(std)
    return round_to(w, dtype)


def bias(Cout: int, rng: np.random.Generator, dtype: str) -> np.ndarray:
    b = rng.standard_normal(Cout, dtype=np.float32) * np.float32(np.sqrt(0.1))
    return round_to(b, dtype)


def small_integer_values(shape, rng: np.random.Generator) -> np.ndarray:
    """Values in {-1, 0, 1}: every partial sum of a conv over them is a small
    integer, exact in fp32, bf16 and fp16 accumulation alike."""
    return rng.integers(-1, 2, size=shape).astype(np.float32)


# ----------------------------------------------------------------------------
# the named workloads
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    name: str
    coords: np.ndarray                 # int32 [N, 4] (b, z, y, x)
    grid: Tuple[int, int, int]         # (Z, Y, X)
    cin: int
    cout: int
    dtypes: Tuple[str, ...]
    layers: int = 1
    ksizes: Tuple[int, ...] = (3,)
    config: int = 0
    note: str = ""
    extra: Dict = dataclasses.field(default_factory=dict)

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])


def _tiny(config=1) -> Workload:
    rng = rng_for(config, 0)
    zyx = random_occupancy(16, 0.1, rng)
    return Workload("tiny_16^3_p0.1_c16", _with_batch(zyx, 0), (16, 16, 16), 16, 16,
                    ("f32",), 1, (3, 1), config,
                    "batch 1, 16^3 grid, 10% random occupancy, 16->16 fp32")


def _shell2(config=2) -> Workload:
    items = []
    for b in range(2):
        rng = rng_for(config, b)
        r = rng.uniform(20, 28)
        items.append(_with_batch(shell_points(64, _random_centre(64, r, rng), r), b))
    return Workload("shell_b2_64^3_c64", np.concatenate(items), (64, 64, 64), 64, 64,
                    ("f32", "bf16"), 4, (3,), config,
                    "batch 2, 64^3 grid, one 2-voxel shell r~U[20,28] per item, 64->64, 4 layers on one map")


def _shells6(config=3, item=0) -> Workload:
    rng = rng_for(config, item)
    zyx = union_of_shells(128, 6, 20, 36, rng)
    tag = "" if item == 0 else f"_draw{item}"
    return Workload(f"shells6_128^3_c128{tag}", _with_batch(zyx, 0), (128, 128, 128), 128, 128,
                    ("bf16",), 1, (3,), config,
                    "batch 1, 128^3 grid, union of 6 shells r~U[20,36], 128->128 bf16, fp32 accumulate"
                    + ("" if item == 0 else f" (draw {item} of the same recipe)"))


def _full128(config=3) -> Workload:
    return Workload("full_128^3_c128", _with_batch(full_grid(128), 0), (128, 128, 128), 128, 128,
                    ("bf16",), 1, (3,), config,
                    "batch 1, fully occupied 128^3 grid, 128->128 bf16, fp32 accumulate")


def _varlen4(config=4, G=256, tmin=300_000, tmax=600_000) -> Workload:
    items = []
    for b in range(4):
        rng = rng_for(config, b)
        target = int(rng.uniform(tmin, tmax))
        items.append(_with_batch(varlen_item(G, target, 40 * G / 256, 120 * G / 256, rng), b))
    return Workload(f"varlen_b4_{G}^3_c64", np.concatenate(items), (G, G, G), 64, 64,
                    ("f16",), 1, (3, 1), config,
                    f"batch 4, {G}^3 grid, per-item shells+planes to U[{tmin},{tmax}] sites, 64->64 fp16, k=3 then k=1")


_C5_STAGES = ((64, 512), (128, 256), (256, 128), (512, 64))


def decoder_stages(config=5, upto: int = 4) -> List[Workload]:
    rng = rng_for(config, 0)
    G0 = _C5_STAGES[0][0]
    r = 28.0
    c = _random_centre(G0, r, rng)
    zyx = shell_points(G0, c, r)
    out = []
    for s in range(upto):
        G, C = _C5_STAGES[s]
        if s > 0:
            zyx, c, r = subdivide_shell(zyx, c, r)
        out.append(Workload(f"decoder_stage{s}_{G}^3_c{C}", _with_batch(zyx, 0), (G, G, G), C, C,
                            ("bf16",), 10, (3,), config,
                            f"decoder stage {s}: {G}^3 grid, C={C}, 10 bf16 k=3 layers on one map",
                            {"stage": s}))
    return out


WORKLOADS = {
    "tiny": _tiny,
    "shell2": _shell2,
    "shells6": _shells6,
    # another seeded draw of the same recipe, whose size (117,818 voxels)
    # matches the "~120k" the configuration states
    "shells6_118k": lambda: _shells6(item=4),
    "full128": _full128,
    "varlen4": _varlen4,
}


def workload(name: str) -> Workload:
    if name.startswith("decoder"):
        s = int(name[len("decoder"):] or 3)
        return decoder_stages(upto=s + 1)[s]
    return WORKLOADS[name]()


def layer_tensors(w: Workload, dtype: str, layer: int = 0, ksize: int = 3,
                  cin: Optional[int] = None, cout: Optional[int] = None):
    """Features, weights and bias for one layer of a workload (fp32 arrays
    holding values already rounded to ``dtype``)."""
    cin = w.cin if cin is None else cin
    cout = w.cout if cout is None else cout
    rng = rng_for(w.config, 100 + 10 * layer + ksize)
    f = features(w.n, cin, rng, dtype)
    wt = weights(cout, cin, ksize, rng, dtype)
    b = bias(cout, rng, dtype)
    return f, wt, b
