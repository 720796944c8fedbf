"""One large item across ranks: z-slabs with one halo exchange per layer.

A submanifold conv with k = 3 reads, for every output voxel, only voxels
whose z differs by at most one.  Splitting the voxels into contiguous
z-slabs, one per rank, therefore makes every layer local except for the
one-voxel-deep boundary planes: before each layer a rank receives the rows of
the plane just below its slab from the rank that owns it, and the plane just
above, then runs the ordinary map build (once) and convs on its own rows plus
those halo rows.  Its own rows' outputs are then exact; the halo rows'
outputs are not used (their neighbours are incomplete) and are refreshed by
the next exchange.

The plan is computed from the full coordinate list, which every rank holds
(16 bytes a voxel); features are what is sharded.  Slabs are balanced by
voxel count using the per-plane histogram.  The exchange is point-to-point
(torch.distributed send/recv: NCCL between GPUs, gloo on the CPU) of the
boundary rows, gathered into and scattered from one contiguous buffer per
neighbour.

Local row order of a rank: its own rows (ascending global row), then the
halo rows from the rank below, then those from the rank above (each
ascending global row).  Both sides of an exchange list the same rows in the
same order, since both derive them from the same global coordinates.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np


def slab_bounds(plane_counts: np.ndarray, world: int) -> List[int]:
    """World + 1 z boundaries 0 = z_0 < z_1 < ... < z_world = Z: rank r owns
    planes [z_r, z_{r+1}).  Each slab holds at least one plane; cuts are placed
    where the running voxel count first reaches r / world of the total."""
    counts = np.asarray(plane_counts, dtype=np.int64)
    Z = counts.shape[0]
    if world < 1 or world > Z:
        raise ValueError(f"need 1 <= world <= Z (world {world}, Z {Z})")
    total = int(counts.sum())
    cum = np.cumsum(counts)
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        z = int(np.searchsorted(cum, target, side="left")) + 1  # first plane past the target
        z = max(z, bounds[-1] + 1)  # at least one plane per slab
        z = min(z, Z - (world - r))  # leave a plane for every later slab
        bounds.append(z)
    bounds.append(Z)
    return bounds


@dataclass
class SlabPlan:
    rank: int
    world: int
    bounds: List[int]
    owned: np.ndarray      # global rows of this rank's slab, ascending
    halo_lo: np.ndarray    # global rows of plane z_lo - 1 (from rank - 1), ascending
    halo_hi: np.ndarray    # global rows of plane z_hi (from rank + 1), ascending
    send_lo: np.ndarray    # local positions of this rank's plane z_lo (to rank - 1)
    send_hi: np.ndarray    # local positions of this rank's plane z_hi - 1 (to rank + 1)

    @property
    def n_owned(self) -> int:
        return int(self.owned.shape[0])

    @property
    def local_rows(self) -> np.ndarray:
        """Global row of every local row, in local order."""
        return np.concatenate([self.owned, self.halo_lo, self.halo_hi])

    @property
    def n_local(self) -> int:
        return self.n_owned + int(self.halo_lo.shape[0]) + int(self.halo_hi.shape[0])


def plan_slabs(coords, grid: Sequence[int], world: int, rank: int) -> SlabPlan:
    """The z-slab plan of `rank` for int32 [N, 4] (b, z, y, x) coordinates on
    a (Z, Y, X) grid (every batch item is split at the same planes)."""
    c = np.asarray(coords.cpu() if hasattr(coords, "cpu") else coords)
    if c.ndim != 2 or c.shape[1] != 4:
        raise ValueError("coords must be [N, 4] (b, z, y, x)")
    Z = int(grid[0])
    z = c[:, 1].astype(np.int64)
    if c.shape[0] and (z.min() < 0 or z.max() >= Z):
        raise ValueError("z outside the grid")
    bounds = slab_bounds(np.bincount(z, minlength=Z), world)
    lo, hi = bounds[rank], bounds[rank + 1]
    owned = np.flatnonzero((z >= lo) & (z < hi))
    halo_lo = np.flatnonzero(z == lo - 1) if rank > 0 else np.zeros(0, dtype=np.int64)
    halo_hi = np.flatnonzero(z == hi) if rank < world - 1 else np.zeros(0, dtype=np.int64)
    z_own = z[owned]
    send_lo = np.flatnonzero(z_own == lo) if rank > 0 else np.zeros(0, dtype=np.int64)
    send_hi = np.flatnonzero(z_own == hi - 1) if rank < world - 1 else np.zeros(0, dtype=np.int64)
    return SlabPlan(rank, world, bounds, owned, halo_lo, halo_hi, send_lo, send_hi)


def exchange_halos(plan: SlabPlan, local_feats, group=None) -> None:
    """Fill the halo rows of `local_feats` [n_local, C] (in place) with the
    neighbours' boundary rows: this rank's plane z_lo goes to rank - 1 and
    its plane z_hi - 1 to rank + 1, while the matching planes come back.
    Collective between neighbours: every rank of the group calls it."""
    import torch
    import torch.distributed as dist

    dev = local_feats.device
    n_own, n_lo = plan.n_owned, int(plan.halo_lo.shape[0])
    ops, recvs = [], []
    if plan.rank > 0:
        send = local_feats.index_select(0, torch.from_numpy(plan.send_lo).to(dev)).contiguous()
        recv = torch.empty((n_lo,) + tuple(local_feats.shape[1:]), dtype=local_feats.dtype, device=dev)
        ops += [dist.P2POp(dist.isend, send, plan.rank - 1, group),
                dist.P2POp(dist.irecv, recv, plan.rank - 1, group)]
        recvs.append((n_own, recv))
    if plan.rank < plan.world - 1:
        send = local_feats.index_select(0, torch.from_numpy(plan.send_hi).to(dev)).contiguous()
        recv = torch.empty((int(plan.halo_hi.shape[0]),) + tuple(local_feats.shape[1:]), dtype=local_feats.dtype,
                           device=dev)
        ops += [dist.P2POp(dist.isend, send, plan.rank + 1, group),
                dist.P2POp(dist.irecv, recv, plan.rank + 1, group)]
        recvs.append((n_own + n_lo, recv))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    for start, recv in recvs:
        local_feats[start:start + recv.shape[0]] = recv


class SlabConv:
    """Per-rank submanifold convs over one z-slab plus its halo: the local
    map is built once by the library; each conv first exchanges the halo
    rows, then runs on the local rows.  Outputs of the first n_owned rows are
    this rank's exact share of the global result."""

    def __init__(self, coords, grid: Sequence[int], world: int, rank: int, batch: Optional[int] = None,
                 device=None, group=None):
        import torch

        from . import _binding as B
        self.plan = plan_slabs(coords, grid, world, rank)
        self.group = group
        c = np.asarray(coords.cpu() if hasattr(coords, "cpu") else coords)
        nb = int(c[:, 0].max()) + 1 if batch is None and c.shape[0] else (batch or 1)
        self.local_coords = torch.from_numpy(np.ascontiguousarray(c[self.plan.local_rows])).to(device)
        self.map = B.build_map(self.local_coords, grid, batch=nb)

    def local_features(self, feats_global):
        """This rank's local feature rows from a global [N, C] array (the
        halo rows too; an exchange overwrites them anyway)."""
        import torch
        idx = torch.from_numpy(self.plan.local_rows).to(feats_global.device)
        return feats_global.index_select(0, idx)

    def conv(self, local_feats, weight, bias=None, **kw):
        from . import _binding as B
        exchange_halos(self.plan, local_feats, self.group)
        return B.conv(self.map, local_feats, weight, bias, **kw)
