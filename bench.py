#!/usr/bin/env python
"""Benchmark of the submanifold-convolution hot path on B200.

One *step* is one pass of the whole path over one synthetic batch: build the
neighbour map of the coordinate set (key generation and validation, hash
build, 27-lookup map, per-offset pair lists, tile schedule) and run the k=3
bf16 convolution over it (the map would then be reused by further layers).
The default workload is the pages' benchmark shape: batch 1, 128^3 grid,
128 -> 128 channels, bf16 with fp32 accumulation, union of 6 random sphere
shells (seeded synthetic data; no dataset is involved).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  ``value`` is active voxels per second of the
whole step (device-timed with CUDA events, L2 flushed before every step,
max over ranks); the line also carries the conv's pair-TFLOP/s, the map
build's GB/s, the roofline of the dominant kernel, an end-to-end figure
through the public API with host buffers, the CPU oracle's throughput on a
bounded sample, and the SM clocks seen during the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from submanifold_sparse_convolution_packed_b200 import synth as S  # noqa: E402

METRIC = "SubMConv3d k=3 Mvoxels/s & pair-TFLOP/s @128^3/128ch bf16; map-build GB/s"
UNIT = "Mvoxels/s"
L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
CONV_SRC = os.path.join(ROOT, "submanifold_sparse_convolution_packed_b200", "csrc", "conv_tc.cu")


# ---------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world: int, backend: str, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity on one rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def source_sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region (samples
    go to a temporary file that is removed when sampling stops)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.id = str(device_index)
        fd, self.path = tempfile.mkstemp(prefix=f"smc_clocks_{device_index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        """Start sampling every 20 ms and wait (at most 3 s) for the first
        sample, so that a short timed region that follows is covered."""
        self.mark_at = 0
        self.end_at = None
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.id}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 3.0 and not self._rows():
            time.sleep(0.01)

    def mark(self):
        """The timed region starts now: later samples are the ones reported."""
        self.mark_at = len(self._rows())

    def mark_end(self):
        """The timed region ended now; samples taken after this belong to the
        window of the same work that may follow it."""
        self.end_at = len(self._rows())

    def region_samples(self) -> int:
        return max(0, (self.end_at if self.end_at is not None else len(self._rows())) - self.mark_at)

    def _rows(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        rows.append(parts)
        except OSError:
            pass
        return rows

    def stop(self, window_note=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = self._rows()
        try:
            os.remove(self.path)
        except OSError:
            pass
        return self.summary(rows, self.mark_at, self.end_at, window_note)

    @staticmethod
    def summary(all_rows, mark_at, end_at=None, window_note=None):
        """Median SM clock, max clock and throttle reasons of the samples
        taken in the timed region (from mark_at to end_at) and, when a window
        of the same work followed it (window_note), of that window too; with
        neither, the last sample before the region, flagged."""
        end = len(all_rows) if end_at is None else end_at
        region = all_rows[mark_at:end]
        window = all_rows[end:] if (end_at is not None and window_note) else []
        rows = region + window
        before = False
        if not rows and all_rows:
            rows, before = all_rows[max(0, mark_at - 1):mark_at] or all_rows[-1:], True
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
               "samples": 0 if before else len(region), "reasons": sorted(reasons)}
        if window:
            out["window_samples"] = len(window)
            out["window"] = window_note
        if before:
            out["note"] = "timed region shorter than the sampling interval: the last sample before it"
        return out


def tap_efficiency(perm: np.ndarray, nbr: np.ndarray, tile: int = 128) -> float:
    """Pairs / (taps issued x 128) of the tensor-core conv's tile schedule."""
    n = len(perm)
    hits = (nbr >= 0)
    pairs = int(hits.sum())
    issued = 0
    for t0 in range(0, n, tile):
        issued += int(hits[perm[t0:t0 + tile]].any(axis=0).sum()) * tile
    return pairs / issued if issued else 0.0


# ------------------------------------------------------------- workloads
def get_workload(name: str) -> S.Workload:
    return S.workload(name)


def algorithmic_map_bytes(n: int, p: int) -> int:
    """coords read (16 B) + map written (108 B) per voxel + pairs written (8 B)."""
    return 16 * n + 108 * n + 8 * p


def pair_flops(p: int, cin: int, cout: int) -> float:
    return 2.0 * p * cin * cout


# ------------------------------------------------------------- GPU arm
STEP_VARIANT = 0  # tensor-core conv variant of the timed steps (0: the library's choice)


def conv_variant_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, w_d, b_d, out_d, reps=5):
    """Median device time (ms) of one conv with each tensor-core variant on
    the bench's map, L2 flushed before each: the fused 27-tap kernel (the
    step's), and the per-offset gather-GEMM-scatter over the pair lists, the
    comparator the pages measure against.  Untimed for the bench value."""
    m = smc.build_map(coords_d, w.grid, batch=batch, stream=stream)
    res = {}
    try:
        for name, v in (("fused", STEP_VARIANT), ("per_offset", 3)):
            smc.set_conv_variant(v)
            ts = []
            for _ in range(reps + 1):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                smc.conv(m, feats_d, w_d, b_d, ksize=3, orientation=1, out=out_d, stream=stream)
                e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1))
            res[name] = round(float(np.median(ts[1:])), 4)
    finally:
        smc.set_conv_variant(STEP_VARIANT)
        m.free()
    smc.status(stream)
    res["fused_speedup"] = round(res["per_offset"] / res["fused"], 2)
    return res


def epilogue_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, w_d, b_d, out_d, reps=5):
    """Median device time (ms) of one conv on the bench's map: plain; with
    SiLU and a residual (smc_conv_ex: the conv, then one row pass that applies
    them in row order); the same plus the GroupNorm-32 statistics of the
    output (in the same row pass); the same SiLU and residual done inside the
    conv's epilogue instead (smc_set_conv_epilogue(1)); and plain followed by
    a statistics pass.  Untimed for the bench value."""
    m = smc.build_map(coords_d, w.grid, batch=batch, stream=stream)
    residual = torch.randn(out_d.shape, device=out_d.device).to(out_d.dtype)
    stats = torch.zeros((batch, 32, 3), dtype=torch.float64, device=out_d.device)
    silu_res = lambda: smc.conv(m, feats_d, w_d, b_d, out=out_d, stream=stream, residual=residual, act="silu")
    runs = {
        "plain": (0, lambda: smc.conv(m, feats_d, w_d, b_d, out=out_d, stream=stream)),
        "silu_residual": (0, silu_res),
        "silu_residual_with_stats": (0, lambda: smc.conv(m, feats_d, w_d, b_d, out=out_d, stream=stream,
                                                         residual=residual, act="silu", coords=coords_d,
                                                         stats=stats, groups=32)),
        "silu_residual_in_conv_epilogue": (1, silu_res),
        "plain_then_stats_pass": (0, lambda: (smc.conv(m, feats_d, w_d, b_d, out=out_d, stream=stream),
                                              smc.group_stats(out_d, coords_d, batch, 32, stats, stream=stream))),
    }
    res = {}
    try:
        for name, (where, fn) in runs.items():
            smc.set_conv_epilogue(where)
            ts = []
            for _ in range(reps + 1):
                flush.zero_()
                stats.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1))
            res[name] = round(float(np.median(ts[1:])), 4)
    finally:
        smc.set_conv_epilogue(0)
    m.free()
    smc.status(stream)
    return res


def subdivide_times(smc, torch, stream, flush, reps=5):
    """Median device time (ms) of one decoder step's map, stage 2 -> 3 of the
    decoder chain (children inside the next shell kept): built from the parent
    map by smc_subdivide (including its host read of the child count), and
    built from scratch from the same child coordinates.  The maps are equal
    (tested); untimed for the bench value."""
    w2, w3 = S.workload("decoder2"), S.workload("decoder3")
    keep = torch.from_numpy(S.subdivision_keep_mask(w2.coords, w3.coords, w3.grid)).cuda()
    pc = torch.from_numpy(w2.coords).cuda()
    parent = smc.build_map(pc, w2.grid, batch=1, stream=stream)
    inc, full = [], []
    for _ in range(reps + 1):
        flush.zero_()
        e0, e1, e2, e3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
        e0.record(stream)
        kids, child = smc.subdivide(parent, pc, keep, stream=stream)
        child.stream_wait(stream)
        e1.record(stream)
        flush.zero_()
        e2.record(stream)
        again = smc.build_map(kids, child.grid, batch=1, stream=stream, sync=False)
        again.stream_wait(stream)
        e3.record(stream)
        e3.synchronize()
        child.wait()
        again.wait()
        inc.append(e0.elapsed_time(e1))
        full.append(e2.elapsed_time(e3))
        child.free()
        again.free()
    parent.free()
    smc.status(stream)
    return {"workload": f"decoder stage 2 -> 3: {w2.n} voxels on {w2.grid[0]}^3 -> {int(keep.sum())} on {w3.grid[0]}^3",
            "incremental": round(float(np.median(inc[1:])), 4), "full_build": round(float(np.median(full[1:])), 4)}


def resample_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, peaks, reps=5):
    """Median device time (ms) of the pooling and expansion calls on the
    bench's voxels and features (bf16, Cin channels), each call whole
    (scratch clears, all kernels, its host read of the count):
    smc_downsample (max and mean) and smc_upsample of the parents with the
    recorded mask, their features and the parents' map (child map included).
    GB/s counts the algorithmic bytes of each call: coordinates, features,
    mask and parent index read or written once.  Untimed for the bench value."""
    c, es, n = feats_d.shape[1], feats_d.element_size(), w.n
    out = {}
    for mode in ("max", "mean"):
        ts = []
        for _ in range(reps + 1):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            pc, pooled, mask, parent = smc.downsample(coords_d, w.grid, feats_d, mode, batch=batch, stream=stream)
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = float(np.median(ts[1:]))
        m = pc.shape[0]
        nbytes = 16 * n + n * c * es + 16 * m + 8 * m + 4 * n + m * c * es
        out[f"downsample_{mode}"] = {"ms": round(ms, 4), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    half = tuple((g + 1) // 2 for g in w.grid)
    pm = smc.build_map(pc, half, batch=batch, stream=stream)
    ts = []
    for _ in range(reps + 1):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kids, kf, child = smc.upsample(pc, mask, pooled, parent=pm, stream=stream)
        child.stream_wait(stream)
        e1.record(stream)
        e1.synchronize()
        child.wait()
        child.free()
        ts.append(e0.elapsed_time(e1))
    pm.free()
    ms = float(np.median(ts[1:]))
    k = kids.shape[0]
    nbytes = 16 * m + 8 * m + m * c * es + 16 * k + k * c * es
    out["upsample_with_child_map"] = {"ms": round(ms, 4), "gbs_features_and_coords": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    out["sizes"] = {"rows": n, "parents": m, "children": k, "channels": c, "dtype": str(feats_d.dtype).replace("torch.", "")}
    out["hbm_peak_gbs"] = peaks["hbm_gbs"]
    smc.status(stream)
    return out


L2_BYTES = 126 << 20  # B200 L2
PIPE_STREAMS = 2       # streams the timed steps alternate over


def input_sets(torch, dev, w, f, tdt, min_sets=2, max_sets=8):
    """Copies of one step's inputs (coordinates, features) and output buffer,
    enough that the copies together hold at least 3x the L2 size, so that a
    step finds none of its inputs in L2 from earlier steps without a flush."""
    per = w.n * (16 + 2 * w.cin + 2 * w.cout)
    k = max(min_sets, min(max_sets, -(-3 * L2_BYTES // per)))
    coords = torch.from_numpy(w.coords)
    feats = torch.from_numpy(f).to(tdt)
    return [(coords.to(dev, copy=True), feats.to(dev, copy=True), torch.empty((w.n, w.cout), dtype=tdt, device=dev))
            for _ in range(k)]


class StepRunner:
    """Steps enqueued up to DEPTH per stream ahead of the host, as a job would run them:
    each step is the asynchronous map build and the conv behind it, on one of
    `streams` in turn and on the next of the input `sets`, bracketed by its
    own CUDA events on its stream.  With `flush`, an L2 flush precedes every
    step on its stream (outside its events).  A step is retired DEPTH steps
    later: its map's outcome is checked, its event times are read and the map
    is freed (stream-ordered)."""
    DEPTH = 3

    def __init__(self, smc, torch, streams, flush, sets, grid, batch, w_d, b_d, profile=False, step_events=True):
        self.smc, self.torch, self.streams, self.flush = smc, torch, list(streams), flush
        self.step_events = step_events  # events around whole steps (else around the conv only)
        self.depth = self.DEPTH * len(self.streams)
        self.sets, self.grid, self.batch, self.w_d, self.b_d = sets, grid, batch, w_d, b_d
        self.profile = profile  # read the library's per-phase timing of each build
        self.pending = []
        self.count = 0
        self.times, self.conv_times, self.map_times = [], [], []

    def submit(self):
        torch, smc = self.torch, self.smc
        stream = self.streams[self.count % len(self.streams)]
        coords_d, feats_d, out_d = self.sets[self.count % len(self.sets)]
        self.count += 1
        if self.flush is not None:
            with torch.cuda.stream(stream):
                self.flush.zero_()
        e0, e2 = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) \
            if self.step_events else (None, None)
        e1, ec = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if e0 is not None:
            e0.record(stream)
        m = smc.build_map(coords_d, self.grid, batch=self.batch, stream=stream, sync=False)
        e1.record(stream)
        smc.conv(m, feats_d, self.w_d, self.b_d, ksize=3, orientation=1, out=out_d, stream=stream)
        ec.record(stream)
        m.stream_wait(stream)  # the step ends when the whole build (pair lists too) is done
        if e2 is not None:
            e2.record(stream)
        self.pending.append((e0, e1, ec, e2, m))
        if len(self.pending) > self.depth:
            self.retire()

    def retire(self):
        e0, e1, ec, e2, m = self.pending.pop(0)
        m.wait()  # the whole build is done (raises if it failed on the device)
        ec.synchronize()
        if e2 is not None:
            e2.synchronize()
            self.times.append(e0.elapsed_time(e2))
        self.conv_times.append(e1.elapsed_time(ec))
        if self.profile:
            self.map_times.append(m.timing())
        m.free()

    def drain(self):
        while self.pending:
            self.retire()


def prime_pool(smc, sets, grid, batch, streams, count):
    """Builds `count` maps at once over the streams and frees them, so that
    the library's memory pool already holds what the pipelined steps keep in
    flight (set-up, not a step: no conv runs)."""
    maps = [smc.build_map(sets[i % len(sets)][0], grid, batch=batch, stream=streams[i % len(streams)], sync=False)
            for i in range(count)]
    for m in maps:
        m.wait()
    for m in maps:
        m.free()


def timed_steps(torch, runner, steps):
    """Device time (ms) of `steps` steps of `runner` from the first one's
    start to the end of the last one, on every stream: an event on the first
    stream that the others wait for, and a join of all streams at the end."""
    s0 = runner.streams[0]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s0)
    for s in runner.streams[1:]:
        s.wait_event(start)
    for _ in range(steps):
        runner.submit()
    for s in runner.streams[1:]:
        ev = torch.cuda.Event()
        ev.record(s)
        s0.wait_event(ev)
    end.record(s0)
    runner.drain()
    end.synchronize()
    return start.elapsed_time(end)


def conv_alone_times(smc, torch, stream, flush, m, feats_d, w_d, b_d, out_d, reps=10):
    """Median device time (ms) of one conv on a built map, with L2 flushed
    before it (flushed) and right after an identical conv (L2 warm: the
    features, weights and map it reads are where the previous one left them).
    Each conv is queued behind device work, so no host latency is timed."""
    cold, warm = [], []
    for _ in range(reps + 1):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        smc.conv(m, feats_d, w_d, b_d, ksize=3, orientation=1, out=out_d, stream=stream)
        ev[1].record(stream)
        ev[2].record(stream)
        smc.conv(m, feats_d, w_d, b_d, ksize=3, orientation=1, out=out_d, stream=stream)
        ev[3].record(stream)
        ev[3].synchronize()
        cold.append(ev[0].elapsed_time(ev[1]))
        warm.append(ev[2].elapsed_time(ev[3]))
    smc.status(stream)
    return float(np.median(cold[1:])), float(np.median(warm[1:]))


def measure_config(smc, torch, stream, flush, dev, peaks, name, dtype, steps, world, wl=None):
    """One workload measured the way the headline is: pipelined steps (build +
    conv, alternating over two streams, inputs rotated over copies larger
    than L2) for throughput; the same steps one at a time with L2 flushed
    before each for latency; the conv alone flushed and L2-warm; and the map
    phases from the library's own events; with the SM clocks sampled while
    the pipelined steps run.  Returns a sub-record for the bench line."""
    w = wl if wl is not None else get_workload(name)
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    f, wt, b = S.layer_tensors(w, dtype)
    sets = input_sets(torch, dev, w, f, tdt)
    w_d = torch.from_numpy(wt).to(tdt).to(dev)
    b_d = torch.from_numpy(b).to(tdt).to(dev)
    batch = int(w.coords[:, 0].max()) + 1
    del f
    streams = [stream] + [torch.cuda.Stream(dev) for _ in range(PIPE_STREAMS - 1)]
    mk = lambda st, fl, profile=False: StepRunner(smc, torch, st, fl, sets, w.grid, batch, w_d, b_d, profile=profile,
                                                  step_events=len(st) == 1)
    # latency: one step at a time on one stream, L2 flushed before each
    lat = mk([stream], flush)
    for _ in range(3):
        lat.submit()
    lat.drain()
    lat.times.clear()
    lat.conv_times.clear()
    for _ in range(steps):
        lat.submit()
    lat.drain()
    latency = float(np.median(lat.times))
    # throughput: pipelined steps, at least 0.3 s of them
    prime_pool(smc, sets, w.grid, batch, streams, StepRunner.DEPTH * len(streams) + 2)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    warm = mk(streams, None)
    for _ in range(2 * StepRunner.DEPTH):
        warm.submit()
    warm.drain()
    n_steps = max(steps, int(0.3 / (latency * 1e-3)))
    clocks.mark()
    run = mk(streams, None)
    total = timed_steps(torch, run, n_steps)
    clocks.mark_end()
    clk = clocks.stop()
    prof = mk([stream], flush, profile=True)
    smc.set_profiling(True)
    for _ in range(min(steps, 20)):
        prof.submit()
    prof.drain()
    smc.set_profiling(False)
    coords_d, feats_d, out_d = sets[0]
    m = smc.build_map(coords_d, w.grid, batch=batch, stream=stream)
    P = m.pairs_total
    conv_cold, conv_warm = conv_alone_times(smc, torch, stream, flush, m, feats_d, w_d, b_d, out_d)
    m.free()
    step_ms = reduce_max(total / n_steps, world, dev)
    latency_ms = reduce_max(latency, world, dev)
    conv_ms = reduce_max(float(np.mean(run.conv_times)), world, dev)
    look = reduce_max(float(np.median([t[0] for t in prof.map_times])), world, dev)
    sched = reduce_max(float(np.median([t[1] for t in prof.map_times])), world, dev)
    pairs_ms = reduce_max(float(np.median([t[2] for t in prof.map_times])), world, dev)
    flops = pair_flops(P, w.cin, w.cout)
    map_bytes = algorithmic_map_bytes(w.n, P)
    tfl = flops / (conv_ms * 1e-3) / 1e12
    gbs = map_bytes / ((look + pairs_ms) * 1e-3) / 1e9
    pk = peaks["bf16_tflops"]
    rec = {
        "workload": f"{w.name}: {w.note}", "dtype": dtype, "n_voxels": w.n, "pairs": P,
        "steps_timed": n_steps, "step_ms": round(step_ms, 4),
        "mvoxels_per_s": round(world * w.n / (step_ms * 1e-3) / 1e6, 2),
        "step_latency_ms": round(latency_ms, 4),
        "input_sets": len(sets),
        "conv_ms": round(conv_ms, 4), "conv_ms_alone_l2_flushed": round(conv_cold, 4),
        "conv_ms_alone_l2_warm": round(conv_warm, 4),
        "conv_roofline": {"bound": "tensor", "achieved": round(tfl, 2), "peak": pk,
                          "unit": "TFLOP/s", "frac": round(tfl / pk, 4),
                          "frac_alone_l2_flushed": round(flops / (conv_cold * 1e-3) / 1e12 / pk, 4),
                          "frac_l2_warm": round(flops / (conv_warm * 1e-3) / 1e12 / pk, 4)},
        "map_ms": {"clears_and_lookups": round(look, 4), "tile_schedule": round(sched, 4),
                   "pair_lists_side_stream": round(pairs_ms, 4)},
        "map_roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes": map_bytes},
    }
    if clk is not None:
        rec["clocks"] = clk
    del sets, feats_d, out_d, coords_d
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    import torch

    import submanifold_sparse_convolution_packed_b200 as smc

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    smc.lib()
    if args.schedule_segment is not None:
        smc.set_schedule_segment(args.schedule_segment)
    if args.conv_variant is not None:
        global STEP_VARIANT
        STEP_VARIANT = args.conv_variant
        smc.set_conv_variant(args.conv_variant)
    peaks = load_peaks()

    w = get_workload(args.workload)
    dtype = "f16" if "f16" in w.dtypes and "bf16" not in w.dtypes else "bf16"
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    f, wt, b = S.layer_tensors(w, dtype)
    sets = input_sets(torch, dev, w, f, tdt)
    coords_d, feats_d, out_d = sets[0]
    w_d = torch.from_numpy(wt).to(tdt).to(dev)
    b_d = torch.from_numpy(b).to(tdt).to(dev)
    batch = int(w.coords[:, 0].max()) + 1
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    streams = [stream] + [torch.cuda.Stream(dev) for _ in range(PIPE_STREAMS - 1)]
    runner = lambda st, fl, profile=False: StepRunner(smc, torch, st, fl, sets, w.grid, batch, w_d, b_d,
                                                      profile=profile, step_events=len(st) == 1)

    smc.set_profiling(False)  # the timed steps carry no instrumentation

    prime_pool(smc, sets, w.grid, batch, streams, StepRunner.DEPTH * len(streams) + 2)
    # reference of the schedule quality (host-side, untimed)
    m0 = smc.build_map(coords_d, w.grid, batch=batch, stream=stream)
    P = m0.pairs_total
    eff = tap_efficiency(m0.schedule().cpu().numpy(), m0.nbr().cpu().numpy())
    m0.free()
    # the clock sampler starts before the warm-up, so that the timed region
    # follows the warm-up steps directly (only its own samples are reported)
    clocks = ClockSampler(local)
    clocks.start()
    # warm-up: W pipelined steps
    warm = runner(streams, None)
    for _ in range(args.warmup):
        warm.submit()
    warm.drain()
    smc.status(stream)

    # the timed region: K steps, alternating over the streams, each on the
    # next copy of the inputs (together more than 3x L2, so no flush)
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    t_wall0 = time.perf_counter()
    launches_before = smc.kernel_launches()
    run = runner(streams, None)
    total_ms = timed_steps(torch, run, args.steps)
    torch.cuda.synchronize()
    times, conv_times = run.times, run.conv_times
    launches = smc.kernel_launches() - launches_before
    wall = time.perf_counter() - t_wall0
    clocks.mark_end()
    # A timed region shorter than a few sampling intervals gets the same
    # steps repeated right after it, untimed, so that the clock record has
    # samples of this work under load.
    window_note = None
    if clocks.region_samples() < 5:
        tw = time.perf_counter()
        extra = runner(streams, None)
        while time.perf_counter() - tw < 0.4:
            extra.submit()
        extra.drain()
        window_note = (f"the same steps repeated untimed for {1e3 * (time.perf_counter() - tw):.0f} ms right "
                       f"after the timed region ({len(extra.conv_times)} steps)")
    clk = clocks.stop(window_note)
    barrier(world)
    smc.status(stream)
    # latency: the same steps one at a time on one stream, L2 flushed before each
    lat = runner([stream], flush)
    for _ in range(min(args.steps, 200)):
        lat.submit()
    lat.drain()
    lat_times = lat.times
    # per-phase breakdown of the build from a separate, untimed pass with the
    # library's own CUDA events on (one stream, L2 flushed before each step)
    smc.set_profiling(True)
    prof = runner([stream], flush, profile=True)
    for _ in range(min(args.steps, 50)):
        prof.submit()
    prof.drain()
    smc.set_profiling(False)
    map_times = prof.map_times
    m1 = smc.build_map(coords_d, w.grid, batch=batch, stream=stream)
    conv_cold, conv_warm = conv_alone_times(smc, torch, stream, flush, m1, feats_d, w_d, b_d, out_d)
    m1.free()
    variants = conv_variant_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, w_d, b_d, out_d)
    subdiv = subdivide_times(smc, torch, stream, flush)
    epilogue = epilogue_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, w_d, b_d, out_d)
    resample = resample_times(smc, torch, stream, flush, coords_d, w, batch, feats_d, peaks)

    total_ms = reduce_max(total_ms, world, dev)
    conv_ms = reduce_max(sum(conv_times) / len(conv_times), world, dev)
    look_ms = reduce_max(sum(t[0] for t in map_times) / len(map_times), world, dev)
    sched_ms = reduce_max(sum(t[1] for t in map_times) / len(map_times), world, dev)
    pairs_ms = reduce_max(sum(t[2] for t in map_times) / len(map_times), world, dev)
    mapk_ms = look_ms + pairs_ms  # the kernels that move the map's bytes
    ms_per_step = total_ms / args.steps
    value = world * w.n * args.steps / (total_ms * 1e-3) / 1e6
    flops = pair_flops(P, w.cin, w.cout)
    conv_tflops = flops / (conv_ms * 1e-3) / 1e12
    map_bytes = algorithmic_map_bytes(w.n, P)
    map_gbs = map_bytes / (mapk_ms * 1e-3) / 1e9

    # traffic of the conv kernel from the committed ncu capture, if still current
    traffic = None
    if os.path.exists(PROFILE_TRAFFIC):
        with open(PROFILE_TRAFFIC) as fh:
            tr = json.load(fh).get("conv_tc", {})
        if tr.get("source_sha") == source_sha(CONV_SRC) and tr.get("workload") == w.name:
            traffic = tr.get("dram_bytes_per_launch")

    # end to end through the public API: pinned host inputs in, result out
    e2e = run_e2e(w, f, wt, b, batch, dev, stream, args, tdt)
    e2e_v = reduce_max(e2e["ms"], world, dev)

    # the other configurations of the metric, measured the same way
    configs = {}
    if not args.skip_configs and args.workload == "shells6":
        del f
        for name, dtype in (("shells6_118k", "bf16"), ("full128", "bf16"), ("varlen4", "f16"), ("decoder3", "bf16")):
            configs[name] = measure_config(smc, torch, stream, flush, dev, peaks, name, dtype, 10, world)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = run_cpu_baseline(w, *S.layer_tensors(w, dtype), budget_s=args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded union of 6 sphere shells; random-init KRSC weights)",
            "config": {
                "workload": f"{w.name}: {w.note}", "n_voxels": w.n, "pairs": P, "grid": list(w.grid),
                "cin": w.cin, "cout": w.cout,
                "step": ("build_map (asynchronous entry point) + conv k=3 s=+1; steps alternate over "
                         f"{PIPE_STREAMS} streams, up to {StepRunner.DEPTH} per stream enqueued ahead, so one step's map build "
                         "overlaps the previous step's conv; every map checked and freed when its step retires; "
                         "value and ms_per_step from the device time of all K steps (first start to last end)"),
                "l2": (f"no flush: steps rotate over {len(sets)} copies of their inputs and outputs "
                       f"({len(sets) * w.n * (16 + 2 * w.cin + 2 * w.cout) / 1e6:.0f} MB, > 3x the 126 MB L2); "
                       "step_latency_ms: one step at a time on one stream, L2 flushed (256 MB write) before each"),
                "parallelism": f"replicas x{world} (no collective on the data path)",
                **({"schedule_segment_rows": args.schedule_segment} if args.schedule_segment is not None else {}),
                **({"conv_variant": args.conv_variant} if args.conv_variant is not None else {}),
            },
            "pair_tflops": round(conv_tflops, 2),
            "map_build_gbs": round(map_gbs, 1),
            "breakdown_ms": {"step": round(ms_per_step, 4), "map_clears_and_lookups": round(look_ms, 4),
                             "tile_schedule": round(sched_ms, 4),
                             "pair_lists_side_stream": round(pairs_ms, 4), "conv": round(conv_ms, 4)},
            "step_latency_ms": {q: round(float(np.quantile(lat_times, v)), 4)
                                for q, v in (("p50", 0.5), ("p90", 0.9), ("p99", 0.99), ("max", 1.0))},
            "conv_alone_ms": {"l2_flushed": round(conv_cold, 4), "l2_warm": round(conv_warm, 4)},
            "conv_mvoxels_per_s": round(w.n / (conv_ms * 1e-3) / 1e6, 2),
            "conv_tap_efficiency": round(eff, 4),
            "conv_variants_ms": variants,
            "subdivide_map_ms": subdiv,
            "conv_epilogue_ms": epilogue,
            "resample": resample,
            "roofline": {"kernel": "k_conv_tc", "bound": "tensor", "achieved": round(conv_tflops, 2),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(conv_tflops / peaks["bf16_tflops"], 4), "traffic": traffic,
                         "frac_alone_l2_flushed": round(flops / (conv_cold * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                         "frac_l2_warm": round(flops / (conv_warm * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                         "peak_source": f"{peaks['source']} bf16 burst (kernel timed alone)",
                         "algorithmic": "2 * pairs * Cin * Cout per launch",
                         "duration": "mean launch time over the timed region (events on its stream, next to the "
                                     "other stream's map build)"},
            "map_roofline": {"kernels": "clears, k_insert, k_neighbours, pair-list scan, k_pairs (time = clears and lookups + pair lists)",
                             "bound": "hbm", "achieved": round(map_gbs, 1),
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": round(map_gbs / peaks["hbm_gbs"], 4),
                             "algorithmic": "16N coords + 108N map + 8P pairs"},
            "configs": configs,
            "e2e": {"value": round(world * w.n / (e2e_v * 1e-3) / 1e6, 3), "unit": UNIT,
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": round(e2e_v, 4)},
            "gpu_launches": int(launches),
            "launches_per_step": launches / args.steps,
            "wall_s": round(wall, 3),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if clk is not None:
            line["clocks"] = clk
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(w, f, wt, b, batch, dev, stream, args, tdt=None):
    """Same step through the public API, with each step's inputs copied from
    pinned host memory and its result copied back inside the timed region.
    Steps are pipelined the way a serving loop runs them: inputs go up on a
    copy stream, the build and the conv run on the compute stream, the result
    comes back on a second copy stream, and two device slots let step k's
    copy-back overlap step k+1's upload and compute.  Timed from the first
    upload to the last copy-back, on the device; ms = that time / steps."""
    import torch

    import submanifold_sparse_convolution_packed_b200 as smc
    tdt = tdt or torch.bfloat16
    coords_h = torch.from_numpy(w.coords).pin_memory()
    feats_h = torch.from_numpy(f).to(tdt).pin_memory()
    w_h = torch.from_numpy(wt).to(tdt).pin_memory()
    b_h = torch.from_numpy(b).to(tdt).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (coords_h, feats_h, w_h, b_h))
    depth = 2
    outs_h = [torch.empty((w.n, w.cout), dtype=tdt).pin_memory() for _ in range(depth)]
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    slots = [dict(c=torch.empty_like(coords_h, device=dev), x=torch.empty_like(feats_h, device=dev),
                  w=torch.empty_like(w_h, device=dev), b=torch.empty_like(b_h, device=dev),
                  y=torch.empty((w.n, w.cout), dtype=tdt, device=dev)) for _ in range(depth)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    inputs_free = [None] * depth   # compute consumed the slot's inputs
    output_free = [None] * depth   # copy-back of the slot's output done
    maps = []

    def step(i):
        k = i % depth
        sl = slots[k]
        with torch.cuda.stream(up):
            if inputs_free[k] is not None:
                up.wait_event(inputs_free[k])
            for name, src in (("c", coords_h), ("x", feats_h), ("w", w_h), ("b", b_h)):
                sl[name].copy_(src, non_blocking=True)
            ready = ev()
            ready.record(up)
        stream.wait_event(ready)
        if output_free[k] is not None:
            stream.wait_event(output_free[k])
        m = smc.build_map(sl["c"], w.grid, batch=batch, stream=stream, sync=False)
        smc.conv(m, sl["x"], sl["w"], sl["b"], ksize=3, orientation=1, out=sl["y"], stream=stream)
        done = ev()
        done.record(stream)
        inputs_free[k] = done
        with torch.cuda.stream(down):
            down.wait_event(done)
            outs_h[k].copy_(sl["y"], non_blocking=True)
            back = ev()
            back.record(down)
        output_free[k] = back
        maps.append((m, back))
        while len(maps) > depth:  # retire old steps: check the build, free its map
            old, e = maps.pop(0)
            e.synchronize()
            old.wait()
            old.free()

    n = max(3, min(args.steps, 50))
    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(3, 3 + n):
        step(i)
    down.wait_stream(stream)
    e1.record(down)
    e1.synchronize()
    for m, e in maps:
        e.synchronize()
        m.wait()
        m.free()
    torch.cuda.synchronize(dev)
    return {"ms": e0.elapsed_time(e1) / n, "h2d": h2d, "d2h": d2h}


# ------------------------------------------------------------- CPU oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def _oracle_rate(w, f, wt, b, budget_s: float, threads: int):
    """Voxels/s of the oracle on a bounded sample: the full neighbour map plus
    the conv on seeded batches of output rows until about budget_s / 2 of
    conv time; returns (rate, description)."""
    from oracle import oracle
    t0 = time.perf_counter()
    oracle.neighbour_map(w.coords, w.grid)
    t_map = time.perf_counter() - t0
    rows_n = min(w.n, 2048 if threads > 1 else 256)
    rng = np.random.default_rng(0)
    t_conv, done = 0.0, 0
    while t_conv < budget_s * 0.5 and done < w.n:
        rows = np.sort(rng.choice(w.n, size=rows_n, replace=False))
        t1 = time.perf_counter()
        oracle.conv(w.coords, w.grid, f, wt, b, 3, 1, rows=rows, threads=threads)
        t_conv += time.perf_counter() - t1
        done += rows_n
    per_voxel = t_map / w.n + t_conv / done
    return 1.0 / per_voxel, (f"map over all {w.n} voxels ({t_map:.2f} s) + fp64 conv on {done} seeded rows "
                             f"({t_conv:.2f} s, {threads} thread{'s' if threads > 1 else ''}), per-voxel cost "
                             f"scaled to the metric")


def run_cpu_baseline(w, f, wt, b, budget_s: float = 20.0, single: bool = True):
    """The CPU oracle, as it stands, on a bounded sample of the same workload,
    on all host cores (the reported figure) and, when `single`, on one thread
    too; the host's CPU model and core count are recorded beside them."""
    threads = os.cpu_count() or 1
    budget_all = budget_s * (0.6 if single else 1.0)
    rate, desc = _oracle_rate(w, f, wt, b, budget_all, threads)
    out = {"value": round(rate / 1e6, 6), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
           "cpu_model": cpu_model(), "nproc": threads}
    if single:
        r1, d1 = _oracle_rate(w, f, wt, b, budget_s - budget_all, 1)
        out["single_thread"] = {"value": round(r1 / 1e6, 6), "unit": UNIT, "cores": 1, "sample": d1}
    return out


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores (the pages
    ship no runnable implementation of this path); rank 0 only.  Each step is
    a bounded sample (full map + conv on seeded rows), sized so that the whole
    run stays within a few minutes; steps that would not fit are not run and
    the line reports the steps actually timed."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = get_workload(args.workload)
    f, wt, b = S.layer_tensors(w, "bf16")
    per_step = max(1.0, min(args.cpu_seconds, 150.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        run_cpu_baseline(w, f, wt, b, budget_s=min(per_step, 2.0), single=False)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(run_cpu_baseline(w, f, wt, b, budget_s=per_step, single=False))
        if time.perf_counter() - t0 > 180.0:
            break
    elapsed = time.perf_counter() - t0
    value = statistics.median(v["value"] for v in vals)
    ms = w.n / (value * 1e6) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": len(vals),
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{w.name}: {w.note}", "n_voxels": w.n},
        "cpu_baseline": vals[-1],
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(elapsed, 2),
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="shells6",
                    help="shells6 (default), full128, varlen4, shell2, decoder0..decoder3")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--conv-variant", type=int, default=None,
                    help="tensor-core conv variant for the step's conv (smc_set_conv_variant; default: the "
                         "library's choice)")
    ap.add_argument("--schedule-segment", type=int, default=None,
                    help="sort the tile schedule within segments of this many rows (0 = whole map; default: "
                         "the library's default)")
    ap.add_argument("--skip-configs", action="store_true",
                    help="measure the default workload only, not the other configurations")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
