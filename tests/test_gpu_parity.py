"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Every case draws seeded inputs from ``synth`` and feeds the same values to
both sides.  Bars:
* neighbour map, pair lists: bit-exact;
* fp32 conv: max|gpu - oracle| <= 1e-5 * max|oracle|;
* bf16 / fp16 conv: max|gpu - oracle| <= 5e-3 * max|oracle|, the oracle run
  in fp64 on the identically rounded inputs;
* small-integer inputs: bit-exact in every dtype.
Large workloads are checked on a seeded sample of output rows.
"""
import os

import numpy as np
import pytest
import torch

import submanifold_sparse_convolution_packed_b200 as smc
from submanifold_sparse_convolution_packed_b200 import synth as S

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
TOL = {"f32": 1e-5, "bf16": 5e-3, "f16": 5e-3}
THREADS = min(32, os.cpu_count() or 1)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    smc.lib()
    yield
    smc.clear_cache()


_WL = {}


def workload(name):
    if name not in _WL:
        _WL[name] = S.workload(name)
    return _WL[name]


def dev(x, dtype="f32"):
    return torch.from_numpy(np.ascontiguousarray(x)).to(TORCH_DT[dtype]).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def build(w, **kw):
    coords = torch.from_numpy(w.coords).cuda()
    batch = int(w.coords[:, 0].max()) + 1 if w.n else 1
    return smc.build_map(coords, w.grid, batch=batch, **kw)


def check_close(got, ref, dtype, what=""):
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    assert err <= TOL[dtype] * scale, f"{what}: max err {err:.3e} vs bound {TOL[dtype] * scale:.3e}"


@pytest.fixture(params=[1, 2, 3, 4], ids=["one_cta", "cta_pair", "per_offset", "two_tiles"])
def conv_variant(request):
    """Runs a test on each tensor-core conv: the fused 27-tap kernel with one
    CTA per 128-row tile, the same with CTA pairs sharing M = 256 MMAs, the
    per-offset gather-GEMM-scatter over the pair lists, and the fused kernel
    with two tiles per CTA sharing each weight stage."""
    smc.set_conv_variant(request.param)
    yield request.param
    smc.set_conv_variant(0)


def sample_rows(n, k, seed):
    if n <= k:
        return None
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False))


# ------------------------------------------------------------------ map
@pytest.fixture(params=[1, 2, 3], ids=["hash", "dense_grid", "dense_occupancy"])
def map_lookup(request):
    """Runs a test with each lookup structure of the map build."""
    smc.set_map_lookup(request.param)
    yield request.param
    smc.set_map_lookup(0)


# The tile order of the tensor-core conv: rows stably sorted by a 20-bit key
# whose bits, most significant first, say whether the 8 corner offsets and
# then the 12 edge offsets have a neighbour; maps of at most ONE_PASS_ROWS
# rows are sorted on the key's high 8 bits alone, the corners (one radix pass).  The sort
# runs within segments of SEGMENT_ROWS consecutive input rows, the segments
# kept in input order (0: the whole map is one segment).
_KEY_TAPS = [0, 2, 6, 8, 18, 20, 24, 26, 1, 3, 5, 7, 9, 11, 15, 17, 19, 21, 23, 25]
ONE_PASS_ROWS = 131072
SEGMENT_ROWS = 0


def expected_schedule(nbr, segment=SEGMENT_ROWS):
    n = nbr.shape[0]
    key = np.zeros(n, dtype=np.int64)
    for i, d in enumerate(_KEY_TAPS):
        key |= (nbr[:, d] >= 0).astype(np.int64) << (19 - i)
    if n <= ONE_PASS_ROWS:
        key >>= 12
    if segment:
        key |= (np.arange(n, dtype=np.int64) // segment) << 20
    return np.argsort(key, kind="stable").astype(np.int32)


MAP_CASES = ["tiny", "shell2", "shells6", "varlen4", "decoder0", "decoder3", "full128"]


@pytest.mark.parametrize("name", MAP_CASES)
def test_map_bit_exact(oracle_mod, name, map_lookup):
    w = workload(name)
    m = build(w)
    nbr = m.nbr().cpu().numpy()
    ref = oracle_mod.neighbour_map(w.coords, w.grid)
    np.testing.assert_array_equal(nbr, ref)
    counts, offsets, in_idx, out_idx = oracle_mod.pair_lists(ref)
    assert m.counts == counts.tolist()
    assert m.offsets == offsets.tolist()
    gi, go, _ = m.pairs()
    np.testing.assert_array_equal(gi.cpu().numpy(), in_idx)
    np.testing.assert_array_equal(go.cpu().numpy(), out_idx)
    perm = m.schedule().cpu().numpy()
    np.testing.assert_array_equal(perm, expected_schedule(ref))


@pytest.mark.parametrize("name,segment", [("shell2", 4096), ("shell2", 2048), ("varlen4", 2048),
                                          ("varlen4", 131072), ("varlen4", 262144)])
def test_schedule_segments(oracle_mod, name, segment):
    """The schedule's sort runs segment by segment: one segment, a segment per
    radix chunk, and lengths between, on the one-pass and two-pass paths."""
    w = workload(name)
    ref = oracle_mod.neighbour_map(w.coords, w.grid)
    smc.set_schedule_segment(segment)
    try:
        m = build(w)
    finally:
        smc.set_schedule_segment(-1)
    perm = m.schedule().cpu().numpy()
    np.testing.assert_array_equal(perm, expected_schedule(ref, segment))
    # the tile tap masks follow the order: a conv on the map stays exact
    f, wt, b = _layer(w, "f16")
    rows = np.sort(np.random.default_rng(5).choice(w.n, size=min(w.n, 2048), replace=False))
    got, ref_out = _conv_pair(oracle_mod, w, m, "f16", f, wt, b, 3, 1, rows=rows)
    check_close(got, ref_out, "f16", f"{name} conv, schedule segment {segment}")


def test_schedule_segment_arguments():
    lib = smc.lib()
    assert lib.smc_set_schedule_segment(-2) == -1
    assert lib.smc_set_schedule_segment(1000) == -1
    assert lib.smc_set_schedule_segment(-1) == 0


def test_map_uncleared_grid_reuse(oracle_mod):
    """The occupancy-bitmap grid is never cleared: a build that reuses the
    memory of an earlier build over the same box (from the library's pool)
    finds that build's rows in it and must ignore every one of them."""
    w = workload("shell2")
    rng = np.random.default_rng(11)
    smc.set_map_lookup(3)
    try:
        for trial in range(4):
            keep = rng.random(w.n) < (0.3 if trial % 2 else 0.9)
            coords = w.coords[keep]
            coords = coords[rng.permutation(len(coords))]
            m = smc.build_map(torch.from_numpy(coords).cuda(), w.grid, batch=2)
            ref = oracle_mod.neighbour_map(coords, w.grid)
            np.testing.assert_array_equal(m.nbr().cpu().numpy(), ref)
            counts, offsets, in_idx, out_idx = oracle_mod.pair_lists(ref)
            gi, go, _ = m.pairs()
            np.testing.assert_array_equal(gi.cpu().numpy(), in_idx)
            np.testing.assert_array_equal(go.cpu().numpy(), out_idx)
            m.free()
    finally:
        smc.set_map_lookup(0)


def test_map_shuffled_rows(oracle_mod, map_lookup):
    w = workload("shell2")
    rng = np.random.default_rng(1)
    coords = w.coords[rng.permutation(w.n)]
    m = smc.build_map(torch.from_numpy(coords).cuda(), w.grid, batch=2)
    ref = oracle_mod.neighbour_map(coords, w.grid)
    np.testing.assert_array_equal(m.nbr().cpu().numpy(), ref)
    np.testing.assert_array_equal(m.schedule().cpu().numpy(), expected_schedule(ref))


def test_map_wide_keys(oracle_mod):
    """batch * Z * Y * X above 2^32 takes the two-word hash slots."""
    rng = np.random.default_rng(2)
    grid = (2048, 2048, 2048)
    base = rng.integers(1, 2040, size=(300, 3))
    pts = {tuple(p + o) for p in base for o in np.argwhere(np.ones((2, 2, 2)))}
    zyx = np.array(sorted(pts), dtype=np.int32)
    coords = np.concatenate([np.zeros((len(zyx), 1), np.int32), zyx], axis=1)
    coords = np.concatenate([coords, coords + np.array([1, 0, 0, 0], np.int32)])
    m = smc.build_map(torch.from_numpy(coords).cuda(), grid, batch=2)
    ref = oracle_mod.neighbour_map(coords, grid)
    np.testing.assert_array_equal(m.nbr().cpu().numpy(), ref)
    np.testing.assert_array_equal(m.schedule().cpu().numpy(), expected_schedule(ref))


def test_map_empty_and_single(map_lookup):
    m = smc.build_map(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4), batch=1)
    assert m.n == 0 and m.counts == [0] * 27
    out = smc.conv(m, torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"),
                   torch.zeros((64, 3, 3, 3, 64), dtype=torch.bfloat16, device="cuda"))
    assert out.shape == (0, 64)
    one = smc.build_map(torch.tensor([[0, 2, 2, 2]], dtype=torch.int32, device="cuda"), (5, 5, 5), batch=1)
    nbr = one.nbr().cpu().numpy()
    assert nbr[0, 13] == 0 and (np.delete(nbr[0], 13) == -1).all()
    assert one.schedule().cpu().numpy().tolist() == [0]


def test_map_errors(map_lookup):
    def err_of(coords, grid=(8, 8, 8), batch=1):
        with pytest.raises(smc.SmcError) as e:
            smc.build_map(torch.tensor(coords, dtype=torch.int32, device="cuda"), grid, batch=batch)
        return e.value.name

    assert err_of([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]]) == "SMC_E_DUPLICATE"
    assert err_of([[0, 8, 0, 0]]) == "SMC_E_RANGE"
    assert err_of([[0, 0, -1, 0]]) == "SMC_E_RANGE"
    assert err_of([[1, 0, 0, 0]], batch=1) == "SMC_E_RANGE"
    coords = [[0, z, y, x] for z in range(4) for y in range(4) for x in range(4)]
    smc.set_hash_capacity(16)
    try:
        assert err_of(coords) == "SMC_E_CAPACITY"
    finally:
        smc.set_hash_capacity(0)
    m = smc.build_map(torch.tensor(coords, dtype=torch.int32, device="cuda"), (8, 8, 8), batch=1)
    assert m.counts[13] == 64
    smc.status()


# ------------------------------------------------------------------ subdivision
def _site_keys(coords, grid):
    c = coords.astype(np.int64)
    return ((c[:, 0] * grid[0] + c[:, 1]) * grid[1] + c[:, 2]) * grid[2] + c[:, 3]


def _check_child_map(oracle_mod, parent_coords, grid, keep, got_coords, child):
    ref_coords = oracle_mod.subdivide(parent_coords, keep)
    np.testing.assert_array_equal(got_coords.cpu().numpy(), ref_coords)
    grid2 = tuple(2 * g for g in grid)
    assert child.n == len(ref_coords) and child.grid == grid2
    ref = oracle_mod.neighbour_map(ref_coords, grid2)  # built from scratch, not from the parent map
    np.testing.assert_array_equal(child.nbr().cpu().numpy(), ref)
    counts, offsets, in_idx, out_idx = oracle_mod.pair_lists(ref)
    assert child.counts == counts.tolist()
    gi, go, _ = child.pairs()
    np.testing.assert_array_equal(gi.cpu().numpy(), in_idx)
    np.testing.assert_array_equal(go.cpu().numpy(), out_idx)
    np.testing.assert_array_equal(child.schedule().cpu().numpy(), expected_schedule(ref))
    return ref_coords


@pytest.mark.parametrize("mode", ["all", "random", "none_kept"])
def test_subdivide_matches_oracle(oracle_mod, mode):
    """Children of the two-item shell workload, all kept, half kept at random,
    or none: coordinates, map, pair lists and schedule bit-exact against the
    oracle's subdivision and a map the oracle builds from scratch."""
    w = workload("shell2")
    parent = build(w)
    pc = torch.from_numpy(w.coords).cuda()
    keep = None
    if mode == "random":
        keep = (np.random.default_rng(5).random((w.n, 8)) < 0.5).astype(np.uint8)
    elif mode == "none_kept":
        keep = np.zeros((w.n, 8), np.uint8)
    kids, child = smc.subdivide(parent, pc, None if keep is None else torch.from_numpy(keep).cuda())
    if mode == "none_kept":
        assert child.n == 0 and kids.shape == (0, 4)
        return
    _check_child_map(oracle_mod, w.coords, w.grid, keep, kids, child)
    smc.status()


def test_subdivide_decoder_chain(oracle_mod):
    """One decoder step: stage-1 voxels split and the children inside the
    stage-2 shell are kept; the child set is stage 2, its map is exact, and a
    conv over it meets the bf16 bar against the oracle."""
    w1, w2 = workload("decoder1"), workload("decoder2")
    kids_all = oracle_mod.subdivide(w1.coords)
    keep = np.isin(_site_keys(kids_all, w2.grid), _site_keys(w2.coords, w2.grid)).reshape(w1.n, 8).astype(np.uint8)
    parent = build(w1)
    kids, child = smc.subdivide(parent, torch.from_numpy(w1.coords).cuda(), torch.from_numpy(keep).cuda())
    ref_coords = _check_child_map(oracle_mod, w1.coords, w1.grid, keep, kids, child)
    assert set(_site_keys(ref_coords, w2.grid).tolist()) == set(_site_keys(w2.coords, w2.grid).tolist())
    sub = S.Workload("decoder2_from_subdivide", ref_coords, w2.grid, w2.cin, w2.cout, ("bf16",))
    f, wt, b = _layer(sub, "bf16")
    rows = sample_rows(sub.n, 2048, 9)
    out = smc.conv(child, dev(f, "bf16"), dev(wt, "bf16"), dev(b, "bf16"))
    ref = oracle_mod.conv(ref_coords, w2.grid, f, wt, b, 3, 1, rows=rows, threads=THREADS)
    check_close(host(out)[rows], ref, "bf16", "conv on the subdivided map")
    smc.status()


def test_subdivide_errors():
    w = workload("tiny")
    parent = build(w)
    pc = torch.from_numpy(w.coords).cuda()
    with pytest.raises(ValueError):
        smc.subdivide(parent, pc[:-1])
    empty = smc.build_map(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4), batch=1)
    kids, child = smc.subdivide(empty, torch.zeros((0, 4), dtype=torch.int32, device="cuda"))
    assert child.n == 0 and child.grid == (8, 8, 8)
    bad = smc.build_map(torch.tensor([[0, 1, 1, 1], [0, 1, 1, 1]], dtype=torch.int32, device="cuda"), (4, 4, 4),
                        batch=1, sync=False)
    with pytest.raises(smc.SmcError) as e:
        smc.subdivide(bad, torch.tensor([[0, 1, 1, 1], [0, 1, 1, 1]], dtype=torch.int32, device="cuda"))
    assert e.value.name == "SMC_E_DUPLICATE"


# ------------------------------------------------------------------ conv
def _layer(w, dtype, layer=0, ksize=3, cin=None, cout=None):
    return S.layer_tensors(w, dtype, layer, ksize, cin, cout)


def _conv_pair(oracle_mod, w, m, dtype, f, wt, b, ksize, orientation, rows=None):
    out = smc.conv(m, dev(f, dtype), dev(wt, dtype), dev(b, dtype), ksize=ksize, orientation=orientation)
    smc.status()
    got = host(out)
    ref = oracle_mod.conv(w.coords, w.grid, f, wt, b, ksize, orientation, rows=rows, threads=THREADS)
    return (got if rows is None else got[rows]), ref


@pytest.mark.parametrize("ksize,orientation", [(3, 1), (3, -1), (1, 1)])
def test_conv_tiny_f32(oracle_mod, ksize, orientation):
    w = workload("tiny")
    m = build(w)
    f, wt, b = _layer(w, "f32", 0, ksize)
    got, ref = _conv_pair(oracle_mod, w, m, "f32", f, wt, b, ksize, orientation)
    check_close(got, ref, "f32", f"tiny k={ksize} s={orientation}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_shell2_stacked(oracle_mod, dtype):
    """One map reused by 4 stacked k=3 layers; each layer is checked against
    the oracle fed the GPU's own (rounded) input to that layer."""
    w = workload("shell2")
    m = build(w, key=("shell2", dtype))
    assert build(w, key=("shell2", dtype)) is m
    x = _layer(w, dtype, 0)[0]
    for layer in range(4):
        _, wt, b = _layer(w, dtype, layer)
        xt = dev(x, dtype)
        out = smc.conv(m, xt, dev(wt, dtype), dev(b, dtype))
        got = host(out)
        ref = oracle_mod.conv(w.coords, w.grid, x, wt, b, 3, 1, threads=THREADS)
        check_close(got, ref, dtype, f"shell2 {dtype} layer {layer}")
        x = got.astype(np.float32)
    smc.status()


@pytest.mark.parametrize("orientation", [1, -1])
def test_conv_shells6_bf16(oracle_mod, orientation, conv_variant):
    w = workload("shells6")
    m = build(w)
    f, wt, b = _layer(w, "bf16")
    rows = sample_rows(w.n, 8192, 3)
    got, ref = _conv_pair(oracle_mod, w, m, "bf16", f, wt, b, 3, orientation, rows)
    check_close(got, ref, "bf16", f"shells6 s={orientation}")


def test_conv_full128_bf16_sampled(oracle_mod, conv_variant):
    w = workload("full128")
    m = build(w)
    f, wt, b = _layer(w, "bf16")
    rows = sample_rows(w.n, 4096, 4)
    got, ref = _conv_pair(oracle_mod, w, m, "bf16", f, wt, b, 3, 1, rows)
    check_close(got, ref, "bf16", "full128")


def test_conv_varlen4_f16_k3_then_k1(oracle_mod, conv_variant):
    w = workload("varlen4")
    m = build(w, key="varlen4")
    f, wt, b = _layer(w, "f16", 0, 3)
    rows = sample_rows(w.n, 4096, 5)
    out3 = smc.conv(m, dev(f, "f16"), dev(wt, "f16"), dev(b, "f16"), ksize=3)
    got3 = host(out3)
    ref3 = oracle_mod.conv(w.coords, w.grid, f, wt, b, 3, 1, rows=rows, threads=THREADS)
    check_close(got3[rows], ref3, "f16", "varlen4 k=3")
    x = got3.astype(np.float32)
    _, w1, b1 = _layer(w, "f16", 1, 1)
    out1 = smc.conv(build(w, key="varlen4"), out3, dev(w1, "f16"), dev(b1, "f16"), ksize=1)
    ref1 = oracle_mod.conv(w.coords, w.grid, x, w1, b1, 1, 1, rows=rows, threads=THREADS)
    check_close(host(out1)[rows], ref1, "f16", "varlen4 k=1")
    smc.status()


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
def test_conv_decoder_stage(oracle_mod, stage):
    """Decoder stack: 10 stacked bf16 k=3 layers on one map; sampled rows of
    every layer checked against the oracle on that layer's actual input."""
    w = workload(f"decoder{stage}")
    m = build(w)
    rows = sample_rows(w.n, 1024 if w.cin >= 256 else 2048, 10 + stage)
    x = _layer(w, "bf16", 0)[0]
    xt = dev(x, "bf16")
    for layer in range(10):
        _, wt, b = _layer(w, "bf16", layer)
        out = smc.conv(m, xt, dev(wt, "bf16"), dev(b, "bf16"))
        if layer in (0, 4, 9):
            ref = oracle_mod.conv(w.coords, w.grid, host(xt), wt, b, 3, 1, rows=rows, threads=THREADS)
            got = host(out)
            check_close(got if rows is None else got[rows], ref, "bf16", f"decoder{stage} layer {layer}")
        xt = out
    smc.status()


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("orientation", [1, -1])
def test_conv_small_integers_bit_exact(oracle_mod, dtype, orientation, conv_variant):
    """Inputs in {-1, 0, 1}: every partial sum is a small integer, so the
    result is exact in any accumulation order and must match bit for bit."""
    w = workload("shell2")
    m = build(w)
    rng = np.random.default_rng(21)
    cin, cout = 64, 64
    f = S.small_integer_values((w.n, cin), rng) * (rng.random((w.n, cin)) < 0.3)
    wt = S.small_integer_values((cout, 3, 3, 3, cin), rng) * (rng.random((cout, 3, 3, 3, cin)) < 0.3)
    b = S.small_integer_values((cout,), rng)
    got, ref = _conv_pair(oracle_mod, w, m, dtype, f.astype(np.float32), wt.astype(np.float32),
                          b.astype(np.float32), 3, orientation)
    assert np.abs(ref).max() <= 256
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("cin,cout", [(64, 16), (64, 512), (96, 48), (48, 64), (200, 24), (128, 272), (96, 64),
                                      (160, 128)])
def test_conv_channel_shapes_bf16(oracle_mod, cin, cout, conv_variant):
    """Tensor-core path with ragged K blocks, narrow and split N tiles; shapes
    outside its limits run on the FMA kernel; all must meet the same bar.
    (96, 64) and (160, 128) take ragged K blocks through the two-tile kernel
    (the default at 64 output channels, the forced variant at 128)."""
    w = workload("shell2")
    m = build(w)
    f, wt, b = _layer(w, "bf16", 7, 3, cin, cout)
    rows = sample_rows(w.n, 3000, 6)
    for s in (1, -1):
        got, ref = _conv_pair(oracle_mod, w, m, "bf16", f, wt, b, 3, s, rows)
        check_close(got, ref, "bf16", f"cin={cin} cout={cout} s={s}")


@pytest.mark.parametrize("rows", [128 * 5 + 37, 128 * 6 + 5, 100])
def test_conv_ragged_tail_and_no_bias(oracle_mod, rows, conv_variant):
    """Ragged last tile; an odd tile count (the last CTA pair has no second
    tile); a single partial tile."""
    w = workload("shell2")
    coords = w.coords[:rows]
    sub = S.Workload("ragged", coords, w.grid, 64, 64, ("bf16",))
    m = build(sub)
    f, wt, _ = _layer(sub, "bf16", 3)
    for dtype in ("bf16", "f32"):
        out = smc.conv(m, dev(f, dtype), dev(wt, dtype), None)
        ref = oracle_mod.conv(coords, w.grid, f, wt, None, 3, 1)
        check_close(host(out), ref, dtype, f"ragged {dtype}")
    smc.status()


@pytest.mark.parametrize("name,dtype", [("shells6", "bf16"), ("decoder3", "bf16"), ("varlen4", "f16")])
def test_conv_variants_agree(name, dtype):
    """The fused tensor-core kernels give the same output bits: one CTA per
    tile, CTA pairs and two tiles per CTA issue the union of their tiles'
    taps, and a tap a row lacks adds exact zeros."""
    w = workload(name)
    m = build(w)
    f, wt, b = _layer(w, dtype)
    outs = []
    for v in (1, 2, 4, 0):
        smc.set_conv_variant(v)
        try:
            outs.append(smc.conv(m, dev(f, dtype), dev(wt, dtype), dev(b, dtype)).cpu())
        finally:
            smc.set_conv_variant(0)
    for o in outs[1:]:
        assert torch.equal(outs[0], o)
    smc.status()


def test_conv_priority_streams_keep_order():
    """Convs forked to the library's high-priority streams stay ordered on the
    caller's stream: three stacked layers, each reading the previous output,
    give the same bits as on the caller's stream itself, on the map's stream
    and on another one."""
    w = workload("shell2")
    f, wt, b = _layer(w, "bf16")
    results = []
    for prio in (0, 1):
        smc.set_conv_priority(bool(prio))
        try:
            for other in (False, True):
                st = torch.cuda.Stream() if other else torch.cuda.current_stream()
                m = smc.build_map(torch.from_numpy(w.coords).cuda(), w.grid, batch=2, sync=False)
                x = dev(f, "bf16")
                with torch.cuda.stream(st):
                    st.wait_stream(torch.cuda.current_stream())
                    for _ in range(3):
                        x = smc.conv(m, x, dev(wt, "bf16"), dev(b, "bf16"), stream=st)
                st.synchronize()
                results.append(x.cpu())
                smc.status(st)
                m.free()
        finally:
            smc.set_conv_priority(True)
    for r in results[1:]:
        assert torch.equal(results[0], r)


# ------------------------------------------------------------------ epilogue (row pass / in the conv) and GroupNorm
@pytest.fixture(params=[0, 1], ids=["row_pass", "in_conv"])
def conv_epilogue(request):
    """Runs a test with the tensor-core conv's activation and residual applied
    by the row pass behind it, and inside its own epilogue."""
    smc.set_conv_epilogue(request.param)
    yield request.param
    smc.set_conv_epilogue(0)


@pytest.mark.parametrize("dtype,variant", [("bf16", 1), ("bf16", 2), ("bf16", 3), ("f32", 1), ("f16", 1)])
@pytest.mark.parametrize("act", [None, "relu", "silu"])
def test_conv_ex_epilogue(oracle_mod, dtype, variant, act, conv_epilogue):
    """out = act(conv + bias) + residual, and the GroupNorm statistics of the
    stored output: the output against the oracle, the statistics against
    fp64 sums of that very output (the two-item shell workload, 64 -> 64
    channels, 32 groups; bf16 on the three tensor-core variants, fp32 and
    fp16 on their kernels)."""
    w = workload("shell2")
    m = build(w)
    f, wt, b = _layer(w, dtype, 2)
    rng = np.random.default_rng(31)
    res = S.round_to(rng.standard_normal((w.n, w.cout)).astype(np.float32), dtype)
    coords = torch.from_numpy(w.coords).cuda()
    stats = torch.zeros((2, 32, 3), dtype=torch.float64, device="cuda")
    smc.set_conv_variant(variant)
    try:
        out = smc.conv(m, dev(f, dtype), dev(wt, dtype), dev(b, dtype), residual=dev(res, dtype), act=act,
                       coords=coords, stats=stats, groups=32)
    finally:
        smc.set_conv_variant(0)
    smc.status()
    got = host(out)
    ref = oracle_mod.activation(oracle_mod.conv(w.coords, w.grid, f, wt, b, 3, 1, threads=THREADS),
                                {None: 0, "relu": 1, "silu": 2}[act]) + res
    check_close(got, ref, dtype, f"conv_ex {dtype} v{variant} act={act}")
    np.testing.assert_allclose(stats.cpu().numpy(), oracle_mod.group_stats(got, w.coords, 2, 32), rtol=1e-9, atol=1e-6)


def test_conv_ex_residual_in_place(oracle_mod, conv_epilogue):
    """y = conv + out: the residual may be the output buffer itself."""
    w = workload("shell2")
    m = build(w)
    f, wt, b = _layer(w, "bf16", 4)
    start = S.round_to(np.random.default_rng(32).standard_normal((w.n, w.cout)).astype(np.float32), "bf16")
    out = dev(start, "bf16")
    smc.conv(m, dev(f, "bf16"), dev(wt, "bf16"), dev(b, "bf16"), out=out, residual=out)
    smc.status()
    ref = oracle_mod.conv(w.coords, w.grid, f, wt, b, 3, 1, threads=THREADS) + start
    check_close(host(out), ref, "bf16", "in-place residual")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_group_norm(oracle_mod, dtype):
    w = workload("shell2")
    rng = np.random.default_rng(33)
    x = S.round_to((rng.standard_normal((w.n, 64)) * 2 + 0.5).astype(np.float32), dtype)
    gamma = S.round_to(rng.standard_normal(64).astype(np.float32), dtype)
    beta = S.round_to(rng.standard_normal(64).astype(np.float32), dtype)
    coords = torch.from_numpy(w.coords).cuda()
    st = smc.group_stats(dev(x, dtype), coords, 2, 32)
    np.testing.assert_allclose(st.cpu().numpy(), oracle_mod.group_stats(x.astype(np.float64), w.coords, 2, 32), rtol=1e-9, atol=1e-6)
    out = smc.group_norm(dev(x, dtype), coords, 2, 32, st, dev(gamma, dtype), dev(beta, dtype), 1e-5, act="silu")
    smc.status()
    ref = oracle_mod.group_norm(x, w.coords, 2, 32, gamma, beta, 1e-5, act=2)
    check_close(host(out), ref, dtype, f"group_norm {dtype}")


def test_resblock_chain(oracle_mod, conv_epilogue):
    """A ResBlock on one cached map: GroupNorm32 + SiLU, conv (statistics of
    its output fused), GroupNorm32 + SiLU, conv + skip.  Every step is checked
    against the oracle fed the GPU's own input to that step."""
    w = workload("shell2")
    m = build(w)
    coords = torch.from_numpy(w.coords).cuda()
    rng = np.random.default_rng(34)
    x = S.round_to(rng.standard_normal((w.n, 64)).astype(np.float32), "bf16")
    _, w1, b1 = _layer(w, "bf16", 5)
    _, w2, b2 = _layer(w, "bf16", 6)
    xt = dev(x, "bf16")
    st0 = smc.group_stats(xt, coords, 2, 32)
    h = smc.group_norm(xt, coords, 2, 32, st0, act="silu")
    check_close(host(h), oracle_mod.group_norm(x, w.coords, 2, 32, act=2), "bf16", "gn1")
    st1 = torch.zeros((2, 32, 3), dtype=torch.float64, device="cuda")
    h1 = smc.conv(m, h, dev(w1, "bf16"), dev(b1, "bf16"), coords=coords, stats=st1, groups=32)
    check_close(host(h1), oracle_mod.conv(w.coords, w.grid, host(h), w1, b1, 3, 1, threads=THREADS), "bf16", "conv1")
    np.testing.assert_allclose(st1.cpu().numpy(), oracle_mod.group_stats(host(h1), w.coords, 2, 32), rtol=1e-9, atol=1e-6)
    h2 = smc.group_norm(h1, coords, 2, 32, st1, act="silu")
    check_close(host(h2), oracle_mod.group_norm(host(h1), w.coords, 2, 32, act=2), "bf16", "gn2")
    y = smc.conv(m, h2, dev(w2, "bf16"), dev(b2, "bf16"), residual=xt)
    ref = oracle_mod.conv(w.coords, w.grid, host(h2), w2, b2, 3, 1, threads=THREADS) + x
    check_close(host(y), ref, "bf16", "conv2 + skip")
    smc.status()


def test_conv_errors():
    w = workload("tiny")
    m = build(w)
    f = torch.zeros((w.n, 16), device="cuda")
    wt = torch.zeros((16, 3, 3, 3, 16), device="cuda")
    with pytest.raises(smc.SmcError) as e:
        smc.conv(m, f, wt, out=f)
    assert e.value.name == "SMC_E_ALIAS"
    lib = smc.lib()
    import ctypes
    rc = lib.smc_conv(m.handle, ctypes.c_void_p(f.data_ptr()), 16, ctypes.c_void_p(wt.data_ptr()), None,
                      ctypes.c_void_p(f.data_ptr() + 10 ** 6), 16, 2, 1, 0, None)
    assert rc == -1  # ksize 2
    rc = lib.smc_conv(m.handle, ctypes.c_void_p(f.data_ptr()), 16, ctypes.c_void_p(wt.data_ptr()), None,
                      ctypes.c_void_p(f.data_ptr() + 10 ** 6), 16, 3, 0, 0, None)
    assert rc == -1  # orientation 0
    rc = lib.smc_conv(m.handle, ctypes.c_void_p(f.data_ptr()), 16, ctypes.c_void_p(wt.data_ptr()), None,
                      ctypes.c_void_p(f.data_ptr() + 10 ** 6), 16, 3, 1, 7, None)
    assert rc == -4  # dtype
    smc.status()


def test_async_build_matches_sync(oracle_mod):
    """The asynchronous build enqueues everything on the stream; a conv queued
    right behind it must see the finished map."""
    w = workload("shells6")
    coords = torch.from_numpy(w.coords).cuda()
    f, wt, b = _layer(w, "bf16")
    ma = smc.build_map(coords, w.grid, batch=1, sync=False)
    out_a = smc.conv(ma, dev(f, "bf16"), dev(wt, "bf16"), dev(b, "bf16"))
    ma.wait()
    ms = smc.build_map(coords, w.grid, batch=1)
    out_s = smc.conv(ms, dev(f, "bf16"), dev(wt, "bf16"), dev(b, "bf16"))
    torch.testing.assert_close(out_a, out_s, rtol=0, atol=0)
    np.testing.assert_array_equal(ma.nbr().cpu().numpy(), ms.nbr().cpu().numpy())
    assert ma.counts == ms.counts


def test_pipelined_builds_reuse_memory():
    """Builds enqueued ahead of the host and retired later (the way a job runs
    them) must reuse the library pool's memory: device memory in use stays
    flat once the pipeline is full."""
    w = workload("shells6")
    coords = torch.from_numpy(w.coords).cuda()
    f, wt, b = (dev(x, "bf16") for x in _layer(w, "bf16"))
    out = torch.empty((w.n, w.cout), dtype=torch.bfloat16, device="cuda")

    def run(steps):
        pending = []
        for _ in range(steps):
            m = smc.build_map(coords, w.grid, batch=1, sync=False)
            smc.conv(m, f, wt, b, out=out)
            pending.append(m)
            if len(pending) > 4:
                old = pending.pop(0)
                old.wait()
                old.free()
        for m in pending:
            m.wait()
            m.free()
        torch.cuda.synchronize()
        return torch.cuda.mem_get_info()[0]

    free0 = run(12)
    free1 = run(60)
    assert free0 - free1 < 64 << 20, f"device memory grew by {(free0 - free1) >> 20} MiB over 60 builds"
    smc.status()


def test_failed_build_map_is_memory_safe(map_lookup):
    """Rows outside the box (SMC_E_RANGE) or repeated (SMC_E_DUPLICATE) still
    leave a map whose every entry is -1 or a valid row, and a schedule that is
    a permutation: a conv enqueued before the error is known stays in bounds."""
    rng = np.random.default_rng(7)
    good = np.unique(rng.integers(0, 8, size=(300, 3)), axis=0)
    coords = np.concatenate([np.zeros((len(good), 1), np.int64), good], axis=1).astype(np.int32)
    bad = np.array([[1, 0, 0, 0], [0, 8, 0, 0], [0, 0, -1, 3], [0, 3, 3, 9], [-1, 2, 2, 2]], np.int32)
    for extra, name in ((bad, "SMC_E_RANGE"), (coords[:3], "SMC_E_DUPLICATE")):
        allc = np.concatenate([coords, extra])
        m = smc.build_map(torch.from_numpy(allc).cuda(), (8, 8, 8), batch=1, sync=False)
        nbr = m.nbr().cpu().numpy()
        perm = m.schedule().cpu().numpy()
        with pytest.raises(smc.SmcError) as e:
            m.wait()
        assert e.value.name == name
        assert ((nbr >= -1) & (nbr < len(allc))).all()
        assert np.array_equal(np.sort(perm), np.arange(len(allc)))
        m.free()
    smc.status()


def test_async_build_reports_errors_late():
    coords = torch.tensor([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], dtype=torch.int32, device="cuda")
    m = smc.build_map(coords, (8, 8, 8), batch=1, sync=False)
    with pytest.raises(smc.SmcError) as e:
        m.wait()
    assert e.value.name == "SMC_E_DUPLICATE"
    with pytest.raises(smc.SmcError) as e:
        smc.conv(m, torch.zeros((3, 16), device="cuda"), torch.zeros((16, 3, 3, 3, 16), device="cuda"))
    assert e.value.name == "SMC_E_DUPLICATE"
    m.free()
    smc.status()


# ------------------------------------------------------------------ downsample / upsample
def _shuffled(w, seed):
    """The workload's rows in a seeded random order, so that first-appearance
    numbering differs from any sorted order."""
    perm = np.random.default_rng(seed).permutation(w.n)
    return np.ascontiguousarray(w.coords[perm])


def _pool_ref_check(got, ref, dtype, mode, what):
    if mode == "max":  # one of the inputs, exactly
        np.testing.assert_array_equal(got, S.round_to(ref, dtype).astype(np.float64), err_msg=what)
    else:
        check_close(got, ref, dtype, what)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("mode", ["max", "mean"])
@pytest.mark.parametrize("c", [128, 3])
def test_downsample_matches_oracle(oracle_mod, map_lookup, dtype, mode, c):
    """Two-item shell workload in shuffled row order: parent coordinates,
    subdivision mask and parent of each row bit-exact; max pooling exact, mean
    within the dtype's bar (16-byte vector path at 128 channels, scalar at 3)."""
    w = workload("shell2")
    coords = _shuffled(w, 31)
    f = S.features(w.n, c, np.random.default_rng(32), dtype)
    pc, pooled, mask, parent = smc.downsample(torch.from_numpy(coords).cuda(), w.grid, dev(f, dtype), mode, batch=2)
    rpc, rpooled, rmask, rparent = oracle_mod.downsample(coords, w.grid, f, oracle_mod.POOL_MAX if mode == "max"
                                                         else oracle_mod.POOL_MEAN, 2)
    np.testing.assert_array_equal(pc.cpu().numpy(), rpc)
    np.testing.assert_array_equal(mask.cpu().numpy(), rmask)
    np.testing.assert_array_equal(parent.cpu().numpy(), rparent)
    _pool_ref_check(host(pooled), rpooled, dtype, mode, f"{mode} pooling")
    smc.status()


def test_downsample_full128_sampled(oracle_mod):
    """The 128^3 full grid (2,097,152 rows, bf16, 128 channels), shuffled:
    structure bit-exact against the oracle, pooled features (max and mean)
    checked on 2048 sampled parents, each recomputed by the oracle from just
    its own children."""
    w = workload("full128")
    coords = _shuffled(w, 33)
    f = S.features(w.n, 128, np.random.default_rng(34), "bf16")
    ct, ft = torch.from_numpy(coords).cuda(), dev(f, "bf16")
    rpc, _, rmask, rparent = oracle_mod.downsample(coords, w.grid)
    rows_of = None
    for mode in ("max", "mean"):
        pc, pooled, mask, parent = smc.downsample(ct, w.grid, ft, mode, batch=1)
        np.testing.assert_array_equal(pc.cpu().numpy(), rpc)
        np.testing.assert_array_equal(mask.cpu().numpy(), rmask)
        np.testing.assert_array_equal(parent.cpu().numpy(), rparent)
        ps = sample_rows(len(rpc), 2048, 35)
        if rows_of is None:
            rows_of = np.flatnonzero(np.isin(rparent, ps))
        spc, sp, _, _ = oracle_mod.downsample(coords[rows_of], w.grid, f[rows_of],
                                              oracle_mod.POOL_MAX if mode == "max" else oracle_mod.POOL_MEAN, 1)
        # the subset's parents are the sampled parents, in the same relative order
        np.testing.assert_array_equal(spc, rpc[ps])
        _pool_ref_check(host(pooled)[ps], sp, "bf16", mode, f"{mode} pooling, sampled parents")
    smc.status()


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("with_map", [False, True], ids=["no_map", "child_map"])
def test_upsample_matches_oracle(oracle_mod, dtype, with_map):
    """Masked expansion of the shell workload with a random mask: children's
    coordinates (parent by parent, z-fastest index ascending) and features
    bit-exact; with the parent's map, the children's map, pair lists and
    schedule bit-exact against a map the oracle builds from scratch."""
    w = workload("shell2")
    mask = (np.random.default_rng(36).random((w.n, 8)) < 0.4).astype(np.uint8)
    c = 128 if dtype != "f32" else 5
    f = S.features(w.n, c, np.random.default_rng(37), dtype)
    ct = torch.from_numpy(w.coords).cuda()
    parent = build(w) if with_map else None
    kids, kf, child = smc.upsample(ct, torch.from_numpy(mask).cuda(), dev(f, dtype), parent=parent)
    rk, rf = oracle_mod.upsample(w.coords, mask, f)
    np.testing.assert_array_equal(kids.cpu().numpy(), rk)
    np.testing.assert_array_equal(host(kf), rf)
    if with_map:
        grid2 = tuple(2 * g for g in w.grid)
        assert child.n == len(rk) and child.grid == grid2
        ref = oracle_mod.neighbour_map(rk, grid2)
        np.testing.assert_array_equal(child.nbr().cpu().numpy(), ref)
        counts, _, in_idx, out_idx = oracle_mod.pair_lists(ref)
        gi, go, _ = child.pairs()
        np.testing.assert_array_equal(gi.cpu().numpy(), in_idx)
        np.testing.assert_array_equal(go.cpu().numpy(), out_idx)
        np.testing.assert_array_equal(child.schedule().cpu().numpy(), expected_schedule(ref))
    else:
        assert child is None
    smc.status()


def test_downsample_upsample_round_trip_gpu(oracle_mod):
    """Downsample the shuffled shell workload, build the parents' map, then
    upsample with the recorded mask: the children are the input sites again,
    their map is exact, and a conv over it meets the bf16 bar."""
    w = workload("shell2")
    coords = _shuffled(w, 38)
    pc, _, mask, _ = smc.downsample(torch.from_numpy(coords).cuda(), w.grid, None, "max", batch=2)
    half = tuple((g + 1) // 2 for g in w.grid)
    pm = smc.build_map(pc, half, batch=2)
    kids, _, child = smc.upsample(pc, mask, None, parent=pm)
    got = kids.cpu().numpy()
    assert sorted(map(tuple, got.tolist())) == sorted(map(tuple, coords.tolist()))
    rk, _ = oracle_mod.upsample(pc.cpu().numpy(), mask.cpu().numpy())
    np.testing.assert_array_equal(got, rk)
    grid2 = tuple(2 * g for g in half)
    np.testing.assert_array_equal(child.nbr().cpu().numpy(), oracle_mod.neighbour_map(rk, grid2))
    sub = S.Workload("round_trip", rk, grid2, 64, 64, ("bf16",))
    f, wt, b = _layer(sub, "bf16")
    rows = sample_rows(sub.n, 2048, 39)
    out = smc.conv(child, dev(f, "bf16"), dev(wt, "bf16"), dev(b, "bf16"))
    ref = oracle_mod.conv(rk, grid2, f, wt, b, 3, 1, rows=rows, threads=THREADS)
    check_close(host(out)[rows], ref, "bf16", "conv on the upsampled map")
    smc.status()


def test_resample_errors_and_edges(oracle_mod, map_lookup):
    d = "cuda"
    dup = torch.tensor([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], dtype=torch.int32, device=d)
    with pytest.raises(smc.SmcError) as e:
        smc.downsample(dup, (4, 4, 4), batch=1)
    assert e.value.name == "SMC_E_DUPLICATE"
    far = torch.tensor([[0, 1, 1, 1], [0, 1, 4, 1]], dtype=torch.int32, device=d)
    with pytest.raises(smc.SmcError) as e:
        smc.downsample(far, (4, 4, 4), torch.ones((2, 8), device=d), batch=1)
    assert e.value.name == "SMC_E_RANGE"
    empty = torch.zeros((0, 4), dtype=torch.int32, device=d)
    pc, pooled, mask, parent = smc.downsample(empty, (4, 4, 4), torch.zeros((0, 8), device=d), "mean", batch=1)
    assert pc.shape == (0, 4) and pooled.shape == (0, 8) and mask.shape == (0, 8) and parent.shape == (0,)
    kids, kf, child = smc.upsample(empty, None, torch.zeros((0, 8), device=d))
    assert kids.shape == (0, 4) and kf.shape == (0, 8) and child is None
    # odd extents: the last window is partial; one voxel per parent keeps its features
    one = torch.tensor([[0, 4, 1, 0], [1, 0, 0, 6]], dtype=torch.int32, device=d)
    x = torch.tensor([[1.5, -2.0], [3.0, 4.25]], device=d)
    pc, pooled, mask, _ = smc.downsample(one, (5, 3, 7), x, "mean", batch=2)
    assert pc.tolist() == [[0, 2, 0, 0], [1, 0, 0, 3]]
    assert pooled.tolist() == x.tolist()
    assert mask.tolist() == [[0, 0, 1, 0, 0, 0, 0, 0], [1, 0, 0, 0, 0, 0, 0, 0]]
    # a mask of all zeros emits nothing; a null mask emits all eight
    kids, _, _ = smc.upsample(pc, torch.zeros_like(mask))
    assert kids.shape == (0, 4)
    kids, _, _ = smc.upsample(pc, None)
    np.testing.assert_array_equal(kids.cpu().numpy(), oracle_mod.upsample(pc.cpu().numpy(), np.ones((2, 8)))[0])
    smc.status()


def test_downsample_upsample_varlen4_sampled(oracle_mod, map_lookup):
    """Four items of 300k-600k voxels on a 256^3 grid (fp16, 64 channels),
    shuffled, under each lookup structure: structure bit-exact, mean pooling
    on 2048 sampled parents (each recomputed from its own children), and the
    expansion back with the children's map bit-exact against the oracle's."""
    w = workload("varlen4")
    coords = _shuffled(w, 41)
    f = S.features(w.n, 64, np.random.default_rng(42), "f16")
    ct = torch.from_numpy(coords).cuda()
    pc, pooled, mask, parent = smc.downsample(ct, w.grid, dev(f, "f16"), "mean", batch=4)
    rpc, _, rmask, rparent = oracle_mod.downsample(coords, w.grid, None, oracle_mod.POOL_MEAN, 4)
    np.testing.assert_array_equal(pc.cpu().numpy(), rpc)
    np.testing.assert_array_equal(mask.cpu().numpy(), rmask)
    np.testing.assert_array_equal(parent.cpu().numpy(), rparent)
    ps = sample_rows(len(rpc), 2048, 43)
    rows_of = np.flatnonzero(np.isin(rparent, ps))
    spc, sp, _, _ = oracle_mod.downsample(coords[rows_of], w.grid, f[rows_of], oracle_mod.POOL_MEAN, 4)
    np.testing.assert_array_equal(spc, rpc[ps])
    check_close(host(pooled)[ps], sp, "f16", "mean pooling, sampled parents")
    half = tuple((g + 1) // 2 for g in w.grid)
    pm = smc.build_map(pc, half, batch=4)
    kids, kf, child = smc.upsample(pc, mask, pooled, parent=pm)
    rk, _ = oracle_mod.upsample(rpc, rmask)
    np.testing.assert_array_equal(kids.cpu().numpy(), rk)
    np.testing.assert_array_equal(kf.cpu().numpy()[:: 97], pooled.cpu().numpy()[np.repeat(np.arange(len(rpc)), rmask.sum(1).astype(np.int64))][:: 97])
    rows = sample_rows(len(rk), 4096, 44)
    ref = oracle_mod.neighbour_map(rk, w.grid)
    np.testing.assert_array_equal(child.nbr().cpu().numpy()[rows], ref[rows])
    smc.status()


@pytest.mark.parametrize("dtype,cout,groups", [("bf16", 128, 32), ("bf16", 256, 8), ("f32", 128, 32), ("f16", 128, 128)])
def test_row_pass_shuffled_items(oracle_mod, dtype, cout, groups):
    """The row pass behind a tensor-core or FMA conv on the two-item shell
    workload with its rows shuffled (batch items alternate row by row):
    act(conv) + residual against the oracle, the GroupNorm statistics against
    fp64 sums of the stored output, and the statistics-only pass alike."""
    w0 = workload("shell2")
    perm = np.random.default_rng(51).permutation(w0.n)
    coords = np.ascontiguousarray(w0.coords[perm])
    w = S.Workload("shell2_shuffled", coords, w0.grid, 64, cout, (dtype,))
    m = build(w)
    f, wt, b = _layer(w, dtype, 0, 3, 64, cout)
    res = S.round_to(np.random.default_rng(52).standard_normal((w.n, cout)).astype(np.float32), dtype)
    ct = torch.from_numpy(coords).cuda()
    stats = torch.zeros((2, groups, 3), dtype=torch.float64, device="cuda")
    out = smc.conv(m, dev(f, dtype), dev(wt, dtype), dev(b, dtype), residual=dev(res, dtype), act="silu",
                   coords=ct, stats=stats, groups=groups)
    smc.status()
    got = host(out)
    rows = sample_rows(w.n, 4096, 53)
    ref = oracle_mod.activation(oracle_mod.conv(coords, w.grid, f, wt, b, 3, 1, rows=rows, threads=THREADS), 2)
    check_close(got[rows], ref + res[rows], dtype, f"row pass {dtype} {cout}")
    np.testing.assert_allclose(stats.cpu().numpy(), oracle_mod.group_stats(got, coords, 2, groups), rtol=1e-9, atol=1e-6)
    st2 = torch.zeros_like(stats)
    smc.group_stats(out, ct, 2, groups, st2)
    smc.status()
    np.testing.assert_allclose(st2.cpu().numpy(), oracle_mod.group_stats(got, coords, 2, groups), rtol=1e-9, atol=1e-6)


def test_slab_conv_two_ranks_in_one_process():
    """The per-rank side of z-slab sharding on the GPU: two ranks' local maps
    (slab plus halo planes) built by the library, the halo rows copied from
    the neighbour's boundary rows by hand (the collective is tested with gloo
    on the CPU), two stacked bf16 layers: each rank's own rows equal the
    unsharded conv's, bit for bit (a row's taps are summed in the same order
    whatever tile it lands in)."""
    from submanifold_sparse_convolution_packed_b200.shard import SlabConv
    w = workload("shells6")
    f, w1, b1 = _layer(w, "bf16", 0)
    _, w2, b2 = _layer(w, "bf16", 1)
    full = build(w)
    ref = smc.conv(full, smc.conv(full, dev(f, "bf16"), dev(w1, "bf16"), dev(b1, "bf16")),
                   dev(w2, "bf16"), dev(b2, "bf16"))
    ranks = [SlabConv(w.coords, w.grid, 2, r, batch=1, device="cuda") for r in range(2)]
    x = [r.local_features(dev(f, "bf16")) for r in ranks]
    for wt, b in ((w1, b1), (w2, b2)):
        lo, hi = ranks[0].plan, ranks[1].plan
        # rank 0's top plane -> rank 1's halo below; rank 1's bottom plane -> rank 0's halo above
        x[1][hi.n_owned:hi.n_owned + hi.halo_lo.size] = x[0][torch.from_numpy(lo.send_hi).cuda()]
        x[0][lo.n_owned + lo.halo_lo.size:] = x[1][torch.from_numpy(hi.send_lo).cuda()]
        x = [smc.conv(r.map, xi, dev(wt, "bf16"), dev(b, "bf16")) for r, xi in zip(ranks, x)]
    got = torch.empty_like(ref)
    for r, xi in zip(ranks, x):
        got[torch.from_numpy(r.plan.owned).cuda()] = xi[:r.plan.n_owned]
    assert torch.equal(got, ref)
    smc.status()
