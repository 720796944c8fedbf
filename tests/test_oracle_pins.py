"""Pins for the CPU oracle: it is checked against things other than itself.

Every test here runs on the CPU (no GPU marker).  The pins are chosen so that
a plausible slip in the oracle -- a dropped tap, a wrong sign, a swapped
coordinate axis, a transposed weight operand, a batch leak -- fails at least
one of them:

* hand-derived worked examples stored under tests/golden/ (each cites the
  page section whose definition it follows);
* dense-conv equivalence: on tiny grids the sparse layer equals a zero-padded
  dense 3-D cross-correlation (torch.nn.functional.conv3d in fp64) sampled at
  the active sites, and with the kernel flipped on all three axes it equals
  the other orientation;
* an independent numpy implementation over a dense grid with explicit shifts;
* closed forms: identity centre tap, single-tap translation, k=1 linear layer,
  full-box hit counts (Z-|dz|)(Y-|dy|)(X-|dx|);
* invariants: centre tap is the identity map, neighbour symmetry, batch
  isolation, linearity, brute-force all-pairs neighbour search;
* subdivision: a hand-listed voxel, a full box that must become the full
  doubled box, and parent/octant recovery from each child;
* downsample / upsample: a hand-worked example, dense max_pool3d and
  avg_pool3d, nearest interpolation, the octant bit reversal against
  subdivide, and the round trip.

Grids are deliberately non-cubic and channel counts unequal so that an axis
swap or an operand transposition cannot cancel out.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
OFFSETS = [(kz - 1, ky - 1, kx - 1) for kz in range(3) for ky in range(3) for kx in range(3)]


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _random_case(rng, grid, batch, p, cin, cout, k=3):
    coords = []
    for b in range(batch):
        occ = rng.random(grid) < p
        for z, y, x in np.argwhere(occ):
            coords.append((b, z, y, x))
    coords = np.array(coords, dtype=np.int32).reshape(-1, 4)
    coords = coords[rng.permutation(len(coords))]  # arbitrary row order
    n = len(coords)
    feats = rng.standard_normal((n, cin))
    weight = rng.standard_normal((cout, k, k, k, cin))
    bias = rng.standard_normal(cout)
    return coords, feats, weight, bias


def _densify(coords, feats, grid, batch):
    dense = np.zeros((batch, feats.shape[1]) + tuple(grid))
    for r, (b, z, y, x) in enumerate(coords):
        dense[b, :, z, y, x] = feats[r]
    return dense


def _torch_dense_conv(coords, feats, weight, bias, grid, batch, k):
    dense = torch.from_numpy(_densify(coords, feats, grid, batch))
    w = torch.from_numpy(np.ascontiguousarray(weight)).permute(0, 4, 1, 2, 3)  # KRSC -> OIDHW
    out = torch.nn.functional.conv3d(dense, w, torch.from_numpy(bias), padding=(k - 1) // 2)
    out = out.numpy()
    return np.stack([out[b, :, z, y, x] for b, z, y, x in coords])


# --------------------------------------------------------------------------
# worked examples (golden)
# --------------------------------------------------------------------------
def test_golden_translation(oracle_mod):
    g = _golden("translation_pair.json")
    coords = np.array(g["coords"], dtype=np.int32)
    feats = np.array(g["feats"])
    c = feats.shape[1]
    w = np.zeros((c, 3, 3, 3, c))
    kz, ky, kx = np.unravel_index(g["tap"], (3, 3, 3))
    assert (kz - 1, ky - 1, kx - 1) == tuple(g["tap_offset_zyx"])
    w[:, kz, ky, kx, :] = np.eye(c)
    plus = oracle_mod.conv(coords, g["grid"], feats, w, None, 3, +1)
    minus = oracle_mod.conv(coords, g["grid"], feats, w, None, 3, -1)
    np.testing.assert_array_equal(plus, np.array(g["expected_plus"]))
    np.testing.assert_array_equal(minus, np.array(g["expected_minus"]))
    nbr = oracle_mod.neighbour_map(coords, g["grid"])
    for v in range(len(coords)):
        hits = {str(d): int(nbr[v, d]) for d in range(27) if nbr[v, d] >= 0}
        assert hits == {k: v2 for k, v2 in g["expected_nbr_hits"][str(v)].items()}
    counts, _, _, _ = oracle_mod.pair_lists(nbr)
    assert {str(d): int(c) for d, c in enumerate(counts) if c} == g["expected_counts_nonzero"]


def test_golden_hand_conv_1d(oracle_mod):
    g = _golden("hand_conv_1d.json")
    coords = np.array(g["coords"], dtype=np.int32)
    feats = np.array(g["feats"])
    w = np.zeros((1, 3, 3, 3, 1))
    for kx, val in g["weight_row_kx"].items():
        w[0, 1, 1, int(kx), 0] = val
    b = np.array(g["bias"])
    plus = oracle_mod.conv(coords, g["grid"], feats, w, b, 3, +1)[:, 0]
    minus = oracle_mod.conv(coords, g["grid"], feats, w, b, 3, -1)[:, 0]
    np.testing.assert_array_equal(plus, g["expected_plus"])
    np.testing.assert_array_equal(minus, g["expected_minus"])


def _tap_class(d):
    l1 = sum(abs(a) for a in OFFSETS[d])
    return ["centre", "face", "edge", "corner"][l1]


def test_golden_full_box_counts(oracle_mod):
    g = _golden("full_cube_counts.json")
    for case in g["cases"]:
        grid = case["grid"]
        coords = np.array([(0, z, y, x) for z in range(grid[0]) for y in range(grid[1])
                           for x in range(grid[2])], dtype=np.int32)
        nbr = oracle_mod.neighbour_map(coords, grid)
        counts, offsets, _, _ = oracle_mod.pair_lists(nbr)
        assert int(offsets[-1]) == case["total"]
        if "per_class" in case:
            for d in range(27):
                assert counts[d] == case["per_class"][_tap_class(d)]


# --------------------------------------------------------------------------
# dense-conv equivalence and an independent numpy implementation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed,grid,batch,p,cin,cout", [
    (0, (5, 6, 7), 2, 0.35, 3, 5),
    (1, (4, 7, 5), 1, 0.6, 4, 2),
    (2, (6, 5, 4), 3, 0.2, 2, 3),
])
def test_dense_equivalence(oracle_mod, seed, grid, batch, p, cin, cout):
    rng = np.random.default_rng(seed)
    coords, feats, w, b = _random_case(rng, grid, batch, p, cin, cout)
    ref = _torch_dense_conv(coords, feats, w, b, grid, batch, 3)
    got = oracle_mod.conv(coords, grid, feats, w, b, 3, +1)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # the other orientation is the dense correlation with the kernel flipped on all axes
    ref_m = _torch_dense_conv(coords, feats, w[:, ::-1, ::-1, ::-1, :], b, grid, batch, 3)
    got_m = oracle_mod.conv(coords, grid, feats, w, b, 3, -1)
    np.testing.assert_allclose(got_m, ref_m, rtol=1e-12, atol=1e-12)
    # k = 1
    w1 = rng.standard_normal((cout, 1, 1, 1, cin))
    ref1 = _torch_dense_conv(coords, feats, w1, b, grid, batch, 1)
    np.testing.assert_allclose(oracle_mod.conv(coords, grid, feats, w1, b, 1, +1), ref1,
                               rtol=1e-12, atol=1e-12)


def _numpy_shift_conv(coords, feats, w, b, grid, batch, sign):
    """Second, independent implementation: dense grid, explicit shifted slices."""
    dense = _densify(coords, feats, grid, batch)             # [B, Cin, Z, Y, X]
    pad = np.pad(dense, ((0, 0), (0, 0), (1, 1), (1, 1), (1, 1)))
    Z, Y, X = grid
    out = np.zeros((batch, w.shape[0], Z, Y, X))
    for kz, ky, kx in itertools.product(range(3), repeat=3):
        dz, dy, dx = sign * (kz - 1), sign * (ky - 1), sign * (kx - 1)
        src = pad[:, :, 1 + dz:1 + dz + Z, 1 + dy:1 + dy + Y, 1 + dx:1 + dx + X]
        out += np.einsum("bizyx,oi->bozyx", src, w[:, kz, ky, kx, :])
    out += b[None, :, None, None, None]
    return np.stack([out[bb, :, z, y, x] for bb, z, y, x in coords])


@pytest.mark.parametrize("sign", [+1, -1])
def test_numpy_shift_implementation(oracle_mod, sign):
    rng = np.random.default_rng(7)
    grid, batch = (6, 4, 5), 2
    coords, feats, w, b = _random_case(rng, grid, batch, 0.4, 3, 4)
    ref = _numpy_shift_conv(coords, feats, w, b, grid, batch, sign)
    got = oracle_mod.conv(coords, grid, feats, w, b, 3, sign)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def test_identity_centre_tap(oracle_mod):
    rng = np.random.default_rng(3)
    coords, feats, _, b = _random_case(rng, (7, 5, 6), 2, 0.3, 4, 4)
    w = np.zeros((4, 3, 3, 3, 4))
    w[:, 1, 1, 1, :] = np.eye(4)
    for s in (+1, -1):
        np.testing.assert_array_equal(oracle_mod.conv(coords, (7, 5, 6), feats, w, b, 3, s),
                                      feats + b)


@pytest.mark.parametrize("tap", [0, 4, 10, 14, 22, 26])
def test_single_tap_translation(oracle_mod, tap):
    rng = np.random.default_rng(tap)
    grid = (5, 6, 4)
    coords, feats, _, _ = _random_case(rng, grid, 2, 0.5, 3, 3)
    w = np.zeros((3, 3, 3, 3, 3))
    kz, ky, kx = np.unravel_index(tap, (3, 3, 3))
    w[:, kz, ky, kx, :] = np.eye(3)
    delta = np.array(OFFSETS[tap])
    where = {tuple(c): r for r, c in enumerate(coords.tolist())}
    for s in (+1, -1):
        got = oracle_mod.conv(coords, grid, feats, w, None, 3, s)
        for r, c in enumerate(coords.tolist()):
            q = (c[0],) + tuple(np.array(c[1:]) + s * delta)
            expect = feats[where[q]] if q in where else np.zeros(3)
            np.testing.assert_array_equal(got[r], expect)


def test_k1_is_linear_layer(oracle_mod):
    rng = np.random.default_rng(11)
    coords, feats, _, b = _random_case(rng, (4, 5, 6), 2, 0.5, 5, 3)
    w1 = rng.standard_normal((3, 1, 1, 1, 5))
    ref = feats @ w1[:, 0, 0, 0, :].T + b
    for s in (+1, -1):
        np.testing.assert_allclose(oracle_mod.conv(coords, (4, 5, 6), feats, w1, b, 1, s), ref,
                                   rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# invariants of the neighbour map and pair lists
# --------------------------------------------------------------------------
def test_map_invariants_and_bruteforce(oracle_mod):
    rng = np.random.default_rng(5)
    grid = (6, 5, 7)
    coords, _, _, _ = _random_case(rng, grid, 2, 0.3, 1, 1)
    nbr = oracle_mod.neighbour_map(coords, grid)
    n = len(coords)
    assert (nbr[:, 13] == np.arange(n)).all()
    for v in range(n):
        for d in range(27):
            u = nbr[v, d]
            if u >= 0:
                assert nbr[u, 26 - d] == v
    # brute force O(N^2): u is the tap-d neighbour of v iff same batch and c_u - c_v = offset(d)
    brute = np.full((n, 27), -1, dtype=np.int32)
    for v in range(n):
        for u in range(n):
            if coords[u, 0] != coords[v, 0]:
                continue
            diff = tuple(coords[u, 1:] - coords[v, 1:])
            if max(abs(x) for x in diff) <= 1:
                brute[v, OFFSETS.index(diff)] = u
    np.testing.assert_array_equal(nbr, brute)
    counts, offsets, in_idx, out_idx = oracle_mod.pair_lists(nbr)
    for d in range(27):
        assert counts[d] == counts[26 - d]
        seg = slice(offsets[d], offsets[d + 1])
        expect = [(int(nbr[v, d]), v) for v in range(n) if nbr[v, d] >= 0]
        assert list(zip(in_idx[seg].tolist(), out_idx[seg].tolist())) == expect


def test_isolated_voxel_hits_only_centre(oracle_mod):
    coords = np.array([[0, 1, 1, 1], [0, 4, 4, 4], [1, 1, 1, 2]], dtype=np.int32)
    nbr = oracle_mod.neighbour_map(coords, (6, 6, 6))
    for v in range(3):
        assert [d for d in range(27) if nbr[v, d] >= 0] == [13]


def test_batch_isolation(oracle_mod):
    rng = np.random.default_rng(9)
    grid = (5, 5, 5)
    coords, feats, w, b = _random_case(rng, grid, 1, 0.5, 3, 2)
    both = np.concatenate([coords, coords + np.array([1, 0, 0, 0], dtype=np.int32)])
    f2 = np.concatenate([feats, 2.0 * feats])
    got = oracle_mod.conv(both, grid, f2, w, b, 3, +1)
    one = oracle_mod.conv(coords, grid, feats, w, b, 3, +1)
    two = oracle_mod.conv(coords, grid, 2.0 * feats, w, b, 3, +1)
    np.testing.assert_allclose(got[:len(coords)], one, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(got[len(coords):], two, rtol=1e-13, atol=1e-13)


def test_linearity(oracle_mod):
    rng = np.random.default_rng(13)
    grid = (6, 6, 5)
    coords, f1, w, b = _random_case(rng, grid, 2, 0.4, 4, 3)
    f2 = rng.standard_normal(f1.shape)
    alpha = 1.75
    lhs = oracle_mod.conv(coords, grid, alpha * f1 + f2, w, b, 3, +1) - b
    rhs = alpha * (oracle_mod.conv(coords, grid, f1, w, b, 3, +1) - b) + \
        (oracle_mod.conv(coords, grid, f2, w, b, 3, +1) - b)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(17)
    grid = (5, 6, 7)
    coords, feats, w, b = _random_case(rng, grid, 2, 0.4, 3, 4)
    full = oracle_mod.conv(coords, grid, feats, w, b, 3, -1, threads=2)
    rows = rng.choice(len(coords), size=len(coords) // 3, replace=False)
    sub = oracle_mod.conv(coords, grid, feats, w, b, 3, -1, rows=rows)
    np.testing.assert_array_equal(sub, full[rows])


def test_errors(oracle_mod):
    grid = (4, 4, 4)
    dup = np.array([[0, 1, 1, 1], [0, 1, 1, 1]], dtype=np.int32)
    with pytest.raises(oracle_mod.OracleError) as e:
        oracle_mod.neighbour_map(dup, grid)
    assert e.value.code == -3
    for bad in ([0, 4, 0, 0], [0, 0, -1, 0], [0, 0, 0, 4], [-1, 0, 0, 0]):
        with pytest.raises(oracle_mod.OracleError) as e:
            oracle_mod.neighbour_map(np.array([bad], dtype=np.int32), grid)
        assert e.value.code == -2


def test_empty_input(oracle_mod):
    coords = np.zeros((0, 4), dtype=np.int32)
    nbr = oracle_mod.neighbour_map(coords, (3, 3, 3))
    assert nbr.shape == (0, 27)
    counts, offsets, in_idx, _ = oracle_mod.pair_lists(nbr)
    assert counts.sum() == 0 and in_idx.size == 0
    out = oracle_mod.conv(coords, (3, 3, 3), np.zeros((0, 2)), np.zeros((3, 3, 3, 3, 2)), None)
    assert out.shape == (0, 3)


# ------------------------------------------------------------------ subdivision
def test_golden_subdivide_one_voxel(oracle_mod):
    g = _golden("subdivide_one_voxel.json")
    coords = np.array(g["coords"], np.int32)
    assert oracle_mod.subdivide(coords).tolist() == g["expected_children"]
    assert oracle_mod.subdivide(coords, np.array(g["keep"], np.uint8)).tolist() == g["expected_kept"]


def test_subdivide_full_box_is_full_doubled_box(oracle_mod):
    """Subdividing every site of a 2 x (2, 3, 4) box gives every site of the
    2 x (4, 6, 8) box exactly once."""
    box = np.array([(b, z, y, x) for b in range(2) for z in range(2) for y in range(3) for x in range(4)], np.int32)
    kids = oracle_mod.subdivide(box)
    full = {(b, z, y, x) for b in range(2) for z in range(4) for y in range(6) for x in range(8)}
    assert len(kids) == 8 * len(box) == len(full)
    assert {tuple(r) for r in kids.tolist()} == full


def test_subdivide_parent_and_octant_recovery(oracle_mod):
    """Each child halves back to its parent; its low bits are its octant, in
    C order, and a keep mask drops exactly the masked children."""
    rng = np.random.default_rng(3)
    coords = np.unique(rng.integers(0, 9, size=(60, 4)), axis=0).astype(np.int32)
    keep = (rng.random((len(coords), 8)) < 0.6).astype(np.uint8)
    kids = oracle_mod.subdivide(coords, keep)
    parents = np.repeat(np.arange(len(coords)), 8).reshape(-1, 8)[keep != 0]
    octs = np.tile(np.arange(8), (len(coords), 1))[keep != 0]
    assert len(kids) == int(keep.sum())
    np.testing.assert_array_equal(kids[:, 0], coords[parents, 0])
    np.testing.assert_array_equal(kids[:, 1:] // 2, coords[parents, 1:])
    np.testing.assert_array_equal(4 * (kids[:, 1] % 2) + 2 * (kids[:, 2] % 2) + kids[:, 3] % 2, octs)


# ------------------------------------------------------------------ norm / activation
def test_activation_matches_torch(oracle_mod):
    x = np.random.default_rng(11).standard_normal((50, 7)) * 4
    t = torch.from_numpy(x)
    np.testing.assert_allclose(oracle_mod.activation(x, 2), torch.nn.functional.silu(t).numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(oracle_mod.activation(x, 1), torch.relu(t).numpy())
    np.testing.assert_array_equal(oracle_mod.activation(x, 0), x)


def test_group_norm_matches_torch_per_item(oracle_mod):
    """GroupNorm over a sparse tensor is torch's GroupNorm applied to each
    batch item's rows laid out as [1, C, rows]; two items of unequal size
    must not mix."""
    rng = np.random.default_rng(12)
    coords = np.array([[b, z, 0, 0] for b, cnt in ((0, 37), (1, 21)) for z in range(cnt)], np.int32)
    x = rng.standard_normal((len(coords), 12)) * 3 + 1
    gamma, beta = rng.standard_normal(12), rng.standard_normal(12)
    got = oracle_mod.group_norm(x, coords, 2, 4, gamma, beta, 1e-5, act=2)
    for item in range(2):
        rows = coords[:, 0] == item
        t = torch.from_numpy(x[rows].T.copy())[None]
        ref = torch.nn.functional.group_norm(t, 4, torch.from_numpy(gamma), torch.from_numpy(beta), 1e-5)
        ref = torch.nn.functional.silu(ref)[0].T.numpy()
        np.testing.assert_allclose(got[rows], ref, rtol=1e-10, atol=1e-12)


def test_group_stats_hand_example(oracle_mod):
    coords = np.array([[0, 0, 0, 0], [1, 0, 0, 0], [0, 1, 0, 0]], np.int32)
    x = np.array([[1.0, 2.0, 3.0, 4.0], [5.0, 6.0, 7.0, 8.0], [-1.0, 0.5, 2.0, -2.0]])
    st = oracle_mod.group_stats(x, coords, 2, 2)
    np.testing.assert_array_equal(st[0, 0], [1 + 2 - 1 + 0.5, 1 + 4 + 1 + 0.25, 4])
    np.testing.assert_array_equal(st[0, 1], [3 + 4 + 2 - 2, 9 + 16 + 4 + 4, 4])
    np.testing.assert_array_equal(st[1, 0], [11, 61, 2])
    np.testing.assert_array_equal(st[1, 1], [15, 113, 2])


# ------------------------------------------------------------------ downsample / upsample
def test_golden_downsample_upsample(oracle_mod):
    g = _golden("downsample_upsample.json")
    coords, feats = np.array(g["coords"], np.int32), np.array(g["feats"])
    pc, mx, mask, parent = oracle_mod.downsample(coords, g["grid"], feats, oracle_mod.POOL_MAX, g["batch"])
    assert pc.tolist() == g["expected_parent_coords"]
    assert parent.tolist() == g["expected_parent_of_row"]
    assert mask.tolist() == g["expected_mask"]
    np.testing.assert_array_equal(mx, g["expected_max"])
    _, mean, _, _ = oracle_mod.downsample(coords, g["grid"], feats, oracle_mod.POOL_MEAN, g["batch"])
    np.testing.assert_allclose(mean, np.array(g["expected_mean_num"]) / np.array(g["expected_mean_den"])[:, None],
                               rtol=1e-15)
    kids, kf = oracle_mod.upsample(pc, mask, np.array(g["upsample_feats"]))
    assert kids.tolist() == g["expected_children"]
    np.testing.assert_array_equal(kf, g["expected_child_feats"])


def _dense_volume(coords, feats, grid, batch, fill):
    vol = torch.full((batch, feats.shape[1], *grid), fill, dtype=torch.float64)
    c = torch.from_numpy(coords.astype(np.int64))
    vol[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(feats)
    return vol


@pytest.mark.parametrize("grid", [(6, 4, 8), (5, 7, 3)])
def test_downsample_matches_dense_pooling(oracle_mod, grid):
    """On a dense grid, max pooling is max_pool3d(2, stride 2) with empty sites
    at -inf, and mean pooling is avg_pool3d of the features over avg_pool3d
    of the occupancy (both zero at empty sites); odd extents pool a partial
    last window (ceil_mode)."""
    rng = np.random.default_rng(21)
    batch = 2
    sites = np.array(list(itertools.product(range(batch), *(range(s) for s in grid))), np.int32)
    coords = sites[rng.random(len(sites)) < 0.3]
    coords = coords[rng.permutation(len(coords))]
    feats = rng.standard_normal((len(coords), 3))
    pool = dict(kernel_size=2, stride=2, ceil_mode=True)
    pc, mx, mask, _ = oracle_mod.downsample(coords, grid, feats, oracle_mod.POOL_MAX, batch)
    ref = torch.nn.functional.max_pool3d(_dense_volume(coords, feats, grid, batch, -np.inf), **pool)
    b, z, y, x = (torch.from_numpy(pc[:, i].astype(np.int64)) for i in range(4))
    np.testing.assert_array_equal(mx, ref[b, :, z, y, x].numpy())
    _, mean, _, _ = oracle_mod.downsample(coords, grid, feats, oracle_mod.POOL_MEAN, batch)
    num = torch.nn.functional.avg_pool3d(_dense_volume(coords, feats, grid, batch, 0.0), **pool)
    occ = torch.nn.functional.avg_pool3d(_dense_volume(coords, np.ones((len(coords), 1)), grid, batch, 0.0), **pool)
    np.testing.assert_allclose(mean, (num / occ)[b, :, z, y, x].numpy(), rtol=1e-12, atol=1e-14)
    # every occupied window is a parent, once; its mask counts its sites
    occupied = torch.nonzero(occ[:, 0] > 0).numpy()
    assert sorted(map(tuple, pc.tolist())) == sorted(map(tuple, occupied.tolist()))
    assert mask.sum() == len(coords)


def test_upsample_matches_nearest_interpolation(oracle_mod):
    """Each kept child carries its parent's features: nearest upsampling by 2
    of the dense parent volume (interpolate, mode 'nearest') sampled at the
    children; the children are exactly the masked sites of the doubled box."""
    rng = np.random.default_rng(22)
    grid, batch = (3, 4, 2), 2
    sites = np.array(list(itertools.product(range(batch), *(range(s) for s in grid))), np.int32)
    coords = sites[rng.random(len(sites)) < 0.6]
    feats = rng.standard_normal((len(coords), 4))
    mask = (rng.random((len(coords), 8)) < 0.5).astype(np.uint8)
    kids, kf = oracle_mod.upsample(coords, mask, feats)
    up = torch.nn.functional.interpolate(_dense_volume(coords, feats, grid, batch, 0.0), scale_factor=2,
                                         mode="nearest")
    b, z, y, x = (torch.from_numpy(kids[:, i].astype(np.int64)) for i in range(4))
    np.testing.assert_array_equal(kf, up[b, :, z, y, x].numpy())
    want = set()
    for p, (cb, cz, cy, cx) in enumerate(coords.tolist()):
        for dz, dy, dx in itertools.product(range(2), repeat=3):
            if mask[p, dz + 2 * dy + 4 * dx]:
                want.add((cb, 2 * cz + dz, 2 * cy + dy, 2 * cx + dx))
    assert len(kids) == int(mask.sum()) and set(map(tuple, kids.tolist())) == want


def test_upsample_index_is_subdivide_octant_reversed(oracle_mod):
    """With every child kept, upsample lists each parent's children at subidx
    j where subdivide lists them at the C-order octant whose three bits are
    j's in reverse (the commit log notes the two orders are reverses)."""
    coords = np.array([[0, 1, 2, 3], [1, 0, 5, 2]], np.int32)
    kids, _ = oracle_mod.upsample(coords, np.ones((2, 8), np.uint8))
    sub = oracle_mod.subdivide(coords)
    rev = [int(f"{j:03b}"[::-1], 2) for j in range(8)]
    for p in range(2):
        assert kids[8 * p:8 * p + 8].tolist() == sub[8 * p + np.array(rev)].tolist()


def test_downsample_upsample_round_trip(oracle_mod):
    """Upsampling the parents with the mask the downsample recorded gives back
    exactly the input sites; every row halves to its parent's coordinates."""
    rng = np.random.default_rng(23)
    coords = np.unique(rng.integers(0, 11, size=(300, 4)), axis=0).astype(np.int32)
    coords[:, 0] %= 3
    coords = np.unique(coords, axis=0)[rng.permutation(len(np.unique(coords, axis=0)))]
    pc, _, mask, parent = oracle_mod.downsample(coords, (11, 11, 11))
    kids, _ = oracle_mod.upsample(pc, mask)
    assert sorted(map(tuple, kids.tolist())) == sorted(map(tuple, coords.tolist()))
    np.testing.assert_array_equal(pc[parent, 0], coords[:, 0])
    np.testing.assert_array_equal(pc[parent, 1:], coords[:, 1:] // 2)
    # first-appearance numbering: parent indices first occur in increasing order
    first = np.unique(parent, return_index=True)[1]
    assert (np.diff(first) > 0).all() and parent[0] == 0


def test_downsample_errors(oracle_mod):
    c = np.array([[0, 0, 0, 0], [0, 0, 0, 0]], np.int32)
    with pytest.raises(oracle_mod.OracleError) as e:
        oracle_mod.downsample(c, (2, 2, 2))
    assert e.value.code == -3
    with pytest.raises(oracle_mod.OracleError) as e:
        oracle_mod.downsample(np.array([[0, 2, 0, 0]], np.int32), (2, 2, 2))
    assert e.value.code == -2
    pc, pooled, mask, parent = oracle_mod.downsample(np.zeros((0, 4), np.int32), (2, 2, 2), np.zeros((0, 3)))
    assert pc.shape == (0, 4) and pooled.shape == (0, 3) and mask.shape == (0, 8) and parent.shape == (0,)
    kids, kf = oracle_mod.upsample(pc, mask, pooled)
    assert kids.shape == (0, 4) and kf.shape == (0, 3)
