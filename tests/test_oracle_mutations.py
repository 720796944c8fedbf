"""Planted mistakes: each is compiled into a throw-away copy of the oracle on
the CPU, and the pins of test_oracle_pins must reject it.  This shows the pins
are strong enough to catch the plausible slips they were chosen for."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from tests.test_oracle_pins import _random_case, _torch_dense_conv

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "smc_oracle.cpp")

MUTATIONS = {
    "orientation_sign": ("c[1] + sign * delta[0], c[2] + sign * delta[1], c[3] + sign * delta[2]",
                         "c[1] - sign * delta[0], c[2] - sign * delta[1], c[3] - sign * delta[2]"),
    "axis_swap": ("delta[0] = kz - h;\n  delta[1] = ky - h;\n  delta[2] = kx - h;",
                  "delta[0] = kx - h;\n  delta[1] = ky - h;\n  delta[2] = kz - h;"),
    "weight_transposed": ("weight + (o * taps + d) * cin", "weight + (d * cout + o) * cin"),
    "dropped_tap": ("const int64_t u = neighbour(index, coords + 4 * v, delta, orientation);\n      if (u < 0) continue;",
                    "const int64_t u = neighbour(index, coords + 4 * v, delta, orientation);\n      if (u < 0 || d == 0) continue;"),
    "batch_leak": ("Site s = {c[0], c[1] + sign", "Site s = {0, c[1] + sign"),
    "bias_missing": ("acc[o] + (bias ? bias[o] : 0.0)", "acc[o]"),
}


def _build_mutant(name, tmpdir):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name} no longer applies"
    path = os.path.join(tmpdir, f"{name}.cpp")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmpdir, f"lib{name}.so")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", path, "-o", lib])
    dll = ctypes.CDLL(lib)
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    dll.oracle_conv.argtypes = [P, i64, P, P, i64, P, P, i64, i32, i32, P, i64, P, i32]
    dll.oracle_conv.restype = ctypes.c_int
    return dll


def _run(dll, coords, grid, feats, w, b, k, s):
    c = np.ascontiguousarray(coords, dtype=np.int32)
    g = np.ascontiguousarray(grid, dtype=np.int32)
    f = np.ascontiguousarray(feats, dtype=np.float64)
    ww = np.ascontiguousarray(w, dtype=np.float64)
    bb = np.ascontiguousarray(b, dtype=np.float64)
    out = np.empty((len(c), ww.shape[0]))
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = dll.oracle_conv(p(c), len(c), p(g), p(f), f.shape[1], p(ww), p(bb), ww.shape[0], k, s,
                         None, len(c), p(out), 1)
    assert rc == 0
    return out


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(name):
    with tempfile.TemporaryDirectory() as tmp:
        dll = _build_mutant(name, tmp)
        rng = np.random.default_rng(0)
        grid, batch = (5, 6, 7), 2
        coords, feats, w, b = _random_case(rng, grid, batch, 0.35, 3, 5)
        caught = False
        for s, wref in ((+1, w), (-1, w[:, ::-1, ::-1, ::-1, :])):
            ref = _torch_dense_conv(coords, feats, wref, b, grid, batch, 3)
            got = _run(dll, coords, grid, feats, w, b, 3, s)
            caught |= not np.allclose(got, ref, rtol=1e-12, atol=1e-12)
        assert caught, f"planted mistake {name!r} passed the dense-equivalence pin"


# Planted mistakes in the Python half of the oracle (resampling): each is
# applied to a copy of oracle.py loaded as a throw-away module, and at least
# one of the resampling pins must fail on it.
PY_SRC = os.path.join(os.path.dirname(SRC), "oracle.py")
PY_MUTATIONS = {
    "subidx_c_order": ("return dz + 2 * dy + 4 * dx", "return 4 * dz + 2 * dy + dx"),
    "upsample_c_order": ("(b, 2 * z + j % 2, 2 * y + j // 2 % 2, 2 * x + j // 4 % 2)",
                         "(b, 2 * z + j // 4 % 2, 2 * y + j // 2 % 2, 2 * x + j % 2)"),
    "parent_rounds_up": ("key = (b, z // 2, y // 2, x // 2)", "key = (b, (z + 1) // 2, y // 2, x // 2)"),
    "mean_not_divided": ("pooled /= mask.sum(axis=1, dtype=np.float64)[:, None]", "pass"),
    "max_sums": ("np.maximum.at(pooled, parent, f)", "pooled[:] = 0.0\n            np.add.at(pooled, parent, f)"),
    "upsample_wrong_source": ("src.append(p)", "src.append(max(p - 1, 0))"),
}
RESAMPLE_PINS = ["test_golden_downsample_upsample", "test_downsample_matches_dense_pooling",
                 "test_upsample_matches_nearest_interpolation", "test_upsample_index_is_subdivide_octant_reversed",
                 "test_downsample_upsample_round_trip"]
# the same for subdivision, the activations and GroupNorm, against their pins
OTHER_MUTATIONS = {
    "subdivide_axes_swapped": ("a, cc, e = o >> 2, (o >> 1) & 1, o & 1", "e, cc, a = o >> 2, (o >> 1) & 1, o & 1"),
    "subdivide_not_doubled": ("children[:, o, 2] = 2 * c[:, 2] + cc", "children[:, o, 2] = c[:, 2] + cc"),
    "silu_sign": ("return y / (1.0 + np.exp(-y))", "return y / (1.0 + np.exp(y))"),
    "relu_leaky": ("return np.maximum(y, 0.0)", "return np.maximum(y, 0.01 * y)"),
    "stats_ignore_item": ("rows = xg[b == item]", "rows = xg"),
    "variance_unbiased": ("var = st[:, :, 1] / cnt - mean * mean", "var = (st[:, :, 1] - cnt * mean * mean) / (cnt - 1)"),
    "eps_outside_sqrt": ("/ np.sqrt(var[b][:, g_of_c] + eps)", "/ (np.sqrt(var[b][:, g_of_c]) + eps)"),
    "gamma_after_beta": ("""    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)[None, :]
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)[None, :]""", """    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)[None, :]
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)[None, :]"""),
}
OTHER_PINS = ["test_golden_subdivide_one_voxel", "test_subdivide_full_box_is_full_doubled_box",
              "test_subdivide_parent_and_octant_recovery", "test_activation_matches_torch",
              "test_group_norm_matches_torch_per_item", "test_group_stats_hand_example"]


def _py_mutant(name):
    import types
    old, new = PY_MUTATIONS[name] if name in PY_MUTATIONS else OTHER_MUTATIONS[name]
    src = open(PY_SRC).read()
    assert src.count(old) == 1, f"mutation {name} no longer applies"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__file__ = PY_SRC
    exec(compile(src.replace(old, new), PY_SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_resample_pins_reject_planted_mistake(name):
    import tests.test_oracle_pins as pins
    mod = _py_mutant(name)
    failed = []
    for pin in RESAMPLE_PINS:
        fn = getattr(pins, pin)
        args = [(6, 4, 8)] if pin == "test_downsample_matches_dense_pooling" else []
        try:
            fn(mod, *args)
        except Exception:
            failed.append(pin)
    assert failed, f"planted mistake {name!r} passed every resampling pin"


@pytest.mark.parametrize("name", sorted(OTHER_MUTATIONS))
def test_subdivide_and_norm_pins_reject_planted_mistake(name):
    import tests.test_oracle_pins as pins
    mod = _py_mutant(name)
    failed = []
    for pin in OTHER_PINS:
        try:
            getattr(pins, pin)(mod)
        except Exception:
            failed.append(pin)
    assert failed, f"planted mistake {name!r} passed every subdivision / norm pin"
