"""CPU checks of bench.py's host-side logic: the clock record's region and
window bookkeeping, and the CPU-baseline record (oracle on all cores and on
one thread, with the host's CPU model and core count)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from submanifold_sparse_convolution_packed_b200 import synth as S  # noqa: E402


def _row(mhz, reason_cap="Not Active", thermal="Not Active"):
    return ["0", str(mhz), "1965", "900.0", "0x0", "Not Active", "Not Active", thermal, reason_cap]


def test_clock_summary_region_only():
    rows = [_row(1500), _row(1965), _row(1965), _row(1935)]
    out = bench.ClockSampler.summary(rows, mark_at=1, end_at=4)
    assert out["samples"] == 3 and out["sm_mhz"] == 1965.0 and out["reasons"] == []
    assert "window" not in out and "note" not in out


def test_clock_summary_with_window_and_reasons():
    rows = [_row(1965), _row(1800, reason_cap="Active"), _row(1965), _row(1965, thermal="Active")]
    out = bench.ClockSampler.summary(rows, mark_at=1, end_at=2, window_note="same steps repeated")
    assert out["samples"] == 1 and out["window_samples"] == 2
    assert out["window"] == "same steps repeated"
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_clock_summary_region_too_short():
    rows = [_row(1700), _row(1965)]
    out = bench.ClockSampler.summary(rows, mark_at=2, end_at=2)
    assert out["samples"] == 0 and "note" in out and out["sm_mhz"] == 1965.0


def test_cpu_baseline_record_fields():
    w = S.workload("tiny")
    f, wt, b = S.layer_tensors(w, "f32")
    rec = bench.run_cpu_baseline(w, f, wt, b, budget_s=0.2)
    assert rec["kind"] == "oracle" and rec["value"] > 0 and rec["cores"] == (os.cpu_count() or 1)
    assert rec["nproc"] == rec["cores"] and rec["cpu_model"]
    assert rec["single_thread"]["cores"] == 1 and rec["single_thread"]["value"] > 0


def test_workload_118k_draw():
    w = S.workload("shells6_118k")
    assert w.n == 117818 and w.grid == (128, 128, 128) and w.cin == w.cout == 128


def test_input_sets_exceed_l2():
    """The pipelined steps rotate over copies of their inputs whose total is
    at least 3x L2 (so no flush is needed), with at least two copies."""
    import torch
    w = S.workload("shell2")
    f, _, _ = S.layer_tensors(w, "bf16")
    sets = bench.input_sets(torch, torch.device("cpu"), w, f, torch.bfloat16)
    per = w.n * (16 + 2 * w.cin + 2 * w.cout)
    assert 2 <= len(sets) <= 8
    assert len(sets) == 8 or len(sets) * per >= 3 * bench.L2_BYTES
    c, x, y = sets[0]
    assert c.shape == (w.n, 4) and x.shape == (w.n, w.cin) and y.shape == (w.n, w.cout)
    assert all(s[0].data_ptr() != sets[0][0].data_ptr() for s in sets[1:])
