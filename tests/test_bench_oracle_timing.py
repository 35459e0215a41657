"""bench.py's oracle timing on the host (no GPU): which matrices the CPU
baseline and the reference arm time, and that the reference arm's line
describes what it ran (ms_per_step x steps within the run's wall time; value
= count-weighted per-shape means when the samples are single matrices)."""
import json
import sys
import time
import types
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import bench  # noqa: E402
from newton_schulz_normalise_b200 import workloads as wl  # noqa: E402


def test_small_sets_are_timed_in_full():
    for name in ("single-256x512-fp32", "batch64-1024x1024-bf16"):
        w = wl.WORKLOADS[name]
        idx, extrapolated = bench.oracle_sample(w)
        assert not extrapolated and idx == list(range(len(w.shapes())))


@pytest.mark.parametrize("name", ["transformer24-h2048-bf16", "skewed-shapes-bf16", "llama8b-matrices-bf16"])
def test_large_sets_time_one_matrix_per_shape(name):
    w = wl.WORKLOADS[name]
    idx, extrapolated = bench.oracle_sample(w)
    shapes = w.shapes()
    assert extrapolated
    assert sorted(shapes[i] for i in idx) == sorted(set(shapes))
    assert all(shapes.index(shapes[i]) == i for i in idx)  # first matrix of each shape


def test_set_time_is_count_weighted():
    w = wl.Workload("t", ((64, 256, 3), (96, 48, 2)), seed=1)
    per = {(64, 256): [0.010, 0.030], (96, 48): [0.004]}
    assert bench.oracle_set_ms(w, per) == pytest.approx(1e3 * (3 * 0.020 + 2 * 0.004))


def _run_reference(monkeypatch, capsys, w, steps, warmup, full_flops):
    monkeypatch.setattr(bench, "FULL_ORACLE_FLOPS", full_flops)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    args = types.SimpleNamespace(steps=steps, warmup=warmup)
    t0 = time.perf_counter()
    assert bench.run_reference(args, w) == 0
    wall = time.perf_counter() - t0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0]), wall


def test_reference_arm_extrapolated_line_matches_what_ran(monkeypatch, capsys):
    w = wl.Workload("t", ((64, 256, 3), (96, 48, 2), (130, 300, 1)), seed=2)
    d, wall = _run_reference(monkeypatch, capsys, w, steps=4, warmup=1, full_flops=0.0)
    assert d["impl"] == "reference" and d["extrapolated"] is True
    assert d["steps"] == 4 and d["ms_per_step"] * d["steps"] <= wall * 1e3
    per = d["cpu_baseline"]["per_shape_ms"]
    assert set(per) == {"64x256", "96x48", "130x300"}
    # value = sum over shapes of count x mean ms per matrix (rounded per shape in the line)
    want = 3 * per["64x256"] + 2 * per["96x48"] + per["130x300"]
    assert d["value"] == pytest.approx(want, rel=1e-3, abs=3e-3)
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["value"] == d["value"]


def test_reference_arm_full_set_steps(monkeypatch, capsys):
    w = wl.Workload("t", ((64, 256, 2), (96, 48, 1)), seed=3)
    d, wall = _run_reference(monkeypatch, capsys, w, steps=3, warmup=1, full_flops=1e18)
    assert d["extrapolated"] is False
    assert d["ms_per_step"] * 3 <= wall * 1e3
    # every step timed the whole set: the set time is the mean step time
    assert d["value"] == pytest.approx(d["ms_per_step"], rel=1e-6)


def test_reference_arm_fewer_steps_than_shapes(monkeypatch, capsys):
    w = wl.Workload("t", ((64, 256, 1), (96, 48, 1), (130, 300, 1)), seed=4)
    d, _ = _run_reference(monkeypatch, capsys, w, steps=1, warmup=0, full_flops=0.0)
    assert set(d["cpu_baseline"]["per_shape_ms"]) == {"64x256", "96x48", "130x300"}
