"""bench.py's host-side accounting (no GPU): Newton-Schulz FLOPs per matrix
for both forms, and the rule that a profiled DRAM traffic figure is reported
only while the kernel source matches the one profiled."""
import hashlib
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import bench  # noqa: E402

# per-matrix NS FLOPs with K = 5: direct 2K(2 m^2 n + m^3), Gram 2(2 m^2 n + 17 m^3)
TABLE = [((256, 512), 0.84e9, 0.71e9), ((1024, 1024), 32.2e9, 40.8e9), ((2048, 6144), 601e9, 395e9),
         ((4096, 14336), 5498e9, 3299e9), ((64, 256), 24e6, 13e6), ((14336, 4096), 5498e9, 3299e9)]


@pytest.mark.parametrize("shape,direct,gram", TABLE)
def test_ns_flops(shape, direct, gram):
    r, c = shape
    m, n = min(r, c), max(r, c)
    assert bench.ns_flops(r, c, 5, "direct") == 2 * 5 * (2 * m * m * n + m ** 3)
    assert bench.ns_flops(r, c, 5, "gram") == 2 * (2 * m * m * n + (1 + 4 * 4) * m ** 3)
    # the table's values are rounded to 2-3 digits
    assert bench.ns_flops(r, c, 5, "direct") == pytest.approx(direct, rel=2e-2)
    assert bench.ns_flops(r, c, 5, "gram") == pytest.approx(gram, rel=2e-2)
    assert bench.ns_flops(r, c, 0, "direct") == 0.0


def test_profile_traffic_needs_matching_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    prof = tmp_path / "profiles"
    prof.mkdir()
    summ = prof / "tc_gemm_pair_batch64-1024x1024.md"
    summ.write_text(f"traffic_bytes_per_launch: 1234\nkernel_source_sha256_16: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.profile_traffic(src, "batch64-1024x1024-bf16") == 1234.0
    assert bench.profile_traffic(src, "skewed-shapes-bf16") is None  # no summary for that workload
    src.write_text("// kernel, changed\n")
    assert bench.profile_traffic(src, "batch64-1024x1024-bf16") is None


def test_fp32_peak_from_unit_counts():
    assert bench.FP32_FFMA_TFLOPS == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_end_to_end_leg_skips_when_the_host_cannot_pin_every_rank():
    """The end-to-end leg pins each rank's gradients and parameters; it is
    skipped, with the reason, when the node's ranks together would not fit in
    the host's available memory (with a quarter to spare)."""
    import psutil
    import bench
    avail = psutil.virtual_memory().available
    assert bench.host_memory_short(avail // 100, 2) is None
    reason = bench.host_memory_short(avail, 8)
    assert reason is not None and "8 rank(s)" in reason and "GB available" in reason
