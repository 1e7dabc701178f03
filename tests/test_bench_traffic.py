"""The bench line's DRAM traffic figures (host logic, CPU).

``bench.py`` keeps one ncu capture of every kernel's DRAM bytes together with
the digest of the CUDA sources it ran; the line reports a figure only while
the sources are the captured ones, and null (with the reason) otherwise.
"""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_recorded_capture_of_the_current_sources():
    """While the recorded capture belongs to the current kernels, every
    kernel of both captured workloads has its figure (after a kernel change
    the figures are null until the capture is taken again)."""
    if bench.MEASURED_TRAFFIC["csrc_digest"] != bench.csrc_digest():
        pytest.skip("the CUDA sources changed since the recorded ncu capture")
    for workload in ("bf16_g8", "stacked_g128_ragged"):
        for op in ("fwd", "dgrad", "wgrad", "quant_x", "quant_w", "quant_dy", "fwd_mx", "dgrad_mx", "wgrad_mx"):
            v, note = bench.measured_traffic(workload, op)
            assert isinstance(v, int) and v > 0, (workload, op)
            assert bench.MEASURED_TRAFFIC["csrc_digest"] in note


def test_digest_follows_every_source_file(tmp_path, monkeypatch):
    """Changing, adding or renaming a CUDA source changes the digest."""
    src = os.path.join(ROOT, "grouped_gemm_splits_b200", "csrc")
    copy = tmp_path / "grouped_gemm_splits_b200" / "csrc"
    shutil.copytree(src, copy)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.csrc_digest()
    assert d0 == bench.csrc_digest()  # deterministic
    f = copy / "gl_offsets.cu"
    f.write_text(f.read_text() + "\n// a comment\n")
    d1 = bench.csrc_digest()
    assert d1 != d0
    (copy / "gl_new.cuh").write_text("// new header\n")
    d2 = bench.csrc_digest()
    assert d2 not in (d0, d1)
    os.rename(copy / "gl_new.cuh", copy / "gl_other.cuh")
    assert bench.csrc_digest() not in (d0, d1, d2)


def test_stale_capture_reports_null(monkeypatch):
    monkeypatch.setattr(bench, "csrc_digest", lambda: "0000000000000000")
    v, note = bench.measured_traffic("bf16_g8", "wgrad")
    assert v is None and "stale" in note


def test_missing_workload_or_capture_reports_null(monkeypatch):
    v, note = bench.measured_traffic("fine_g64", "wgrad")
    assert v is None and "fine_g64" in note
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {})
    v, note = bench.measured_traffic("bf16_g8", "wgrad")
    assert v is None and "no ncu capture" in note
