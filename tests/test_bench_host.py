"""Host-side pieces of bench.py (no GPU): the per-op roofline arithmetic."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_sweep_entry_roofline_fractions():
    peaks = {"hbm_gbs": 6528.7, "bf16_tflops": 1648.3}
    # HBM-bound decode point: 16 x 28672 x 8192, 4-bit weights
    op = bench.Op("decode", None, 2.0 * 16 * 28672 * 8192, 28672 * 8192 // 2, 16 * 8192 * 2 + 16 * 28672 * 2, 1)
    e = bench.sweep_entry(op, 0.054, peaks)
    t = 0.054e-3
    assert abs(e["hbm_frac"] - op.bytes / t / 1e9 / 6528.7) < 1e-3
    assert abs(e["hbm_frac_nominal"] - op.bytes / t / 1e9 / 8000.0) < 1e-3
    assert e["roofline_frac"] == e["hbm_frac"]  # the bytes bound is the larger one here
    # tensor-bound point with an FP4 MMA (4 x the bf16 peak)
    op2 = bench.Op("fp4", None, 2.0 * 8192 * 7168 * 7168, 7168 * 7168 // 2, 8192 * 7168 * 3, 1, peak_ratio=4.0)
    e2 = bench.sweep_entry(op2, 0.43, peaks)
    assert abs(e2["tensor_frac"] - op2.flops / 0.43e-3 / 1e12 / (4 * 1648.3)) < 1e-3
    assert e2["roofline_frac"] == e2["tensor_frac"]


def test_every_workload_has_a_title_and_its_configs():
    for name in bench.WORKLOADS:
        assert name in bench.WORKLOAD_CONFIGS, name
        if name != "all":
            assert name in bench.WORKLOAD_TITLE, name


def test_measured_traffic_follows_the_kernel_source_digest(tmp_path, monkeypatch):
    digest = bench.kernel_source_digest()
    assert len(digest) == 16 and int(digest, 16) >= 0
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.md").write_text(
        "| op | kernel | read | write | traffic | digest |\n|---|---|---|---|---|---|\n"
        f"| op_a | k | 1 | 2 | 3 | {digest} |\n"
        "| op_b | k | 1 | 2 | 5 | 0000000000000000 |\n")
    # the digest is taken of the real kernel sources, the table from the temporary root
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("op_a") == 3.0
    assert bench.measured_traffic("op_b") is None  # captured on other sources
    assert bench.measured_traffic("op_c") is None
