"""bench.py's host-side report helpers, on hand-countable inputs (CPU)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_issued_column_efficiency():
    # 3 tiles of 16 rows (48 issued centre columns) and 32 span columns for 40 pairs
    assert bench.issued_column_efficiency(pairs=40, npad=48, span_cols=32) == pytest.approx(40 / 80)
    assert bench.issued_column_efficiency(pairs=0, npad=0, span_cols=0) == 1.0


def test_roofline_picks_the_slower_bound():
    # 10 voxels, 30 pairs, 16 -> 32 channels: bytes vs FLOPs at chosen peaks
    byts, flops = bench.roofline_bytes_flops(n=10, pairs=30, cin=16, cout=32)
    r = bench.roofline(10, 30, 16, 32, 27, layer_s=1e-6, hbm_gbs=byts / 1e3, tflops=flops / 1e6 * 2)
    assert r["bound"] == "hbm" and r["t_roof_us"] == pytest.approx(1.0) and r["frac"] == pytest.approx(1.0)
    r = bench.roofline(10, 30, 16, 32, 27, layer_s=2e-6, hbm_gbs=byts / 1e3 * 4, tflops=flops / 1e6)
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(0.5)
    # kernel size 1: the weights are one [Cin, Cout] matrix and no neighbour indices
    b1, f1 = bench.roofline_bytes_flops(n=10, pairs=10, cin=16, cout=32, kvol=1)
    assert b1 == 10 * 16 * 2 + 16 * 32 * 2 + 32 * 2 + 10 * 32 * 2 and f1 == 2 * 16 * 32 * 10


def test_roofline_bytes_and_flops():
    byts, flops = bench.roofline_bytes_flops(n=10, pairs=30, cin=16, cout=32)
    assert byts == 10 * 16 * 2 + 27 * 16 * 32 * 2 + 32 * 2 + 10 * 32 * 2 + 4 * 20
    assert flops == 2 * 16 * 32 * 30


def test_clock_sampler_parses_nvidia_smi_lines():
    """Median SM clock, max clock and the throttle reasons seen, from the csv rows
    nvidia-smi prints during the timed region (fields in ClockSampler.FIELDS order)."""
    s = bench.ClockSampler("0")
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]

    class _Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc = _Done()
    c = s.stop()
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]
    s.lines.append("0, 1400, 1965, 990.0, 0x48, Active, Not Active, Active, Not Active")
    c = s.stop()
    assert c["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_sampler_without_nvidia_smi_reports_unavailable():
    s = bench.ClockSampler("0")
    assert s.stop() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}


def test_kernel_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """roofline.traffic is reported only while the profiled kernel's code is
    unchanged: comment and whitespace edits keep the hash, a code edit changes it."""
    import shutil

    csrc = tmp_path / "submanifold_sparse_convolution_submconv3d_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(ROOT, "submanifold_sparse_convolution_submconv3d_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_sha256()
    f = csrc / "forward_win.cu"
    src = f.read_text()
    f.write_text("// a new comment line\n" + src.replace("\n", "  \n", 3) + "\n/* trailing\n block */\n")
    assert bench.kernel_sources_sha256() == h0
    f.write_text(src.replace("kUnitRows = 64", "kUnitRows = 32", 1))
    assert bench.kernel_sources_sha256() != h0


def test_tc_kernel_name_follows_the_dispatch():
    assert bench.tc_kernel_name(128, 128) == "k_subm_win<128,128>"
    assert bench.tc_kernel_name(64, 64) == "k_subm_win<64,64>"
    assert bench.tc_kernel_name(48, 192) == "k_subm_win<64,16>"
    assert bench.tc_kernel_name(32, 256) == "k_subm_win<128,32>"
    # the map's launch counters name the kernel-size-1 GEMM when it ran
    assert bench.tc_kernel_name(512, 512, {"simt": 0, "tcgen05": 0, "tcgen05_gemm": 1}) == "k_gemm1<128>"
    assert bench.tc_kernel_name(64, 192, {"simt": 0, "tcgen05": 0, "tcgen05_gemm": 1}) == "k_gemm1<64>"
    assert bench.tc_kernel_name(48, 128, {"simt": 0, "tcgen05": 1, "tcgen05_gemm": 0}) == "k_subm_win<128,16>"
