"""bench.py's host-side report helpers, on hand-countable inputs (CPU)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _map(rows: int, hits_per_offset: dict) -> np.ndarray:
    """[rows, 27] map: the centre always hits; offset k hits its first hits_per_offset[k] rows."""
    nbr = np.full((rows, 27), -1, dtype=np.int32)
    nbr[:, 13] = np.arange(rows)
    for k, h in hits_per_offset.items():
        nbr[:h, k] = 0
    return nbr


def test_column_efficiency_full_jobs_is_one():
    # one 48-row tile, every offset full: every job is exactly 48 columns
    nbr = _map(48, {k: 48 for k in range(27) if k != 13})
    assert bench.mma_column_efficiency(nbr, tile_rows=48, bm=128) == 1.0


def test_column_efficiency_counts_padding():
    # 48-row tile: centre 48 columns (48 issued), offset 0 has 10 hits -> 16 issued,
    # offset 5 has 40 hits -> 48 issued, others none
    nbr = _map(48, {0: 10, 5: 40})
    assert bench.mma_column_efficiency(nbr, tile_rows=48) == pytest.approx((48 + 10 + 40) / (48 + 16 + 48))
    # two tiles of 24 rows: centre 24 + 24 (rounded to 32 each); offset 0: 10 in tile 0 -> 16
    nbr = _map(48, {0: 10})
    assert bench.mma_column_efficiency(nbr, tile_rows=24) == pytest.approx((48 + 10) / (32 + 32 + 16))


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


def test_column_efficiency_of_the_bench_workload():
    """The bench reports the fraction of issued MMA columns that carry a pair. On the
    128^3 / 10 % workload, with the 355-row tiles the library picks on 148 SMs
    (ceil(209715 / (384 * 148)) = 4 waves, ceil(209715 / (4 * 148)) = 355 rows),
    the oracle's map gives 85.4 %."""
    import oracle
    import workloads

    wl = workloads.make_workload("uniform", 0, n_layers=1)
    nbr = oracle.neighbor_map(wl.coords, wl.grid)
    assert -(-wl.n // (384 * 148)) == 4 and -(-wl.n // (4 * 148)) == 355
    assert int((nbr >= 0).sum()) == 745983
    assert bench.mma_column_efficiency(nbr, 355) == pytest.approx(0.8541, abs=1e-4)
