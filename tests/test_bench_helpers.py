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
