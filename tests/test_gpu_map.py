"""GPU neighbour-map build vs the CPU oracle: bit-exact, every workload and edge case."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import coords_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sp():
    import submanifold_sparse_convolution_submconv3d_b200 as p
    return p


def _check_map(sp, coords, extent, kernel_size=3):
    m = sp.spconv_build_map(coords_dev(coords), extent, kernel_size)
    try:
        got = m.neighbor_map().cpu().numpy()
        ref = oracle.neighbor_map(coords, extent, kernel_size)
        assert got.shape == ref.shape
        assert np.array_equal(got, ref)
        assert m.pairs == int((ref >= 0).sum())
        assert m.n == coords.shape[0] and m.kernel_size == kernel_size
    finally:
        m.free()


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
def test_map_bit_exact_on_workloads(sp, name):
    wl = workloads.make_workload(name, 0, n_layers=1)
    _check_map(sp, wl.coords, wl.grid)


@pytest.mark.parametrize("seed", [1, 2])
def test_map_bit_exact_other_seeds(sp, seed):
    for name in ("tiny", "batched"):
        wl = workloads.make_workload(name, seed, n_layers=1)
        _check_map(sp, wl.coords, wl.grid)
    rng = np.random.default_rng(seed)
    _check_map(sp, workloads.uniform_coords(rng, 64, 30000), (64, 64, 64))


def test_map_kernel_size_one(sp):
    wl = workloads.make_workload("tiny", 0)
    _check_map(sp, wl.coords, wl.grid, kernel_size=1)


def test_map_edge_cases(sp):
    # N = 1
    _check_map(sp, np.array([[0, 3, 3, 3]], np.int32), (8, 8, 8))
    # extent 1 in every axis, several batches
    _check_map(sp, np.array([[b, 0, 0, 0] for b in range(5)], np.int32), (1, 1, 1))
    # grid corners and faces, non-cubic extent, large coordinates
    ext = (65535, 3, 70)
    pts = np.array([[0, 0, 0, 0], [0, 65534, 2, 69], [0, 65533, 2, 69], [0, 1, 0, 0], [7, 65534, 1, 35],
                    [7, 65534, 2, 35], [65535, 0, 0, 0]], np.int32)
    _check_map(sp, pts, ext)
    # fully occupied block (all 26 neighbours present in the interior)
    blk = np.array([[0, x, y, z] for x in range(10) for y in range(10) for z in range(10)], np.int32)
    _check_map(sp, blk[np.random.default_rng(0).permutation(1000)], (10, 10, 10))


def test_map_empty(sp):
    m = sp.spconv_build_map(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4))
    assert m.n == 0 and m.pairs == 0
    assert m.neighbor_map().shape == (0, 27)
    x = torch.zeros((0, 16), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((27, 16, 64), dtype=torch.bfloat16, device="cuda")
    assert sp.spconv_subm_forward(m, x, w).shape == (0, 64)
    m.free()


def test_map_errors(sp):
    dup = np.array([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], np.int32)
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_build_map(coords_dev(dup), (4, 4, 4))
    assert e.value.status == sp.DUPLICATE
    for bad in ([[0, 4, 0, 0]], [[0, 0, -1, 0]], [[-1, 0, 0, 0]], [[65536, 0, 0, 0]]):
        with pytest.raises(sp.SpconvError) as e:
            sp.spconv_build_map(coords_dev(np.array(bad, np.int32)), (4, 4, 4))
        assert e.value.status == sp.COORD_RANGE
    # a forced tiny table fills up
    coords = workloads.uniform_coords(np.random.default_rng(0), 16, 100)
    sp.spconv_debug_set_table_slots(64)
    try:
        with pytest.raises(sp.SpconvError) as e:
            sp.spconv_build_map(coords_dev(coords), (16, 16, 16))
        assert e.value.status == sp.TABLE_FULL
    finally:
        sp.spconv_debug_set_table_slots(0)
    # the library still works afterwards
    _check_map(sp, coords, (16, 16, 16))


def test_tile_height_fills_whole_waves(sp):
    """The map picks the smallest tile that keeps the wave count 384-row tiles need."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3)
    try:
        rows, n = m.tile_rows, wl.n
        waves = -(-n // (384 * sms))
        assert rows <= 384 and -(-n // rows) <= waves * sms
        assert rows == 384 or -(-n // (rows - 1)) > waves * sms
    finally:
        m.free()
