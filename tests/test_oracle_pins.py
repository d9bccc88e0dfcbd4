"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test fixes the oracle to something the pages or the mathematics decide:
dense brute-force cross-correlation on a zero-filled grid, torch's CPU conv3d
(a library cross-correlation), closed forms for special weights and special
coordinate sets, invariants (permutation, linearity, map symmetry), the
closed-form expected hit count of uniform occupancy, and the numbers printed in
the lato.2_mrp_mlx README's "Fleet benchmark" table.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _offset_index(dx, dy, dz):
    return (dx + 1) * 9 + (dy + 1) * 3 + (dz + 1)


def _random_sparse(rng, extent, n, batches=1, cin=3, cout=4):
    ex, ey, ez = extent
    cells = ex * ey * ez
    coords = []
    for b in range(batches):
        idx = rng.choice(cells, n, replace=False)
        c = np.stack([np.full(n, b), idx // (ey * ez), (idx // ez) % ey, idx % ez], axis=1)
        coords.append(c)
    coords = np.concatenate(coords).astype(np.int32)
    coords = coords[rng.permutation(coords.shape[0])]
    x = rng.standard_normal((coords.shape[0], cin))
    w = rng.standard_normal((27, cin, cout))
    bias = rng.standard_normal(cout)
    return coords, x, w, bias


def _dense_brute_force(coords, extent, x, w, bias):
    """Zero-filled dense grid, cross-correlate every cell, read active cells."""
    nb = int(coords[:, 0].max()) + 1
    ex, ey, ez = extent
    cin, cout = w.shape[1], w.shape[2]
    grid = np.zeros((nb, ex + 2, ey + 2, ez + 2, cin))
    grid[coords[:, 0], coords[:, 1] + 1, coords[:, 2] + 1, coords[:, 3] + 1] = x
    full = np.zeros((nb, ex, ey, ez, cout))
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                shifted = grid[:, 1 + dx:1 + dx + ex, 1 + dy:1 + dy + ey, 1 + dz:1 + dz + ez, :]
                full += shifted @ w[_offset_index(dx, dy, dz)]
    full += bias
    return full[coords[:, 0], coords[:, 1], coords[:, 2], coords[:, 3]]


@pytest.mark.parametrize("seed,extent,n,batches", [
    (0, (6, 6, 6), 60, 1),
    (1, (5, 7, 4), 140, 1),   # all-active grid
    (2, (8, 8, 8), 200, 2),
    (3, (4, 4, 4), 1, 1),
])
def test_oracle_matches_dense_brute_force(seed, extent, n, batches):
    rng = np.random.default_rng(seed)
    coords, x, w, bias = _random_sparse(rng, extent, n, batches)
    got = oracle.subm_conv3d(coords, extent, x, w, bias)
    ref = _dense_brute_force(coords, extent, x, w, bias)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_oracle_matches_torch_conv3d(seed):
    """torch.nn.functional.conv3d is cross-correlation; with padding 1 and the
    output read at active sites it is SubMConv3d on a zero-filled grid."""
    rng = np.random.default_rng(100 + seed)
    extent = (7, 6, 8)
    coords, x, w, bias = _random_sparse(rng, extent, 90, 1, cin=5, cout=3)
    got = oracle.subm_conv3d(coords, extent, x, w, bias)
    dense = torch.zeros((1, 5) + extent, dtype=torch.float64)
    c = torch.from_numpy(coords.astype(np.int64))
    dense[0, :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(x).T
    wt = torch.empty((3, 5, 3, 3, 3), dtype=torch.float64)
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                wt[:, :, dx + 1, dy + 1, dz + 1] = torch.from_numpy(w[_offset_index(dx, dy, dz)]).T
    y = torch.nn.functional.conv3d(dense, wt, torch.from_numpy(bias), padding=1)
    ref = y[0, :, c[:, 1], c[:, 2], c[:, 3]].T.numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_kernel_size_one_is_a_per_voxel_linear_map():
    rng = np.random.default_rng(7)
    coords, x, _, bias = _random_sparse(rng, (9, 9, 9), 120, 1, cin=6, cout=5)
    w1 = rng.standard_normal((1, 6, 5))
    nbr = oracle.neighbor_map(coords, (9, 9, 9), 1)
    assert np.array_equal(nbr[:, 0], np.arange(coords.shape[0]))
    got = oracle.forward(nbr, x, w1, bias)
    np.testing.assert_allclose(got, x @ w1[0] + bias, rtol=1e-13, atol=1e-13)


def test_single_tap_weights_give_exact_shifted_copies():
    """A line of voxels (0, t, 5, 5), t = 0..9, stored shuffled.  With W[k] = I at
    one offset and zero elsewhere, out at voxel t is x at voxel t + d (or zero).
    Pins the orientation (gather p + d) and the offset order (dx slowest)."""
    rng = np.random.default_rng(11)
    order = rng.permutation(10)
    coords = np.array([[0, t, 5, 5] for t in order], dtype=np.int32)
    x = rng.standard_normal((10, 4))
    row_of_t = {int(t): i for i, t in enumerate(order)}
    for d in [(1, 0, 0), (-1, 0, 0)]:
        w = np.zeros((27, 4, 4))
        w[_offset_index(*d)] = np.eye(4)
        out = oracle.subm_conv3d(coords, (16, 16, 16), x, w)
        for i, t in enumerate(order):
            src = int(t) + d[0]
            expect = x[row_of_t[src]] if 0 <= src < 10 else np.zeros(4)
            assert np.array_equal(out[i], expect)
    # The same along y and z, and one diagonal, on a 3x3x3 block fully active.
    block = np.array([[0, a, b, c] for a in range(3) for b in range(3) for c in range(3)], dtype=np.int32)
    perm = rng.permutation(27)
    block = block[perm]
    xb = rng.standard_normal((27, 2))
    where = {tuple(int(v) for v in block[i, 1:]): i for i in range(27)}
    for d in [(0, 1, 0), (0, 0, 1), (0, 0, -1), (-1, 1, 0), (1, -1, 1)]:
        w = np.zeros((27, 2, 2))
        w[_offset_index(*d)] = np.eye(2)
        out = oracle.subm_conv3d(block, (3, 3, 3), xb, w)
        for i in range(27):
            p = tuple(int(v) + dd for v, dd in zip(block[i, 1:], d))
            expect = xb[where[p]] if p in where else np.zeros(2)
            assert np.array_equal(out[i], expect)


def test_hand_worked_two_voxel_example():
    """Two voxels (0,1,1,1) and (0,2,1,1); Cin = Cout = 1; W[k] = k + 1; x = [1, 10].
    Voxel 0 sees itself (k=13, weight 14) and voxel 1 at d=(+1,0,0) (k=22, weight 23):
    14*1 + 23*10 = 244.  Voxel 1 sees itself (14) and voxel 0 at d=(-1,0,0) (k=4,
    weight 5): 14*10 + 5*1 = 145.  With bias 0.5 both shift by 0.5."""
    coords = np.array([[0, 1, 1, 1], [0, 2, 1, 1]], dtype=np.int32)
    w = (np.arange(27, dtype=np.float64) + 1).reshape(27, 1, 1)
    x = np.array([[1.0], [10.0]])
    out = oracle.subm_conv3d(coords, (4, 4, 4), x, w, np.array([0.5]))
    assert out[:, 0].tolist() == [244.5, 145.5]
    nbr = oracle.neighbor_map(coords, (4, 4, 4))
    assert nbr[0].tolist() == [-1] * 13 + [0] + [-1] * 8 + [1] + [-1] * 4
    assert nbr[1].tolist() == [-1] * 4 + [0] + [-1] * 8 + [1] + [-1] * 13


def test_isolated_voxel_uses_centre_tap_only():
    coords = np.array([[0, 0, 0, 0], [0, 5, 5, 5], [0, 2, 2, 2]], dtype=np.int32)
    nbr = oracle.neighbor_map(coords, (8, 8, 8))
    for i in range(3):
        assert nbr[i].tolist() == [-1] * 13 + [i] + [-1] * 13
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 4))
    w = rng.standard_normal((27, 4, 2))
    b = rng.standard_normal(2)
    np.testing.assert_allclose(oracle.forward(nbr, x, w, b), x @ w[13] + b, rtol=1e-13)


def test_batch_isolation():
    """Two batch items with identical xyz sets never see each other; each item's
    output equals that item convolved alone."""
    rng = np.random.default_rng(5)
    coords0, x0, w, bias = _random_sparse(rng, (6, 6, 6), 80, 1)
    coords1 = coords0.copy()
    coords1[:, 0] = 1
    x1 = rng.standard_normal(x0.shape)
    coords = np.concatenate([coords0, coords1])
    x = np.concatenate([x0, x1])
    nbr = oracle.neighbor_map(coords, (6, 6, 6))
    n0 = coords0.shape[0]
    assert np.all((nbr[:n0] < n0)) and np.all((nbr[n0:] == -1) | (nbr[n0:] >= n0))
    out = oracle.forward(nbr, x, w, bias)
    np.testing.assert_allclose(out[:n0], oracle.subm_conv3d(coords0, (6, 6, 6), x0, w, bias), rtol=1e-13)
    np.testing.assert_allclose(out[n0:], oracle.subm_conv3d(coords1, (6, 6, 6), x1, w, bias), rtol=1e-13)


def test_permutation_invariance():
    rng = np.random.default_rng(9)
    coords, x, w, bias = _random_sparse(rng, (10, 10, 10), 300, 2)
    out = oracle.subm_conv3d(coords, (10, 10, 10), x, w, bias)
    perm = rng.permutation(coords.shape[0])
    out_p = oracle.subm_conv3d(coords[perm], (10, 10, 10), x[perm], w, bias)
    np.testing.assert_allclose(out_p, out[perm], rtol=1e-12, atol=1e-12)
    nbr = oracle.neighbor_map(coords, (10, 10, 10))
    nbr_p = oracle.neighbor_map(coords[perm], (10, 10, 10))
    inv = np.argsort(perm)
    expect = np.where(nbr[perm] >= 0, inv[np.maximum(nbr[perm], 0)], -1)
    assert np.array_equal(nbr_p, expect)


def test_linearity():
    rng = np.random.default_rng(13)
    coords, x1, w, _ = _random_sparse(rng, (7, 7, 7), 100, 1)
    x2 = rng.standard_normal(x1.shape)
    w2 = rng.standard_normal(w.shape)
    nbr = oracle.neighbor_map(coords, (7, 7, 7))
    a = oracle.forward(nbr, x1 + 2.0 * x2, w)
    b = oracle.forward(nbr, x1, w) + 2.0 * oracle.forward(nbr, x2, w)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)
    c = oracle.forward(nbr, x1, w + w2)
    d = oracle.forward(nbr, x1, w) + oracle.forward(nbr, x1, w2)
    np.testing.assert_allclose(c, d, rtol=1e-11, atol=1e-11)


def _check_symmetry(nbr):
    n = nbr.shape[0]
    i, k = np.nonzero(nbr >= 0)
    j = nbr[i, k]
    assert np.all(nbr[j, 26 - k] == i)
    assert np.all(nbr[np.arange(n), 13] == np.arange(n))


def test_map_symmetry_on_workloads():
    for name in ("tiny", "uniform"):
        wl = workloads.make_workload(name, 0, n_layers=1)
        _check_symmetry(oracle.neighbor_map(wl.coords, wl.grid))
    rng = np.random.default_rng(1)
    coords = workloads.shell_coords(rng, 64, 4, 5.0, 25.0)
    _check_symmetry(oracle.neighbor_map(coords, (64, 64, 64)))


def _expected_hits(n, g):
    """E[pairs per voxel] for n voxels uniform without replacement in a g^3 grid:
    1 + sum_{d != 0} (n-1)/(g^3-1) * prod_a (1 - |d_a|/g)."""
    s = 0.0
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                if (dx, dy, dz) == (0, 0, 0):
                    continue
                s += (1 - abs(dx) / g) * (1 - abs(dy) / g) * (1 - abs(dz) / g)
    return 1.0 + (n - 1) / (g ** 3 - 1) * s


def test_hit_rate_matches_closed_form_uniform():
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    nbr = oracle.neighbor_map(wl.coords, wl.grid)
    measured = (nbr >= 0).sum() / wl.n
    expected = _expected_hits(wl.n, 128)
    assert abs(expected - 3.558) < 1e-3
    assert abs(measured - expected) < 0.01, (measured, expected)
    # smaller grids over several seeds: the mean over seeds is tight
    vals = []
    for seed in range(8):
        rng = np.random.default_rng(seed)
        coords = workloads.uniform_coords(rng, 24, 2000)
        vals.append((oracle.neighbor_map(coords, (24, 24, 24)) >= 0).sum() / 2000)
    assert abs(np.mean(vals) - _expected_hits(2000, 24)) < 0.03


def test_errors_out_of_range_and_duplicates():
    good = np.array([[0, 1, 2, 3], [0, 3, 2, 1]], dtype=np.int32)
    assert oracle.neighbor_map(good, (4, 4, 4)).shape == (2, 27)
    for bad in ([[0, 4, 0, 0]], [[0, 0, -1, 0]], [[-1, 0, 0, 0]], [[65536, 0, 0, 0]]):
        with pytest.raises(oracle.OracleError) as e:
            oracle.neighbor_map(np.array(bad, dtype=np.int32), (4, 4, 4))
        assert e.value.code == oracle.COORD_RANGE
    dup = np.array([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], dtype=np.int32)
    with pytest.raises(oracle.OracleError) as e:
        oracle.neighbor_map(dup, (4, 4, 4))
    assert e.value.code == oracle.DUPLICATE
    with pytest.raises(oracle.OracleError):
        oracle.neighbor_map(good, (4, 4, 4), kernel_size=5)
    assert oracle.neighbor_map(np.zeros((0, 4), np.int32), (4, 4, 4)).shape == (0, 27)


def test_grid_edge_neighbours_are_holes():
    coords = np.array([[0, 0, 0, 0], [0, 2, 2, 2]], dtype=np.int32)
    nbr = oracle.neighbor_map(coords, (3, 3, 3))
    assert (nbr[0] >= 0).sum() == 1 and (nbr[1] >= 0).sum() == 1
    # extent 1 in every axis: a single cell, its own centre only
    one = np.array([[0, 0, 0, 0], [1, 0, 0, 0]], dtype=np.int32)
    nb1 = oracle.neighbor_map(one, (1, 1, 1))
    assert nb1.tolist() == [[-1] * 13 + [0] + [-1] * 13, [-1] * 13 + [1] + [-1] * 13]


def test_python_twin_agrees_with_c_oracle_on_tiny():
    wl = workloads.make_workload("tiny", 0)
    nbr_c = oracle.neighbor_map(wl.coords, wl.grid)
    nbr_py = oracle.neighbor_map_py(wl.coords, wl.grid)
    assert np.array_equal(nbr_c, nbr_py)
    l3 = wl.layers[0]
    np.testing.assert_allclose(oracle.forward(nbr_c, wl.x, l3.w, l3.bias),
                               oracle.forward_py(nbr_py, wl.x, l3.w, l3.bias), rtol=1e-12, atol=1e-12)


def test_row_subset_matches_full_forward():
    rng = np.random.default_rng(21)
    coords, x, w, bias = _random_sparse(rng, (9, 9, 9), 150, 1)
    nbr = oracle.neighbor_map(coords, (9, 9, 9))
    full = oracle.forward(nbr, x, w, bias)
    rows = rng.choice(150, 17, replace=False)
    assert np.array_equal(oracle.forward(nbr, x, w, bias, rows=rows), full[rows])


def _read_fleet_table():
    rows, meta = [], {}
    with open(os.path.join(GOLDEN, "fleet_benchmark.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.replace('"', "").split()
            if len(parts) == 2:
                meta[parts[0]] = int(parts[1])
            else:
                rows.append((parts[0], int(parts[-3]), float(parts[-2]), float(parts[-1])))
    return meta, rows


def test_pages_fleet_table_defines_mvox_metric():
    """Mvox/s in the pages' table is active voxels / conv seconds / 1e6 at
    N = 209,715 = floor(10 % of 128^3); the uniform workload draws exactly that."""
    meta, rows = _read_fleet_table()
    n = meta["active_voxels"]
    assert n == math.floor(0.1 * meta["grid"] ** 3)
    assert len(rows) == 4
    for box, cores, conv_ms, mvox in rows:
        implied_ms = n / (mvox * 1e6) * 1e3
        slack = 0.05 + implied_ms * 0.005 / mvox
        assert abs(implied_ms - conv_ms) <= slack, (box, implied_ms, conv_ms)
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    assert wl.n == n and wl.grid == (128, 128, 128) and wl.x.shape[1] == meta["channels"]
