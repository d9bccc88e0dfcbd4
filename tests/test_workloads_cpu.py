"""Pins of the seeded input generators (CPU).

Both sides of every parity test draw their inputs from workloads.py.  A mistake
here would reach both sides at once and go unnoticed by parity.  So each
generator is checked against an independent statement of its recipe: torch's
bf16 rounding, a brute-force shell over a whole grid, and the coordinate recipes
of the workloads."""
import numpy as np
import torch

import workloads


def test_round_to_bf16_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # exact ties: finite normal values whose low 16 bits are 0x8000, with both
    # parities of the last kept bit
    exp = rng.integers(100, 155, 4000, dtype=np.uint32) << np.uint32(23)
    mant = rng.integers(0, 128, 4000, dtype=np.uint32) << np.uint32(16)
    ties = (exp | mant | np.uint32(0x8000)).view(np.float32)
    assert np.all(np.isfinite(ties))
    a = np.concatenate([a, ties, -ties, np.float32([0.0, -0.0, 1.0, 65504.0])])
    ref = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    got = workloads.round_to_bf16(a)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_uniform_coords_recipe():
    rng = np.random.default_rng(3)
    c = workloads.uniform_coords(rng, 16, 410, batch=2)
    idx = np.random.default_rng(3).choice(16 ** 3, 410, replace=False)  # the recipe's draw, in draw order
    assert c.dtype == np.int32 and c.shape == (410, 4)
    assert np.all(c[:, 0] == 2)
    assert np.array_equal(c[:, 1] * 256 + c[:, 2] * 16 + c[:, 3], idx)  # x slowest, z fastest
    assert len({tuple(r) for r in c.tolist()}) == 410


def _brute_shell(grid, c, r):
    """Every voxel of [0, grid)^3 with f <= 1 and a 6-neighbour (in or out of the grid) with f > 1."""
    ax = np.arange(-1, grid + 1, dtype=np.float64)
    f = (((ax - c[0]) / r[0]) ** 2)[:, None, None] + (((ax - c[1]) / r[1]) ** 2)[None, :, None] \
        + (((ax - c[2]) / r[2]) ** 2)[None, None, :]
    core = f[1:-1, 1:-1, 1:-1]
    out_nb = ((f[:-2, 1:-1, 1:-1] > 1) | (f[2:, 1:-1, 1:-1] > 1) | (f[1:-1, :-2, 1:-1] > 1)
              | (f[1:-1, 2:, 1:-1] > 1) | (f[1:-1, 1:-1, :-2] > 1) | (f[1:-1, 1:-1, 2:] > 1))
    return {tuple(p) for p in np.argwhere((core <= 1) & out_nb).tolist()}


def test_ellipsoid_shell_matches_brute_force():
    rng = np.random.default_rng(5)
    grid = 28
    cases = [(np.array([14.0, 14.0, 14.0]), np.array([6.0, 6.0, 6.0])),        # sphere
             (np.array([13.3, 15.7, 12.1]), np.array([9.5, 4.2, 7.7])),         # ellipsoid
             (np.array([2.5, 20.0, 26.5]), np.array([8.0, 5.0, 9.0])),          # clipped by the grid
             (np.array([14.0, 14.0, 14.0]), np.array([0.6, 0.6, 0.6]))]         # a single voxel
    for _ in range(4):
        cases.append((rng.uniform(0, grid, 3), rng.uniform(1.5, 12.0, 3)))
    for c, r in cases:
        got = {tuple(p) for p in workloads._ellipsoid_shell(grid, c, r).tolist()}
        assert got == _brute_shell(grid, c, r), (c, r)


def test_shell_coords_are_unique_sorted_union():
    rng = np.random.default_rng(7)
    c = workloads.shell_coords(rng, 48, 3, 4.0, 15.0, batch=1)
    assert np.all(c[:, 0] == 1)
    keys = [tuple(r) for r in c[:, 1:].tolist()]
    assert keys == sorted(set(keys))
    # the union of the three shells, drawn in the documented order (centre, then semi-axes)
    rng = np.random.default_rng(7)
    union = set()
    for _ in range(3):
        ctr = rng.uniform(12.0, 36.0, size=3)
        r = rng.uniform(4.0, 15.0, size=3)
        union |= _brute_shell(48, ctr, r)
    assert set(keys) == union


def test_workloads_are_deterministic_and_bf16_exact():
    for name in ("tiny", "batched"):
        a, b = workloads.make_workload(name, 1), workloads.make_workload(name, 1)
        assert np.array_equal(a.coords, b.coords) and np.array_equal(a.x, b.x)
        for la, lb in zip(a.layers, b.layers):
            assert np.array_equal(la.w, lb.w) and np.array_equal(la.bias, lb.bias)
    wl = workloads.make_workload("batched", 0)
    assert sorted(set(wl.coords[:, 0].tolist())) == [0, 1, 2, 3]
    assert [(l.kernel_size, l.w.shape) for l in wl.layers] == [(3, (27, 512, 512)), (1, (1, 512, 512))]
    for arr in [wl.x] + [l.w for l in wl.layers] + [l.bias for l in wl.layers]:
        assert np.array_equal(workloads.round_to_bf16(arr), arr)  # every side sees the same exact values
    tiny = workloads.make_workload("tiny", 0)
    assert tiny.n == 410 and tiny.x.dtype == np.float32 and tiny.dtype == "f32"
    # weight standard deviation (27 Cin)^-1/2: the variance reading of N(0, 1/(27 C))
    assert abs(wl.layers[0].w.std() * np.sqrt(27 * 512) - 1.0) < 0.01
