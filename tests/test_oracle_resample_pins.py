"""Pins for the oracle's kernel-orientation option, its resampling functions
(SparseDownsample with amax, its paired SparseUpsample, SparseSubdivide) and its
fused decoder epilogue (activation, residual, per-channel statistics).

Each is checked against something other than the oracle itself: torch's CPU
conv3d with the kernel mirrored (a true convolution), torch's dense max_pool3d
and nearest-neighbour interpolate on zero/-inf-filled grids, hand-worked
examples, the pure-Python twins, and invariants that tie the functions together
(downsampling a subdivision gives back the original set and features).
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _offset_index(dx, dy, dz):
    return (dx + 1) * 9 + (dy + 1) * 3 + (dz + 1)


def _random_set(rng, extent, n, batches=1):
    ex, ey, ez = extent
    out = []
    for b in range(batches):
        idx = rng.choice(ex * ey * ez, n, replace=False)
        out.append(np.stack([np.full(n, b), idx // (ey * ez), (idx // ez) % ey, idx % ez], axis=1))
    c = np.concatenate(out).astype(np.int32)
    return c[rng.permutation(c.shape[0])]


# ------------------------------------------------------------------ orientation

def test_flipped_map_is_the_map_with_mirrored_offsets():
    """gather p - d_k is gather p + d_{26-k}: -d_k has index 26 - k."""
    rng = np.random.default_rng(3)
    coords = _random_set(rng, (9, 8, 7), 150, batches=2)
    m = oracle.neighbor_map(coords, (9, 8, 7))
    mf = oracle.neighbor_map(coords, (9, 8, 7), flip=True)
    assert np.array_equal(mf, m[:, ::-1])
    assert np.array_equal(mf[:, 13], np.arange(coords.shape[0]))


def test_flipped_forward_is_a_true_convolution():
    """torch's conv3d is cross-correlation; with the kernel mirrored in all three
    spatial axes it is a true convolution, which the flipped map computes."""
    rng = np.random.default_rng(5)
    extent = (6, 7, 5)
    coords = _random_set(rng, extent, 80)
    x = rng.standard_normal((coords.shape[0], 4))
    w = rng.standard_normal((27, 4, 3))
    bias = rng.standard_normal(3)
    got = oracle.forward(oracle.neighbor_map(coords, extent, flip=True), x, w, bias)
    dense = torch.zeros((1, 4) + extent, dtype=torch.float64)
    c = torch.from_numpy(coords.astype(np.int64))
    dense[0, :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(x).T
    wt = torch.empty((3, 4, 3, 3, 3), dtype=torch.float64)
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                wt[:, :, dx + 1, dy + 1, dz + 1] = torch.from_numpy(w[_offset_index(dx, dy, dz)]).T
    y = torch.nn.functional.conv3d(dense, torch.flip(wt, dims=(2, 3, 4)), torch.from_numpy(bias), padding=1)
    ref = y[0, :, c[:, 1], c[:, 2], c[:, 3]].T.numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_flipped_single_tap_copies_from_the_opposite_side():
    """Voxels (0, t, 2, 2), t = 0..7; W[k] = I at d = (+1, 0, 0) only.  Flipped,
    voxel t receives x of voxel t - 1 (zero at t = 0)."""
    coords = np.array([[0, t, 2, 2] for t in range(8)], dtype=np.int32)
    x = np.arange(8 * 2, dtype=np.float64).reshape(8, 2) + 1.0
    w = np.zeros((27, 2, 2))
    w[_offset_index(1, 0, 0)] = np.eye(2)
    out = oracle.forward(oracle.neighbor_map(coords, (8, 4, 4), flip=True), x, w)
    assert np.array_equal(out[0], [0.0, 0.0])
    assert np.array_equal(out[1:], x[:-1])
    assert np.array_equal(oracle.neighbor_map_py(coords, (8, 4, 4), flip=True),
                          oracle.neighbor_map(coords, (8, 4, 4), flip=True))


# ------------------------------------------------------------------ downsample

def _dense_pool(coords, extent, x, factor):
    """Dense max_pool3d on a grid filled with -inf outside the active voxels
    (ceil mode covers a ragged edge); occupancy by pooling the indicator."""
    b_max = int(coords[:, 0].max()) + 1 if coords.size else 1
    c = torch.from_numpy(coords.astype(np.int64))
    dense = torch.full((b_max, x.shape[1]) + tuple(extent), -np.inf, dtype=torch.float64)
    dense[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(x)
    occ = torch.zeros((b_max, 1) + tuple(extent), dtype=torch.float64)
    occ[c[:, 0], 0, c[:, 1], c[:, 2], c[:, 3]] = 1.0
    pooled = torch.nn.functional.max_pool3d(dense, factor, factor, ceil_mode=True)
    occp = torch.nn.functional.max_pool3d(occ, factor, factor, ceil_mode=True)
    active = torch.nonzero(occp[:, 0] > 0)  # row-major: lexicographic (b, x, y, z)
    vals = pooled[active[:, 0], :, active[:, 1], active[:, 2], active[:, 3]]
    return active.numpy().astype(np.int32), vals.numpy(), tuple(occp.shape[2:])


@pytest.mark.parametrize("seed,extent,n,batches,factor", [
    (0, (8, 8, 8), 60, 1, 2), (1, (9, 7, 5), 120, 2, 2), (2, (10, 10, 10), 300, 3, 3), (3, (5, 6, 7), 40, 1, 1)])
def test_downsample_matches_dense_max_pool(seed, extent, n, batches, factor):
    rng = np.random.default_rng(seed)
    coords = _random_set(rng, extent, n, batches)
    x = rng.standard_normal((coords.shape[0], 5))
    coarse, parent, cext = oracle.downsample(coords, extent, factor)
    got = oracle.downsample_amax(parent, coarse.shape[0], x)
    ref_coords, ref_vals, ref_ext = _dense_pool(coords, extent, x, factor)
    assert cext == ref_ext
    assert np.array_equal(coarse, ref_coords)
    assert np.array_equal(got, ref_vals)


def test_downsample_hand_worked_example():
    """Voxels (0,0,0,0), (0,1,1,1), (0,3,0,0), (1,0,0,1) with factor 2 fall in the
    blocks (0,0,0,0), (0,0,0,0), (0,1,0,0), (1,0,0,0)."""
    coords = np.array([[0, 3, 0, 0], [0, 0, 0, 0], [1, 0, 0, 1], [0, 1, 1, 1]], dtype=np.int32)
    x = np.array([[1.0, -5.0], [2.0, -7.0], [3.0, 4.0], [-1.0, -6.0]])
    coarse, parent, cext = oracle.downsample(coords, (4, 2, 2), 2)
    assert coarse.tolist() == [[0, 0, 0, 0], [0, 1, 0, 0], [1, 0, 0, 0]]
    assert parent.tolist() == [1, 0, 2, 0]
    assert cext == (2, 1, 1)
    got = oracle.downsample_amax(parent, 3, x)
    assert got.tolist() == [[2.0, -6.0], [1.0, -5.0], [3.0, 4.0]]
    c2, p2 = oracle.downsample_py(coords, 2)
    assert np.array_equal(c2, coarse) and np.array_equal(p2, parent)


def test_amax_signed_zero_follows_total_order():
    parent = np.array([0, 0, 1, 1, 2, 2])
    x = np.array([[-0.0], [0.0], [-0.0], [-0.0], [-1.0], [-0.0]])
    got = oracle.downsample_amax(parent, 3, x)[:, 0]
    assert got.tolist() == [0.0, 0.0, 0.0]
    assert np.signbit(got).tolist() == [False, True, True]


def test_downsample_python_twin_on_random_sets():
    rng = np.random.default_rng(9)
    coords = _random_set(rng, (12, 9, 10), 200, batches=2)
    for f in (2, 3, 4):
        c1, p1, _ = oracle.downsample(coords, (12, 9, 10), f)
        c2, p2 = oracle.downsample_py(coords, f)
        assert np.array_equal(c1, c2) and np.array_equal(p1, p2)


def test_downsample_rejects_out_of_range():
    with pytest.raises(oracle.OracleError):
        oracle.downsample(np.array([[0, 4, 0, 0]], dtype=np.int32), (4, 4, 4), 2)
    with pytest.raises(oracle.OracleError):
        oracle.subdivide(np.array([[-1, 0, 0, 0]], dtype=np.int32), (4, 4, 4))


# ------------------------------------------------------------------ upsample

def test_upsample_of_pooled_matches_dense_pool_then_nearest():
    """Pool then upsample: every voxel gets its block's maximum, which a dense
    max_pool3d followed by nearest interpolation back to the fine grid gives."""
    rng = np.random.default_rng(12)
    extent = (8, 6, 10)
    coords = _random_set(rng, extent, 150)
    x = rng.standard_normal((coords.shape[0], 3))
    coarse, parent, _ = oracle.downsample(coords, extent, 2)
    got = oracle.upsample(parent, oracle.downsample_amax(parent, coarse.shape[0], x))
    c = torch.from_numpy(coords.astype(np.int64))
    dense = torch.full((1, 3) + extent, -np.inf, dtype=torch.float64)
    dense[0, :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(x).T
    back = torch.nn.functional.interpolate(torch.nn.functional.max_pool3d(dense, 2, 2), scale_factor=2,
                                           mode="nearest")
    ref = back[0, :, c[:, 1], c[:, 2], c[:, 3]].T.numpy()
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ subdivide

def test_subdivide_hand_worked_example():
    coords = np.array([[2, 1, 0, 3]], dtype=np.int32)
    out, xo = oracle.subdivide(coords, (2, 1, 4), np.array([[7.0, 8.0]]))
    assert out.tolist() == [[2, 2, 0, 6], [2, 2, 0, 7], [2, 2, 1, 6], [2, 2, 1, 7],
                            [2, 3, 0, 6], [2, 3, 0, 7], [2, 3, 1, 6], [2, 3, 1, 7]]
    assert xo.tolist() == [[7.0, 8.0]] * 8


def test_subdivide_matches_dense_nearest_interpolation():
    rng = np.random.default_rng(14)
    extent = (5, 4, 6)
    coords = _random_set(rng, extent, 50)
    x = rng.standard_normal((coords.shape[0], 2))
    out, xo = oracle.subdivide(coords, extent, x)
    c = torch.from_numpy(coords.astype(np.int64))
    dense = torch.zeros((1, 2) + extent, dtype=torch.float64)
    dense[0, :, c[:, 1], c[:, 2], c[:, 3]] = torch.from_numpy(x).T
    up = torch.nn.functional.interpolate(dense, scale_factor=2, mode="nearest")
    o = torch.from_numpy(out.astype(np.int64))
    assert np.array_equal(xo, up[0, :, o[:, 1], o[:, 2], o[:, 3]].T.numpy())
    # the children are distinct and fill exactly the 2x2x2 blocks of the voxels
    assert np.unique(out, axis=0).shape[0] == 8 * coords.shape[0]
    assert np.array_equal(out[:, 1:] // 2, np.repeat(coords[:, 1:], 8, axis=0))


def test_downsample_inverts_subdivide():
    rng = np.random.default_rng(15)
    extent = (7, 9, 6)
    coords = _random_set(rng, extent, 90, batches=2)
    x = rng.standard_normal((coords.shape[0], 4))
    fine, xf = oracle.subdivide(coords, extent, x)
    coarse, parent, cext = oracle.downsample(fine, tuple(2 * e for e in extent), 2)
    order = np.lexsort(coords.T[::-1])
    assert cext == extent
    assert np.array_equal(coarse, coords[order])
    assert np.array_equal(oracle.downsample_amax(parent, coarse.shape[0], xf), x[order])


# ------------------------------------------------------------------ epilogue

@pytest.mark.parametrize("act", ["relu", "silu", "gelu"])
def test_activations_match_torch(act):
    y = np.concatenate([np.linspace(-12, 12, 2001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]])
    got = oracle.activation(act, y)
    t = torch.from_numpy(y)
    ref = {"relu": torch.nn.functional.relu, "silu": torch.nn.functional.silu,
           "gelu": lambda v: torch.nn.functional.gelu(v, approximate="none")}[act](t).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-15)


def test_activation_hand_values():
    assert oracle.activation("relu", [-2.0, 3.0]).tolist() == [0.0, 3.0]
    assert oracle.activation("silu", [0.0])[0] == 0.0
    assert abs(oracle.activation("silu", [1.0])[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(oracle.activation("gelu", [1.0])[0] - 0.8413447460685429) < 1e-15  # 1 * Phi(1)
    assert oracle.activation("none", [-5.0])[0] == -5.0
    with pytest.raises(ValueError):
        oracle.activation("tanh", [0.0])


def test_epilogue_order_and_residual():
    """act applies to conv + bias, then the residual is added: relu(-1) + 5 = 5, not relu(4)."""
    conv = np.array([[-1.0, 2.0]])
    res = np.array([[5.0, -3.0]])
    assert oracle.epilogue(conv, "relu", res).tolist() == [[5.0, -1.0]]
    assert oracle.epilogue(conv, "none", None).tolist() == [[-1.0, 2.0]]


def test_residual_conv_equals_conv_of_identity_tap_plus_conv():
    """A residual x added to conv(x, W) equals conv(x, W') with W'[13] = W[13] + I
    (the centre tap sees the voxel itself): an identity of the definition."""
    rng = np.random.default_rng(22)
    coords = _random_set(rng, (6, 6, 6), 60)
    x = rng.standard_normal((60, 4))
    w = rng.standard_normal((27, 4, 4))
    nbr = oracle.neighbor_map(coords, (6, 6, 6))
    lhs = oracle.epilogue(oracle.forward(nbr, x, w), "none", x)
    w2 = w.copy()
    w2[13] += np.eye(4)
    np.testing.assert_allclose(lhs, oracle.forward(nbr, x, w2), rtol=1e-12, atol=1e-12)


def test_channel_stats_match_torch_moments():
    rng = np.random.default_rng(23)
    out = rng.standard_normal((500, 7))
    s = oracle.channel_stats(out)
    t = torch.from_numpy(out)
    n = out.shape[0]
    np.testing.assert_allclose(s[0] / n, t.mean(dim=0).numpy(), rtol=1e-12, atol=1e-14)
    var = s[1] / n - (s[0] / n) ** 2
    np.testing.assert_allclose(var, t.var(dim=0, unbiased=False).numpy(), rtol=1e-9, atol=1e-12)
    assert oracle.channel_stats(np.array([[1.0, -2.0], [3.0, 4.0]])).tolist() == [[4.0, 2.0], [10.0, 20.0]]
