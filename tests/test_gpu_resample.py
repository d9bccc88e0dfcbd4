"""GPU resampling ops vs the CPU oracle, bit for bit: SparseDownsample coordinates
and amax pooling, the paired SparseUpsample, SparseSubdivide, and a convolution
on each new coordinate set through a freshly built map."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import assert_close, coords_dev, oracle_forward_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sp():
    import submanifold_sparse_convolution_submconv3d_b200 as p
    return p


def _bits(t: torch.Tensor) -> np.ndarray:
    """Raw bits of a float tensor (so -0 and +0 differ)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy()
    return t.view(torch.int32).cpu().numpy()


def _ref_bits(a: np.ndarray, dtype) -> np.ndarray:
    return _bits(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dtype))


def _check_downsample(sp, coords, extent, factor, channels=(), dtypes=(torch.bfloat16,), seed=0):
    ds = sp.spconv_downsample_build(coords_dev(coords), extent, factor)
    try:
        coarse, parent, cext = oracle.downsample(coords, extent, factor)
        assert ds.n == coords.shape[0] and ds.n_coarse == coarse.shape[0]
        assert ds.coarse_extent == cext
        assert np.array_equal(ds.coarse_coords().cpu().numpy(), coarse)
        assert np.array_equal(ds.parent().cpu().numpy(), parent)
        rng = np.random.default_rng(seed)
        for c in channels:
            for dt in dtypes:
                x = rng.standard_normal((coords.shape[0], c)).astype(np.float32)
                xd = torch.from_numpy(x).cuda().to(dt)
                xr = xd.double().cpu().numpy()
                pooled = sp.spconv_downsample_amax(ds, xd)
                ref = oracle.downsample_amax(parent, coarse.shape[0], xr)
                assert np.array_equal(_bits(pooled), _ref_bits(ref, dt)), (c, dt)
                up = sp.spconv_upsample(ds, pooled)
                assert np.array_equal(_bits(up), _bits(pooled)[parent] if parent.size else _bits(up))
    finally:
        ds.free()


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
def test_downsample_bit_exact_on_workloads(sp, name):
    wl = workloads.make_workload(name, 0, n_layers=1)
    ch = (16, 3) if name == "tiny" else ((128, 5) if name in ("uniform", "batched") else (64,))
    dts = (torch.float32, torch.bfloat16) if name in ("tiny", "batched") else (torch.bfloat16,)
    _check_downsample(sp, wl.coords, wl.grid, 2, ch, dts)


@pytest.mark.parametrize("factor", [1, 3, 4])
def test_downsample_other_factors(sp, factor):
    wl = workloads.make_workload("batched", 0, n_layers=1)
    _check_downsample(sp, wl.coords, wl.grid, factor, (8,), (torch.float32, torch.bfloat16))


def test_downsample_edge_cases(sp):
    # n = 0
    ds = sp.spconv_downsample_build(torch.empty((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4), 2)
    assert ds.n == 0 and ds.n_coarse == 0
    out = sp.spconv_downsample_amax(ds, torch.empty((0, 8), device="cuda"))
    assert out.shape == (0, 8)
    ds.free()
    # one voxel; one full block of 8; odd extents (ragged coarse edge); several batches
    _check_downsample(sp, np.array([[3, 4, 0, 6]], np.int32), (5, 1, 7), 2, (4, 8), (torch.float32, torch.bfloat16))
    block = np.array([[0, a, b, c] for a in (2, 3) for b in (4, 5) for c in (0, 1)], np.int32)[::-1].copy()
    _check_downsample(sp, block, (6, 6, 6), 2, (8, 2), (torch.float32, torch.bfloat16))
    rng = np.random.default_rng(4)
    pts = np.unique(np.stack([rng.integers(0, 4, 3000), rng.integers(0, 9, 3000), rng.integers(0, 7, 3000),
                              rng.integers(0, 5, 3000)], 1), axis=0).astype(np.int32)
    pts = pts[rng.permutation(pts.shape[0])]
    _check_downsample(sp, pts, (9, 7, 5), 2, (24, 7), (torch.float32, torch.bfloat16))


def test_amax_signed_zeros_and_ties(sp):
    coords = np.array([[0, 0, 0, 0], [0, 1, 0, 0], [0, 2, 0, 0], [0, 3, 0, 0], [0, 4, 0, 0], [0, 5, 0, 0]], np.int32)
    x = np.array([[-0.0, -1.0, 2.0, -0.0], [0.0, -1.0, 2.0, -0.0], [-0.0, -3.0, 1.0, -0.0],
                  [-0.0, -2.0, 1.0, -0.0], [-1.0, -0.0, -5.0, 0.0], [-0.0, -7.0, -5.0, -0.0]])
    for dt in (torch.float32, torch.bfloat16):
        ds = sp.spconv_downsample_build(coords_dev(coords), (6, 1, 1), 2)
        pooled = sp.spconv_downsample_amax(ds, torch.from_numpy(x).float().cuda().to(dt))
        coarse, parent, _ = oracle.downsample(coords, (6, 1, 1), 2)
        ref = oracle.downsample_amax(parent, coarse.shape[0], x)
        assert np.array_equal(_bits(pooled), _ref_bits(ref, dt))
        ds.free()


def test_downsample_errors(sp):
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_downsample_build(coords_dev(np.array([[0, 4, 0, 0]], np.int32)), (4, 4, 4), 2)
    assert e.value.status == sp.COORD_RANGE
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_downsample_build(coords_dev(np.array([[0, 1, 0, 0]], np.int32)), (4, 4, 4), 0)
    assert e.value.status == sp.INVALID_ARG


@pytest.mark.parametrize("name", ["tiny", "shells", "batched"])
def test_subdivide_bit_exact(sp, name):
    wl = workloads.make_workload(name, 0, n_layers=1)
    for dt, c in ((torch.bfloat16, 64), (torch.float32, 3), (torch.bfloat16, 5)):
        x = np.random.default_rng(1).standard_normal((wl.n, c)).astype(np.float32)
        xd = torch.from_numpy(x).cuda().to(dt)
        co, xo = sp.spconv_subdivide(coords_dev(wl.coords), wl.grid, xd)
        ref_c, ref_x = oracle.subdivide(wl.coords, wl.grid, xd.double().cpu().numpy())
        assert np.array_equal(co.cpu().numpy(), ref_c)
        assert np.array_equal(_bits(xo), _ref_bits(ref_x, dt))
    co, xo = sp.spconv_subdivide(coords_dev(wl.coords), wl.grid)
    assert xo is None and np.array_equal(co.cpu().numpy(), oracle.subdivide(wl.coords, wl.grid)[0])


def test_subdivide_edge_cases_and_errors(sp):
    co, xo = sp.spconv_subdivide(torch.empty((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4),
                                 torch.empty((0, 8), device="cuda"))
    assert co.shape == (0, 4) and xo.shape == (0, 8)
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_subdivide(coords_dev(np.array([[0, 1, 1, 1]], np.int32)), (32768, 4, 4))
    assert e.value.status == sp.INVALID_ARG
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_subdivide(coords_dev(np.array([[0, 1, 4, 1]], np.int32)), (4, 4, 4))
    assert e.value.status == sp.COORD_RANGE
    one = np.array([[9, 32766, 0, 5]], np.int32)
    co, _ = sp.spconv_subdivide(coords_dev(one), (32767, 1, 6))
    assert np.array_equal(co.cpu().numpy(), oracle.subdivide(one, (32767, 1, 6))[0])


def test_convolution_after_each_coordinate_change(sp):
    """shells: downsample(2) -> new map -> conv, and subdivide -> new map -> conv,
    each against the oracle on the new coordinate set."""
    wl = workloads.make_workload("shells", 0, n_layers=1)
    rng = np.random.default_rng(31)
    w = (rng.standard_normal((27, 64, 64)) / np.sqrt(27 * 64)).astype(np.float32)
    wd = to_dev(w, "bf16")
    wr = wd.double().cpu().numpy()
    xd = to_dev(wl.x, "bf16")
    ds = sp.spconv_downsample_build(coords_dev(wl.coords), wl.grid, 2)
    pooled = sp.spconv_downsample_amax(ds, xd)
    cm = sp.spconv_build_map(ds.coarse_coords(), ds.coarse_extent, 3)
    out = sp.spconv_subm_forward(cm, pooled, wd)
    cm.check()
    coarse, parent, cext = oracle.downsample(wl.coords, wl.grid, 2)
    ref = oracle_forward_rows(oracle, oracle.neighbor_map(coarse, cext), pooled.double().cpu().numpy(), wr, None)
    assert_close(out, ref, "bf16", label="downsample -> conv")
    cm.free()
    # subdivide the coarse set back up and convolve there
    co, xo = sp.spconv_subdivide(ds.coarse_coords(), ds.coarse_extent, out)
    fext = tuple(2 * e for e in ds.coarse_extent)
    fm = sp.spconv_build_map(co, fext, 3)
    rows = np.random.default_rng(0).choice(co.shape[0], 40000, replace=False)
    out2 = sp.spconv_subm_forward(fm, xo, wd)
    fm.check()
    ref_c, _ = oracle.subdivide(coarse, cext)
    ref2 = oracle_forward_rows(oracle, oracle.neighbor_map(ref_c, fext), xo.double().cpu().numpy(), wr, None, rows)
    assert_close(out2[torch.from_numpy(rows).cuda()], ref2, "bf16", label="subdivide -> conv")
    fm.free()
    ds.free()
