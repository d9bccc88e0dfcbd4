"""The allocation-free neighbour-map build (spconv_build_neighbor_map_noalloc).

It serves callers that cannot call cudaMalloc/cudaFree (another component owns
the device memory, or a latency-critical loop cannot afford cudaFree's device
synchronisation): its hash table lives in a static device array.  These checks
call it through the C ABI and compare its map, bit for bit, with the map of
spconv_build_map, on two calls in a row -- the second call reuses the array the
first one left behind.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sp():
    import submanifold_sparse_convolution_submconv3d_b200 as p
    return p


def _reference(sp, coords_dev, extent):
    m = sp.spconv_build_map(coords_dev, extent, 3)
    try:
        return m.neighbor_map(), m.pairs
    finally:
        m.free()


def test_noalloc_map_equals_build_map_on_two_calls(sp):
    wl = workloads.make_workload("uniform", 0, n_layers=1)           # 209,715 voxels
    small = workloads.uniform_coords(np.random.default_rng(3), 40, 6000)
    cases = [(wl.coords, wl.grid), (small, (40, 40, 40))]
    for coords, extent in cases:
        c = torch.from_numpy(coords).cuda()
        ref, ref_pairs = _reference(sp, c, extent)
        out = torch.full((c.shape[0], 27), 7, dtype=torch.int32, device="cuda")  # caller-owned output
        ext = (ctypes.c_int32 * 3)(*extent)
        pairs = ctypes.c_int64(-1)
        status = sp.lib.spconv_build_neighbor_map_noalloc(c.data_ptr(), c.shape[0], ext, out.data_ptr(),
                                                           ctypes.byref(pairs), torch.cuda.current_stream().cuda_stream)
        assert status == sp.OK, sp.lib.spconv_last_error()
        assert torch.equal(out, ref)
        assert pairs.value == ref_pairs


def test_noalloc_binding_and_limits(sp):
    coords = workloads.uniform_coords(np.random.default_rng(4), 24, 2500)
    c = torch.from_numpy(coords).cuda()
    got, pairs = sp.spconv_build_neighbor_map_noalloc(c, (24, 24, 24))
    ref, ref_pairs = _reference(sp, c, (24, 24, 24))
    assert torch.equal(got, ref) and pairs == ref_pairs
    # errors surface as on the allocating build
    dup = torch.from_numpy(np.array([[0, 1, 1, 1], [0, 1, 1, 1]], np.int32)).cuda()
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_build_neighbor_map_noalloc(dup, (4, 4, 4))
    assert e.value.status == sp.DUPLICATE
    # beyond the static array's limit: rejected before any device work
    ext = (ctypes.c_int32 * 3)(8, 8, 8)
    assert sp.lib.spconv_build_neighbor_map_noalloc(c.data_ptr(), (1 << 19) + 1, ext, None, None, None) == sp.UNSUPPORTED
    assert b"524288" in sp.lib.spconv_last_error()
