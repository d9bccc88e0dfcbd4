"""GPU map-build options vs the CPU oracle: the mirrored kernel orientation and
the sorted-key dictionary.  Maps bit-exact; forwards on them within tolerance
(and bit-identical between the two dictionaries, which give the same map)."""
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


def _map(sp, coords, extent, ks=3, flip=False, sorted_keys=False):
    m = sp.spconv_build_map(coords_dev(coords), extent, ks, flip_kernel=flip, sorted_keys=sorted_keys)
    got = m.neighbor_map().cpu().numpy()
    return m, got


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
@pytest.mark.parametrize("flip,sorted_keys", [(False, False), (True, False), (False, True), (True, True)])
def test_option_maps_bit_exact_on_workloads(sp, name, flip, sorted_keys):
    wl = workloads.make_workload(name, 0, n_layers=1)
    m, got = _map(sp, wl.coords, wl.grid, flip=flip, sorted_keys=sorted_keys)
    try:
        ref = oracle.neighbor_map(wl.coords, wl.grid, flip=flip)
        assert np.array_equal(got, ref)
        assert m.pairs == int((ref >= 0).sum())
    finally:
        m.free()


def test_sorted_keys_edge_cases(sp):
    cases = [
        (np.array([[0, 3, 3, 3]], np.int32), (8, 8, 8)),
        (np.array([[b, 0, 0, 0] for b in range(5)], np.int32), (1, 1, 1)),
        (np.array([[0, 0, 0, 0], [0, 65534, 2, 69], [0, 65533, 2, 69], [0, 1, 0, 0], [7, 65534, 1, 35],
                   [7, 65534, 2, 35], [65535, 0, 0, 0]], np.int32), (65535, 3, 70)),
        # a full 5^3 block: every interior voxel has all 26 neighbours
        (np.array([[0, a, b, c] for a in range(5) for b in range(5) for c in range(5)], np.int32)[::-1].copy(),
         (5, 5, 5)),
    ]
    for coords, ext in cases:
        for flip in (False, True):
            m, got = _map(sp, coords, ext, flip=flip, sorted_keys=True)
            m.free()
            assert np.array_equal(got, oracle.neighbor_map(coords, ext, flip=flip))
    m = sp.spconv_build_map(torch.empty((0, 4), dtype=torch.int32, device="cuda"), (4, 4, 4), 3, sorted_keys=True)
    assert m.n == 0 and m.pairs == 0
    m.free()
    m = sp.spconv_build_map(coords_dev(cases[0][0]), (8, 8, 8), 1, sorted_keys=True)
    assert m.n == 1 and m.kernel_size == 1
    m.free()


def test_sorted_keys_errors(sp):
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_build_map(coords_dev(np.array([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], np.int32)), (4, 4, 4),
                            3, sorted_keys=True)
    assert e.value.status == sp.DUPLICATE
    with pytest.raises(sp.SpconvError) as e:
        sp.spconv_build_map(coords_dev(np.array([[0, 4, 1, 1]], np.int32)), (4, 4, 4), 3, sorted_keys=True)
    assert e.value.status == sp.COORD_RANGE
    with pytest.raises(sp.SpconvError) as e:  # 16 + 16 * 3 key bits do not fit
        sp.spconv_build_map(coords_dev(np.array([[0, 1, 1, 1]], np.int32)), (65535, 65535, 65535), 3,
                            sorted_keys=True)
    assert e.value.status == sp.UNSUPPORTED
    # unknown flag bits are rejected by the C entry point itself
    import ctypes
    h = ctypes.c_void_p()
    st = sp.lib.spconv_build_map_ex(None, 0, (ctypes.c_int32 * 3)(4, 4, 4), 3, 16, None, ctypes.byref(h))
    assert st == sp.INVALID_ARG
    st = sp.lib.spconv_build_map_ex(None, 0, (ctypes.c_int32 * 3)(4, 4, 4), 3, sp.MAP_SORTED_KEYS | sp.MAP_HASH_TABLE,
                                    None, ctypes.byref(h))
    assert st == sp.INVALID_ARG


@pytest.mark.parametrize("name,cin,cout", [("tiny", 16, 16), ("shells", 64, 64)])
def test_flipped_forward_matches_oracle(sp, name, cin, cout):
    wl = workloads.make_workload(name, 0, n_layers=1)
    dtype = wl.dtype
    rng = np.random.default_rng(21)
    w = rng.standard_normal((27, cin, cout)) / np.sqrt(27 * cin)
    bias = rng.standard_normal(cout) * 0.1
    x = wl.x[:, :cin]
    xd, wd, bd = to_dev(x, dtype), to_dev(w, dtype), to_dev(bias, dtype)
    # the oracle sees the values the GPU sees (rounded to the dtype)
    xr = xd.double().cpu().numpy()
    wr = wd.double().cpu().numpy()
    br = bd.double().cpu().numpy()
    ref_nbr = oracle.neighbor_map(wl.coords, wl.grid, flip=True)
    rows = np.arange(wl.n) if wl.n <= 60000 else np.random.default_rng(0).choice(wl.n, 60000, replace=False)
    ref = oracle_forward_rows(oracle, ref_nbr, xr, wr, br, rows)
    outs = []
    for sorted_keys in (False, True):
        m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3, flip_kernel=True, sorted_keys=sorted_keys)
        out = sp.spconv_subm_forward(m, xd, wd, bd)
        m.check()
        m.free()
        outs.append(out)
        assert_close(out[torch.from_numpy(rows).cuda()], ref, dtype, label=f"flip sorted={sorted_keys}")
    assert torch.equal(outs[0], outs[1])  # same map, same metadata: identical bits


def test_sorted_and_hash_maps_give_identical_forwards(sp):
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    xd = to_dev(wl.x, "bf16")
    wd = to_dev(wl.layers[0].w, "bf16")
    bd = to_dev(wl.layers[0].bias, "bf16")
    outs = []
    for sorted_keys in (False, True):
        m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3, sorted_keys=sorted_keys)
        st = m.stats(copy_arrays=True)
        outs.append((sp.spconv_subm_forward(m, xd, wd, bd), st))
        m.check()
        m.free()
    assert torch.equal(outs[0][0], outs[1][0])
    for key in ("perm", "nbr_t", "order"):
        assert torch.equal(outs[0][1][key], outs[1][1][key])
    # tile records: the header and the J job words (words past them are padding)
    j0, j1 = outs[0][1]["jobs"], outs[1][1]["jobs"]
    used = torch.arange(j0.shape[1], device=j0.device)[None, :] < 4 + j0[:, :1]
    assert torch.equal(j0[:, 0], j1[:, 0]) and torch.equal(j0[used], j1[used])
