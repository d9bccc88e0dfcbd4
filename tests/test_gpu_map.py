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


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
def test_tile_height_balances_the_sms(sp, name):
    """The map's tile height: 192 rows, or 128 with short tiles; a set too small to
    give every SM a 192-row tile takes the multiple of 16 in [128, 192] whose busiest
    SM gets the fewest rows when the tiles are dealt out round-robin (ties: taller)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    wl = workloads.make_workload(name, 0, n_layers=1)
    heights = {}
    for short in (False, True):
        m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3, short_tiles=short)
        try:
            heights[short] = m.tile_rows
        finally:
            m.free()
    n = wl.n

    def busiest(r):
        return -(-(-(-n // r)) // sms) * r

    assert heights[True] == 128
    if n >= sms * 192:
        assert heights[False] == 192
    else:
        best = min(range(192, 127, -16), key=lambda r: (busiest(r), -r))
        assert heights[False] == best


# ---------------------------------------------------------------------------
# The tensor-core forward's metadata, against a host derivation from the oracle's
# map: the row order is fully determined (a stable sort by the Gray-code rank of
# the 26-bit neighbour mask), so it and the permuted table compare bit for bit;
# the spans are a cost-model choice, so they are checked for what any valid cover
# must satisfy.

def _gray_rank(v: np.ndarray) -> np.ndarray:
    r = v.copy()
    s = v >> 1
    while s.any():
        r ^= s
        s >>= 1
    return r


def _expected_order(nbr: np.ndarray) -> np.ndarray:
    nc = np.delete(nbr >= 0, 13, axis=1)
    key = nc.astype(np.int64) @ (1 << np.arange(25, -1, -1)).astype(np.int64)
    return np.argsort(_gray_rank(key), kind="stable")


def _check_window_meta(sp, coords, extent):
    m = sp.spconv_build_map(coords_dev(coords), extent, 3)
    try:
        st = m.stats(copy_arrays=True)
    finally:
        m.free()
    ref = oracle.neighbor_map(coords, extent)
    n = ref.shape[0]
    rows, tiles = st["rows_per_tile"], st["tiles"]
    assert rows % 16 == 0 and 16 <= rows <= 256 and tiles == -(-n // rows)
    perm = st["perm"].cpu().numpy()
    assert np.array_equal(perm, _expected_order(ref))
    npad = rows * tiles
    exp_t = np.full((27, npad), -1, np.int32)
    exp_t[:, :n] = ref[perm].T
    assert np.array_equal(st["nbr_t"].cpu().numpy(), exp_t)
    jobs = st["jobs"].cpu().numpy()
    nwin = rows // 16
    occ = (exp_t.reshape(27, tiles, nwin, 16) >= 0).any(axis=3)  # [27, tiles, windows]
    spans = cols = 0
    stream_start = 0
    for t in range(tiles):
        nj = int(jobs[t, 0])
        js = jobs[t, 4:4 + nj]
        # header: the tile's index stream length and start (tiles' streams are consecutive)
        assert int(jobs[t, 2]) | (int(jobs[t, 3]) << 32) == stream_start
        assert int(jobs[t, 1]) == int(((js >> 16) & 31).sum()) * 16
        stream_start += int(jobs[t, 1])
        k, w0, nw = js & 31, (js >> 8) & 31, (js >> 16) & 31
        assert (k[0], w0[0], nw[0]) == (13, 0, nwin)  # the centre job covers the tile
        k, w0, nw = k[1:], w0[1:], nw[1:]
        assert np.all(k != 13) and np.all(k < 27) and np.all(nw >= 1) and np.all(w0 + nw <= nwin)
        # each offset's spans are listed together, in increasing window order, without overlap
        runs = k[np.r_[True, k[1:] != k[:-1]]] if k.size else k
        assert len(runs) == len(set(runs.tolist()))
        cover = np.zeros((27, nwin), np.int32)
        for kk, a, b in zip(k, w0, nw):
            cover[kk, a:a + b] += 1
        assert cover.max(initial=0) <= 1
        need = occ[:, t, :].copy()
        need[13] = False
        assert np.all(cover[need] == 1), f"tile {t}: a window with a neighbour is not covered"
        spans += len(k)
        cols += int(nw.sum()) * 16
    assert spans == st["spans"] and cols == st["span_cols"]
    # claim order: a stable sort of the tiles by descending cost (4 * J + stream length // 16) // 4
    cost = np.minimum((4 * jobs[:, 0] + jobs[:, 1] // 16) // 4, 511)
    order = st["order"].cpu().numpy()
    assert np.array_equal(order, np.argsort(-cost, kind="stable"))


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
def test_window_metadata_on_workloads(sp, name):
    wl = workloads.make_workload(name, 0, n_layers=1)
    _check_window_meta(sp, wl.coords, wl.grid)


@pytest.mark.parametrize("rows", [16, 256, 112])
def test_window_metadata_forced_tile_heights(sp, rows):
    sp.spconv_debug_set_tile_rows(rows)
    try:
        rng = np.random.default_rng(rows)
        _check_window_meta(sp, workloads.uniform_coords(rng, 24, 3000), (24, 24, 24))
        blk = np.array([[0, a, b, c] for a in range(10) for b in range(10) for c in range(10)], np.int32)
        _check_window_meta(sp, blk[rng.permutation(1000)], (10, 10, 10))
    finally:
        sp.spconv_debug_set_tile_rows(0)
