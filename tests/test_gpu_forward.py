"""GPU forward vs the CPU oracle (fp64), through the C ABI.

Every comparison takes its reference from the oracle alone: the oracle's own
neighbour map and the oracle's forward, never a map or value from the CUDA path.
Small cases and the full-size workloads are compared on every output row (the
oracle runs on row chunks in parallel host threads); the ten chained layers of
the 128^3 workload are compared on sampled rows per layer, beside one full layer.
"""
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


def _run(sp, coords, extent, x, w, bias, dtype, algo=0, m=None):
    own = m is None
    if own:
        m = sp.spconv_build_map(coords_dev(coords), extent, 1 if w.shape[0] == 1 else 3)
    try:
        out = sp.spconv_subm_forward(m, to_dev(x, dtype), to_dev(w, dtype),
                                     None if bias is None else to_dev(bias, dtype), algo=algo)
        m.check()
        return out
    finally:
        if own:
            m.free()


def _ref(coords, extent, x, w, bias, rows=None):
    return oracle.subm_conv3d(coords, extent, x, w, bias, rows)


def test_tiny_fp32_k3_and_k1(sp):
    wl = workloads.make_workload("tiny", 0)
    for layer in wl.layers:
        out = _run(sp, wl.coords, wl.grid, wl.x, layer.w, layer.bias, "f32")
        assert_close(out, _ref(wl.coords, wl.grid, wl.x, layer.w, layer.bias), "f32")
        out = _run(sp, wl.coords, wl.grid, wl.x, layer.w, None, "f32")
        assert_close(out, _ref(wl.coords, wl.grid, wl.x, layer.w, None), "f32")


def _case(seed, grid, n, cin, cout, kvol=27, bias=True):
    rng = np.random.default_rng(seed)
    coords = workloads.uniform_coords(rng, grid, n)
    x = workloads.round_to_bf16(rng.standard_normal((n, cin), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((kvol, cin, cout), dtype=np.float32) * (kvol * cin) ** -0.5)
    b = workloads.round_to_bf16(rng.standard_normal(cout, dtype=np.float32) * 0.1) if bias else None
    return coords, (grid,) * 3, x, w, b


# Several tiles with a ragged tail; every kernel variant (Cout block 64 or
# 128; input chunk 16, 32 or 64 channels); with and without bias.
@pytest.mark.parametrize("cin,cout,bias", [
    (64, 64, True), (128, 128, True), (128, 128, False), (32, 64, True), (16, 64, True),
    (64, 128, True), (128, 256, True), (48, 192, True), (512, 512, True),
])
def test_bf16_tcgen05_matches_oracle(sp, cin, cout, bias):
    coords, ext, x, w, b = _case(1, 24, 2000, cin, cout, bias=bias)
    out = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(coords, ext, x, w, b), "bf16")


@pytest.mark.parametrize("cin,cout", [(64, 64), (128, 128), (512, 512), (32, 64), (16, 64), (48, 128)])
def test_bf16_kernel_size_one(sp, cin, cout):
    coords, ext, x, w, b = _case(2, 30, 1500, cin, cout, kvol=1)
    out = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(coords, ext, x, w, b), "bf16")
    np.testing.assert_allclose(_ref(coords, ext, x, w, b), x.astype(np.float64) @ w[0] + b, rtol=1e-10, atol=1e-10)


def test_bf16_simt_matches_oracle_and_tcgen05(sp):
    coords, ext, x, w, b = _case(3, 20, 1200, 64, 128)
    ref = _ref(coords, ext, x, w, b)
    simt = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_SIMT)
    tc = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(simt, ref, "bf16")
    assert_close(tc, ref, "bf16")


def test_bf16_auto_uses_simt_for_other_cout(sp):
    coords, ext, x, w, b = _case(4, 16, 500, 32, 48)
    out = _run(sp, coords, ext, x, w, b, "bf16")
    assert_close(out, _ref(coords, ext, x, w, b), "bf16")
    with pytest.raises(sp.SpconvError) as e:
        _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert e.value.status == sp.UNSUPPORTED


def test_dense_block_and_isolated_voxels(sp):
    rng = np.random.default_rng(5)
    # fully occupied 12^3 block: up to 384 hits per offset in a tile (several jobs per offset)
    blk = np.array([[0, a, b, c] for a in range(12) for b in range(12) for c in range(12)], np.int32)
    blk = blk[rng.permutation(blk.shape[0])]
    x = workloads.round_to_bf16(rng.standard_normal((blk.shape[0], 64), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((27, 64, 128), dtype=np.float32) * 0.03)
    b = workloads.round_to_bf16(rng.standard_normal(128, dtype=np.float32) * 0.1)
    out = _run(sp, blk, (12, 12, 12), x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(blk, (12, 12, 12), x, w, b), "bf16")
    # isolated voxels only: centre tap alone
    iso = np.array([[0, 4 * i % 64, 4 * (i // 16) % 64, 4 * (i // 256)] for i in range(1000)], np.int32)
    xi = workloads.round_to_bf16(rng.standard_normal((1000, 64), dtype=np.float32))
    out = _run(sp, iso, (64, 64, 64), xi, w[:, :, :64].copy(), b[:64].copy(), "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, xi.astype(np.float64) @ w[13, :, :64] + b[:64], "bf16")


@pytest.fixture
def tile_rows(sp):
    """Force the tile height of the maps a test builds; restores the automatic choice."""
    def force(rows):
        sp.spconv_debug_set_tile_rows(rows)
    yield force
    sp.spconv_debug_set_tile_rows(0)


# The same cases through full-height (256-row) tiles, the shortest (16-row) tiles
# and an odd number of windows per tile: spans of every length, many tiles per
# CTA (both accumulator buffers, several rounds each) and ragged tails.
@pytest.mark.parametrize("rows", [256, 16, 112])
@pytest.mark.parametrize("cin,cout,kvol", [(128, 128, 27), (64, 128, 27), (16, 64, 27), (512, 512, 27),
                                           (128, 128, 1), (48, 128, 1)])
def test_bf16_tcgen05_forced_tile_heights(sp, tile_rows, rows, cin, cout, kvol):
    tile_rows(rows)
    coords, ext, x, w, b = _case(9, 24, 2000, cin, cout, kvol=kvol)
    out = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(coords, ext, x, w, b), "bf16")


def test_dense_block_full_height_tiles(sp, tile_rows):
    rng = np.random.default_rng(11)
    tile_rows(256)
    blk = np.array([[0, a, b, c] for a in range(12) for b in range(12) for c in range(12)], np.int32)
    blk = blk[rng.permutation(blk.shape[0])]
    x = workloads.round_to_bf16(rng.standard_normal((blk.shape[0], 128), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((27, 128, 128), dtype=np.float32) * 0.02)
    b = workloads.round_to_bf16(rng.standard_normal(128, dtype=np.float32) * 0.1)
    out = _run(sp, blk, (12, 12, 12), x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(blk, (12, 12, 12), x, w, b), "bf16")


def test_single_voxel_and_single_tile_edge(sp):
    for n in (1, 15, 16, 17, 127, 128, 129, 255, 256, 257, 705):  # around windows and tile heights
        coords, ext, x, w, b = _case(6 + n, 12, n, 64, 64)
        out = _run(sp, coords, ext, x, w, b, "bf16", algo=sp.ALGO_TCGEN05)
        assert_close(out, _ref(coords, ext, x, w, b), "bf16")


def test_single_tap_shift_is_exact_in_bf16(sp):
    """W = identity at one offset: the output is an exact shifted copy even in bf16."""
    rng = np.random.default_rng(8)
    coords = workloads.uniform_coords(rng, 10, 600)
    x = workloads.round_to_bf16(rng.standard_normal((600, 64), dtype=np.float32))
    for k in (22, 4, 16, 14, 0, 26):
        w = np.zeros((27, 64, 64), np.float32)
        w[k] = np.eye(64, dtype=np.float32)
        out = _run(sp, coords, (10, 10, 10), x, w, None, "bf16", algo=sp.ALGO_TCGEN05).float().cpu().numpy()
        assert np.array_equal(out, _ref(coords, (10, 10, 10), x, w, None).astype(np.float32))


def _sample_rows(n, count, seed=0):
    rng = np.random.default_rng(seed)
    rows = rng.choice(n, min(count, n), replace=False)
    return np.sort(np.concatenate([rows, [0, n - 1]]))


@pytest.mark.parametrize("name", ["shells", "batched", "large"])
def test_full_size_workloads_every_row(sp, name):
    """Every output row of the full-size workloads (batched: its k=3 layer and
    the chained k=1 layer) against the oracle run on the same input."""
    wl = workloads.make_workload(name, 0)
    m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3)
    nbr = oracle.neighbor_map(wl.coords, wl.grid)
    m1 = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 1) if any(l.kernel_size == 1 for l in wl.layers) else None
    try:
        x_host = wl.x
        x_dev = to_dev(wl.x, "bf16")
        for li, layer in enumerate(wl.layers):
            mm = m if layer.kernel_size == 3 else m1
            out = sp.spconv_subm_forward(mm, x_dev, to_dev(layer.w, "bf16"), to_dev(layer.bias, "bf16"))
            mm.check()
            nb = nbr if layer.kernel_size == 3 else np.arange(wl.n, dtype=np.int32).reshape(-1, 1)
            ref = oracle_forward_rows(oracle, nb, x_host, layer.w, layer.bias)
            assert_close(out, ref, "bf16", label=f"{name} layer {li} k={layer.kernel_size}")
            if wl.chained:  # next layer consumes this layer's GPU output
                x_dev = out
                x_host = out.float().cpu().numpy()
    finally:
        m.free()
        if m1 is not None:
            m1.free()


def test_uniform_ten_layers_chained_sampled(sp):
    """The pages' benchmark shape: ten 128->128 layers on one map, ping-pong buffers;
    each layer is checked on sampled rows against the oracle run on its GPU input."""
    wl = workloads.make_workload("uniform", 0)
    m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3)
    nbr = oracle.neighbor_map(wl.coords, wl.grid)
    try:
        bufs = [to_dev(wl.x, "bf16"), torch.empty((wl.n, 128), dtype=torch.bfloat16, device="cuda")]
        for i, layer in enumerate(wl.layers):
            src, dst = bufs[i % 2], bufs[(i + 1) % 2]
            x_host = src.float().cpu().numpy()
            sp.spconv_subm_forward(m, src, to_dev(layer.w, "bf16"), to_dev(layer.bias, "bf16"), out=dst)
            m.check()
            rows = _sample_rows(wl.n, 800, seed=i)
            ref = oracle.forward(nbr, x_host, layer.w, layer.bias, rows=rows)
            assert_close(dst[torch.from_numpy(rows).cuda()], ref, "bf16")
    finally:
        m.free()


def test_uniform_full_output_every_row(sp):
    """Every row of one full-size layer of the pages' shape, both kernels, against
    the fp64 oracle over the whole output."""
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    layer = wl.layers[0]
    m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3)
    try:
        x, w, b = to_dev(wl.x, "bf16"), to_dev(layer.w, "bf16"), to_dev(layer.bias, "bf16")
        tc = sp.spconv_subm_forward(m, x, w, b, algo=sp.ALGO_TCGEN05)
        simt = sp.spconv_subm_forward(m, x, w, b, algo=sp.ALGO_SIMT)
        m.check()
        ref = oracle_forward_rows(oracle, oracle.neighbor_map(wl.coords, wl.grid), wl.x, layer.w, layer.bias)
        assert_close(tc, ref, "bf16", label="uniform tcgen05")
        assert_close(simt, ref, "bf16", label="uniform simt")
    finally:
        m.free()


def test_repeat_calls_identical(sp):
    """Many launches on one map reuse its tile-scheduler counters in turn (each
    launch leaves its counter at zero): every output must be the same."""
    coords, ext, x, w, b = _case(9, 20, 2500, 128, 128)
    m = sp.spconv_build_map(coords_dev(coords), ext, 3)
    try:
        xd, wd, bd = to_dev(x, "bf16"), to_dev(w, "bf16"), to_dev(b, "bf16")
        o1 = sp.spconv_subm_forward(m, xd, wd, bd)
        outs = [sp.spconv_subm_forward(m, xd, wd, bd) for _ in range(130)]  # > 2 x the 64 counter slots
        m.check()
        assert all(torch.equal(o1, o) for o in outs)
        assert_close(o1, _ref(coords, ext, x, w, b), "bf16", label="repeat")
    finally:
        m.free()


@pytest.mark.parametrize("name", ["tiny", "uniform", "shells", "batched", "large"])
def test_auto_kernel_choice_on_workloads(sp, name):
    """AUTO runs every bf16 layer of the five workloads on the tensor cores (kernel
    size 1 with 64-channel multiples on the GEMM kernel, the rest on the window
    kernel) and the fp32 tiny layers on the CUDA-core kernel; the map's launch
    counters show it."""
    wl = workloads.make_workload(name, 0, n_layers=1)
    x = to_dev(wl.x, wl.dtype)
    for layer in wl.layers:
        cin = layer.w.shape[1]
        expected = ("simt" if wl.dtype == "f32" else
                    "tcgen05_gemm" if layer.kernel_size == 1 and cin % 64 == 0 and wl.n >= 128 else "tcgen05")
        m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, layer.kernel_size)
        try:
            sp.spconv_subm_forward(m, x, to_dev(layer.w, wl.dtype), to_dev(layer.bias, wl.dtype))
            m.check()
            counts = m.launch_counts()
        finally:
            m.free()
        assert counts[expected] == 1 and sum(counts.values()) == 1, (name, layer.kernel_size, counts)


@pytest.fixture
def ring_depths(sp):
    """Force the forward's ring depths; restores the automatic choice."""
    def force(a, b):
        sp.spconv_debug_set_ring_depths(a, b)
    yield force
    sp.spconv_debug_set_ring_depths(0, 0)


# Shallow rings: the weight ring and the B-ring units wrap around on nearly every
# job (jobs that do not fit before the end start over at unit 0), including the
# several input-channel chunks of 512-channel layers.
@pytest.mark.parametrize("a,b", [(2, 4), (2, 5), (3, 5)])
@pytest.mark.parametrize("cin,cout,kvol", [(128, 128, 27), (512, 512, 27), (64, 64, 27), (32, 64, 27),
                                           (512, 512, 1)])
def test_bf16_tcgen05_shallow_rings(sp, ring_depths, a, b, cin, cout, kvol):
    ring_depths(a, b)
    coords, ext, x, w, bias = _case(13, 22, 2500, cin, cout, kvol=kvol)
    out = _run(sp, coords, ext, x, w, bias, "bf16", algo=sp.ALGO_TCGEN05)
    assert_close(out, _ref(coords, ext, x, w, bias), "bf16", label=f"rings {a},{b}")
