"""Kernel size 1 on the weight-stationary tcgen05 GEMM vs the CPU oracle (fp64).

A map of kernel size 1 makes the layer out = x . W[0] + bias row by row; AUTO
runs it on the GEMM kernel when cin % 64 == 0, the weight slice fits shared
memory and n >= 128.  Cases cover both output-channel block widths (64, 128),
one to many tiles per CTA (all four accumulators and the x-stage ring wrapping
many times), a ragged last tile, the widest slices that fit, x stages shared
across clusters of 2, 4 and 8 CTAs, forced shallow stage rings, the fused
epilogue, and the shapes that go to the window kernel instead.  Every reference
comes from the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import assert_close, coords_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sp():
    import submanifold_sparse_convolution_submconv3d_b200 as p
    return p


def _case(seed, n, cin, cout):
    rng = np.random.default_rng(seed)
    grid = max(8, int(np.ceil((4 * n) ** (1 / 3))))
    coords = workloads.uniform_coords(rng, grid, n)
    x = workloads.round_to_bf16(rng.standard_normal((n, cin), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((1, cin, cout), dtype=np.float32) * cin ** -0.5)
    b = workloads.round_to_bf16(rng.standard_normal(cout, dtype=np.float32) * 0.1)
    return coords, (grid,) * 3, x, w, b


def _forward(sp, coords, ext, x, w, b, **kw):
    m = sp.spconv_build_map(coords_dev(coords), ext, 1)
    try:
        out = sp.spconv_subm_forward(m, to_dev(x, "bf16"), to_dev(w, "bf16"), to_dev(b, "bf16"), **kw)
        m.check()
        return out, m.launch_counts()
    finally:
        m.free()


# (cin, cout, n): one tile (n = 128), a ragged second tile, several channel
# blocks, the widest weight slices that fit (704 x 128 and 1472 x 64), sets large
# enough that every CTA takes more tiles than it has accumulators, and every
# cluster size: x stages shared by 2 (cout 256), 4 (cout 512) and 8 (cout 1024)
# CTAs, none for 1 or 3 channel blocks.
@pytest.mark.parametrize("cin,cout,n", [
    (64, 64, 128), (64, 128, 129), (128, 128, 4133), (192, 64, 1000), (256, 192, 777),
    (512, 512, 3000), (704, 128, 640), (1472, 64, 300), (64, 64, 100003), (512, 512, 28493),
    (128, 256, 5000), (256, 1024, 2000), (128, 1024, 128), (64, 384, 1500), (64, 512, 300),
    (704, 256, 40000),
])
def test_gemm1_matches_oracle(sp, cin, cout, n):
    coords, ext, x, w, b = _case(cin * 7 + cout + n, n, cin, cout)
    out, counts = _forward(sp, coords, ext, x, w, b)
    assert counts["tcgen05_gemm"] == 1 and sum(counts.values()) == 1, counts
    assert_close(out, oracle.subm_conv3d(coords, ext, x, w, b), "bf16", label=f"{cin}x{cout} n={n}")


@pytest.mark.parametrize("stages", [2, 3, 5])
def test_gemm1_forced_stages(sp, stages):
    """Few x stages: the ring wraps on every chunk of every tile."""
    sp.spconv_debug_set_ring_depths(stages, 8)
    try:
        coords, ext, x, w, b = _case(stages, 20000, 512, 512)
        out, counts = _forward(sp, coords, ext, x, w, b)
    finally:
        sp.spconv_debug_set_ring_depths(0, 0)
    assert counts["tcgen05_gemm"] == 1, counts
    assert_close(out, oracle.subm_conv3d(coords, ext, x, w, b), "bf16", label=f"stages {stages}")


@pytest.mark.parametrize("cin,cout,n", [(48, 128, 1500), (64, 64, 100), (1536, 64, 400), (768, 128, 400)])
def test_shapes_the_gemm_does_not_take_run_on_the_window_kernel(sp, cin, cout, n):
    """cin not a multiple of 64, fewer than 128 rows, or a weight slice too wide:
    AUTO runs the window kernel, still against the oracle."""
    coords, ext, x, w, b = _case(cin + n, n, cin, cout)
    out, counts = _forward(sp, coords, ext, x, w, b)
    assert counts["tcgen05"] == 1 and sum(counts.values()) == 1, counts
    assert_close(out, oracle.subm_conv3d(coords, ext, x, w, b), "bf16", label=f"{cin}x{cout} n={n}")


@pytest.mark.parametrize("act", ["none", "relu", "silu", "gelu"])
@pytest.mark.parametrize("cin,cout", [(128, 128), (64, 64), (256, 512)])
def test_gemm1_fused_epilogue(sp, act, cin, cout):
    n = 5000
    coords, ext, x, w, b = _case(11 + cin, n, cin, cout)
    r = workloads.round_to_bf16(np.random.default_rng(5).standard_normal((n, cout), dtype=np.float32))
    stats = torch.empty((2, cout), dtype=torch.float32, device="cuda")
    out, counts = _forward(sp, coords, ext, x, w, b, act=act, residual=to_dev(r, "bf16"), stats=stats)
    assert counts["tcgen05_gemm"] == 1, counts
    ref = oracle.epilogue(oracle.subm_conv3d(coords, ext, x, w, b), act, r.astype(np.float64))
    assert_close(out, ref, "bf16", label=f"{act}")
    o = out.double().cpu().numpy()
    want = oracle.channel_stats(o)
    scale = np.stack([np.abs(o).sum(axis=0), (o * o).sum(axis=0)]) + 1e-30
    assert (np.abs(stats.double().cpu().numpy() - want) / scale).max() < 2e-5


def test_gemm1_in_place_residual(sp):
    """residual == out: each element is read before its own store overwrites it."""
    n, cin, cout = 3000, 128, 128
    coords, ext, x, w, b = _case(21, n, cin, cout)
    r = workloads.round_to_bf16(np.random.default_rng(6).standard_normal((n, cout), dtype=np.float32))
    buf = to_dev(r, "bf16")
    m = sp.spconv_build_map(coords_dev(coords), ext, 1)
    try:
        out = sp.spconv_subm_forward(m, to_dev(x, "bf16"), to_dev(w, "bf16"), to_dev(b, "bf16"), out=buf,
                                     residual=buf, act="relu")
        m.check()
        assert m.launch_counts()["tcgen05_gemm"] == 1
    finally:
        m.free()
    ref = oracle.epilogue(oracle.subm_conv3d(coords, ext, x, w, b), "relu", r.astype(np.float64))
    assert_close(out, ref, "bf16")
