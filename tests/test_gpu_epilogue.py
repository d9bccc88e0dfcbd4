"""GPU fused decoder epilogue vs the CPU oracle: out = act(conv + bias) (+ residual),
per-channel sums of out and out^2, on both kernel families."""
import ctypes

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


def _case(seed, grid, n, cin, cout, dtype):
    rng = np.random.default_rng(seed)
    coords = workloads.uniform_coords(rng, grid, n)
    x = rng.standard_normal((n, cin), dtype=np.float32)
    w = rng.standard_normal((27, cin, cout), dtype=np.float32) * np.float32((27 * cin) ** -0.5)
    b = rng.standard_normal(cout, dtype=np.float32) * np.float32(0.1)
    r = rng.standard_normal((n, cout), dtype=np.float32)
    return coords, (grid,) * 3, to_dev(x, dtype), to_dev(w, dtype), to_dev(b, dtype), to_dev(r, dtype)


def _check_stats(stats, out):
    """GPU sums (fp32 atomics) against the fp64 sums of the GPU's own stored output."""
    o = out.double().cpu().numpy()
    ref = oracle.channel_stats(o)
    got = stats.double().cpu().numpy()
    scale = np.stack([np.abs(o).sum(axis=0), (o * o).sum(axis=0)]) + 1e-30
    err = np.abs(got - ref) / scale
    assert err.max() < 2e-5, f"stats error / scale = {err.max():.3e}"


@pytest.mark.parametrize("cin,cout,algo", [(128, 128, "tc"), (64, 64, "tc"), (512, 512, "tc"), (64, 64, "simt")])
@pytest.mark.parametrize("act", ["none", "relu", "silu", "gelu"])
@pytest.mark.parametrize("with_residual", [False, True])
def test_fused_epilogue_matches_oracle(sp, cin, cout, algo, act, with_residual):
    coords, ext, x, w, b, r = _case(41, 24, 2000 if cin < 512 else 900, cin, cout, "bf16")
    m = sp.spconv_build_map(coords_dev(coords), ext, 3)
    stats = torch.empty((2, cout), dtype=torch.float32, device="cuda")
    try:
        out = sp.spconv_subm_forward(m, x, w, b, act=act, residual=r if with_residual else None, stats=stats,
                                     algo=sp.ALGO_TCGEN05 if algo == "tc" else sp.ALGO_SIMT)
        m.check()
        conv = oracle_forward_rows(oracle, oracle.neighbor_map(coords, ext), x.double().cpu().numpy(),
                                   w.double().cpu().numpy(), b.double().cpu().numpy())
        ref = oracle.epilogue(conv, act, r.double().cpu().numpy() if with_residual else None)
        assert_close(out, ref, "bf16", label=f"{algo} {act} res={with_residual}")
        _check_stats(stats, out)
        assert m.launch_counts()["tcgen05" if algo == "tc" else "simt"] == 1
    finally:
        m.free()


def test_residual_in_place_and_fp32(sp):
    coords, ext, x, w, b, r = _case(42, 20, 1500, 64, 128, "bf16")
    m = sp.spconv_build_map(coords_dev(coords), ext, 3)
    try:
        conv = oracle_forward_rows(oracle, oracle.neighbor_map(coords, ext), x.double().cpu().numpy(),
                                   w.double().cpu().numpy(), b.double().cpu().numpy())
        ref = oracle.epilogue(conv, "silu", r.double().cpu().numpy())
        out = r.clone()  # the residual is the output buffer: out += silu(conv + bias)
        sp.spconv_subm_forward(m, x, w, b, out=out, act="silu", residual=out)
        m.check()
        assert_close(out, ref, "bf16", label="in place")
    finally:
        m.free()
    # fp32 on the CUDA-core kernel
    coords, ext, x, w, b, r = _case(43, 16, 400, 16, 16, "f32")
    m = sp.spconv_build_map(coords_dev(coords), ext, 3)
    stats = torch.empty((2, 16), dtype=torch.float32, device="cuda")
    try:
        out = sp.spconv_subm_forward(m, x, w, b, act="gelu", residual=r, stats=stats)
        m.check()
        conv = oracle.forward(oracle.neighbor_map(coords, ext), x.double().cpu().numpy(),
                              w.double().cpu().numpy(), b.double().cpu().numpy())
        assert_close(out, oracle.epilogue(conv, "gelu", r.double().cpu().numpy()), "f32", label="fp32 gelu")
        _check_stats(stats, out)
    finally:
        m.free()


def test_fused_epilogue_full_size_uniform_sampled(sp):
    """One 128 -> 128 layer of the 128^3 workload with SiLU, a residual and statistics."""
    wl = workloads.make_workload("uniform", 0, n_layers=1)
    layer = wl.layers[0]
    m = sp.spconv_build_map(coords_dev(wl.coords), wl.grid, 3)
    rng = np.random.default_rng(44)
    res = to_dev(rng.standard_normal((wl.n, 128), dtype=np.float32), "bf16")
    stats = torch.empty((2, 128), dtype=torch.float32, device="cuda")
    try:
        out = sp.spconv_subm_forward(m, to_dev(wl.x, "bf16"), to_dev(layer.w, "bf16"), to_dev(layer.bias, "bf16"),
                                     act="silu", residual=res, stats=stats)
        m.check()
        rows = rng.choice(wl.n, 4000, replace=False)
        conv = oracle.forward(oracle.neighbor_map(wl.coords, wl.grid), wl.x, layer.w, layer.bias, rows=rows)
        ref = oracle.epilogue(conv, "silu", res[torch.from_numpy(rows).cuda()].double().cpu().numpy())
        assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", label="uniform silu+res")
        _check_stats(stats, out)
    finally:
        m.free()


def test_epilogue_argument_errors(sp):
    coords, ext, x, w, b, r = _case(45, 12, 300, 64, 64, "bf16")
    m = sp.spconv_build_map(coords_dev(coords), ext, 3)
    out = torch.empty((300, 64), dtype=torch.bfloat16, device="cuda")
    try:
        epi = sp._Epilogue(7, None, None)
        st = sp.lib.spconv_subm_forward_ex(m.handle, 1, x.data_ptr(), 64, w.data_ptr(), b.data_ptr(), out.data_ptr(),
                                           64, ctypes.byref(epi), 0, None)
        assert st == sp.INVALID_ARG
        epi = sp._Epilogue(0, x.data_ptr(), None)  # residual overlapping x
        st = sp.lib.spconv_subm_forward_ex(m.handle, 1, x.data_ptr(), 64, w.data_ptr(), b.data_ptr(), out.data_ptr(),
                                           64, ctypes.byref(epi), 0, None)
        assert st == sp.INVALID_ARG
        epi = sp._Epilogue(0, out.data_ptr() + 32, None)  # partly overlapping out
        st = sp.lib.spconv_subm_forward_ex(m.handle, 1, x.data_ptr(), 64, w.data_ptr(), b.data_ptr(), out.data_ptr(),
                                           64, ctypes.byref(epi), 0, None)
        assert st == sp.INVALID_ARG
        with pytest.raises(ValueError):
            sp.spconv_subm_forward(m, x, w, b, act="tanh")
        with pytest.raises(ValueError):
            sp.spconv_subm_forward(m, x, w, b, stats=torch.empty((2, 64), device="cuda", dtype=torch.float64))
    finally:
        m.free()
