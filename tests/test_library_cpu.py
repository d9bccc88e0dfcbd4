"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every
symbol include/spconv.h declares, and rejects bad arguments before any device work."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spconv.h")


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SPCONV_API\s+[\w\s\*]+?\b(spconv_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def pkg():
    from submanifold_sparse_convolution_submconv3d_b200 import build as b
    b.build()
    import submanifold_sparse_convolution_submconv3d_b200 as p
    return p


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for name in ("spconv_build_map", "spconv_subm_forward", "spconv_free"):
        assert name in syms
    assert len(syms) >= 8


def _header_enum(prefix):
    """{name: value} of the header's enumerators starting with prefix."""
    text = open(HEADER).read()
    return {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(" + prefix + r"\w+)\s*=\s*(\d+)", text)}


def test_binding_constants_match_the_header(pkg):
    """The binding's copies of the header's enumerators (map flags, algorithms,
    activations, kernel families) carry the header's values."""
    maps = _header_enum("SPCONV_MAP_")
    assert (pkg.MAP_DEFAULT, pkg.MAP_FLIP_KERNEL, pkg.MAP_SORTED_KEYS, pkg.MAP_HASH_TABLE, pkg.MAP_SHORT_TILES) == (
        maps["SPCONV_MAP_DEFAULT"], maps["SPCONV_MAP_FLIP_KERNEL"], maps["SPCONV_MAP_SORTED_KEYS"],
        maps["SPCONV_MAP_HASH_TABLE"], maps["SPCONV_MAP_SHORT_TILES"])
    algos = _header_enum("SPCONV_ALGO_")
    assert (pkg.ALGO_AUTO, pkg.ALGO_SIMT, pkg.ALGO_TCGEN05) == (
        algos["SPCONV_ALGO_AUTO"], algos["SPCONV_ALGO_SIMT"], algos["SPCONV_ALGO_TCGEN05"])
    acts = _header_enum("SPCONV_ACT_")
    for name in ("none", "relu", "silu", "gelu"):
        assert pkg.ACTIVATIONS[name] == acts["SPCONV_ACT_" + name.upper()]
    kinds = _header_enum("SPCONV_KERNEL_")
    assert len(pkg.KERNEL_NAMES) == kinds["SPCONV_KERNEL_KINDS"]
    assert (pkg.KERNEL_SIMT, pkg.KERNEL_TCGEN05, pkg.KERNEL_TCGEN05_GEMM) == (
        kinds["SPCONV_KERNEL_SIMT"], kinds["SPCONV_KERNEL_TCGEN05"], kinds["SPCONV_KERNEL_TCGEN05_GEMM"])
    assert pkg.KERNEL_NAMES[pkg.KERNEL_TCGEN05_GEMM] == "tcgen05_gemm"


def test_library_exports_every_declared_symbol(pkg):
    lib = ctypes.CDLL(pkg.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) == set(pkg.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (spconv_\w+)", out))
    assert exported == set(_declared_symbols())


def test_host_validation_without_device_work(pkg):
    lib = pkg.lib
    handle = ctypes.c_void_p()
    ext = (ctypes.c_int32 * 3)(4, 4, 4)
    assert lib.spconv_build_map(None, 0, ext, 5, None, ctypes.byref(handle)) == pkg.INVALID_ARG
    assert b"kernel_size" in lib.spconv_last_error()
    bad_ext = (ctypes.c_int32 * 3)(0, 4, 4)
    assert lib.spconv_build_map(None, 0, bad_ext, 3, None, ctypes.byref(handle)) == pkg.INVALID_ARG
    big_ext = (ctypes.c_int32 * 3)(70000, 4, 4)
    assert lib.spconv_build_map(None, 0, big_ext, 3, None, ctypes.byref(handle)) == pkg.INVALID_ARG
    assert lib.spconv_build_map(None, -1, ext, 3, None, ctypes.byref(handle)) == pkg.INVALID_ARG
    assert lib.spconv_build_map(None, 5, ext, 3, None, ctypes.byref(handle)) == pkg.INVALID_ARG  # null coords
    assert lib.spconv_build_map(None, 1 << 31, ext, 3, None, ctypes.byref(handle)) == pkg.INVALID_ARG
    assert lib.spconv_build_map(None, 0, ext, 3, None, None) == pkg.INVALID_ARG
    assert handle.value is None
    assert lib.spconv_map_info(None, None, None, None, None) == pkg.INVALID_ARG
    assert lib.spconv_free(None) == pkg.OK
    assert lib.spconv_subm_forward(None, 1, None, 16, None, None, None, 16, None) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_table_slots(3) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_table_slots(0) == pkg.OK
    rows = ctypes.c_int32()
    assert lib.spconv_map_tile_rows(None, ctypes.byref(rows)) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_tile_rows(-1) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_tile_rows(272) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_tile_rows(100) == pkg.INVALID_ARG  # not a multiple of 16
    assert lib.spconv_debug_set_tile_rows(256) == pkg.OK
    assert lib.spconv_debug_set_tile_rows(16) == pkg.OK
    assert lib.spconv_debug_set_tile_rows(0) == pkg.OK
    assert lib.spconv_debug_set_ring_depths(1, 8) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_ring_depths(3, 3) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_ring_depths(3, 33) == pkg.INVALID_ARG
    assert lib.spconv_debug_set_ring_depths(2, 4) == pkg.OK
    assert lib.spconv_debug_set_ring_depths(0, 0) == pkg.OK
    assert lib.spconv_map_stats(None, None) == pkg.INVALID_ARG
    counts = (ctypes.c_int64 * 2)()
    assert lib.spconv_map_launch_counts(None, counts, 2) == pkg.INVALID_ARG


def test_python_binding_rejects_bad_tensors(pkg):
    import torch
    with pytest.raises(ValueError):
        pkg.spconv_build_map(torch.zeros((3, 4), dtype=torch.int64), (4, 4, 4))
    with pytest.raises(ValueError):
        pkg.spconv_build_map(torch.zeros((3, 3), dtype=torch.int32), (4, 4, 4))


def test_binding_refuses_bad_tensors_before_the_library(pkg):
    """The binding checks shapes and devices before it passes raw pointers down:
    a host tensor or a short bias must never reach a kernel.  The map here has no
    library handle, so any call that got through would fail differently."""
    import torch

    m = object.__new__(pkg.SubmMap)
    m.handle, m.device, m.n, m.kernel_size, m.pairs, m.tile_rows = None, torch.device("cuda", 0), 4, 3, 4, 4
    x = torch.zeros((4, 16), dtype=torch.bfloat16)
    w = torch.zeros((27, 16, 64), dtype=torch.bfloat16)
    b = torch.zeros(64, dtype=torch.bfloat16)
    cases = [
        (dict(x=x, w=w, bias=b), "CUDA tensors"),                                   # host tensors
        (dict(x=x, w=w, bias=torch.zeros(32, dtype=torch.bfloat16)), "bias must be"),  # short bias
        (dict(x=x, w=w, bias=b.view(1, 64)), "bias must be"),
        (dict(x=x, w=w[0]), "w [K^3, Cin, Cout]"),                                  # 2-D weights
        (dict(x=x, w=torch.zeros((1, 16, 64), dtype=torch.bfloat16)), "shape mismatch"),
        (dict(x=x[:3], w=w), "shape mismatch"),
        (dict(x=x, w=w.float()), "match x"),
        (dict(x=x, w=w, out=torch.zeros((4, 32), dtype=torch.bfloat16)), "out must be"),
        (dict(x=x.to(torch.float16), w=w.to(torch.float16)), "float32 or bfloat16"),
    ]
    for kw, msg in cases:
        with pytest.raises(ValueError, match=re.escape(msg)):
            pkg.spconv_subm_forward(m, **kw)
