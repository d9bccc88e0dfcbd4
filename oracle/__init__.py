"""CPU oracle for SubMConv3d -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its binding)
never imports or calls it, and it imports nothing from the product path.

Two independent implementations of the same definition:

* ``neighbor_map`` / ``forward``: plain C (``subm_oracle.c``), fp64, a sorted-key
  dictionary searched with ``bsearch`` and a per-voxel loop over offsets.
* ``neighbor_map_py`` / ``forward_py``: pure Python with a ``dict`` and loops,
  for tiny inputs only.

The definition (lato.2_mrp_mlx README, "Status" and "Correctness" sections;
pixal3d_mrp_mlx README, "Status", for the [K^3, in, out] weight layout):

    out[i] = bias + sum_{d in {-1,0,1}^3, p_i + d active} W[k(d)]^T x[index(p_i + d)]

with the offset order k(d) = (dx+1)*9 + (dy+1)*3 + (dz+1) (a reading: the
pages do not fix it), cross-correlation orientation (gather p + d), batch
isolation, and grid-boundary neighbours treated as holes.  With ``flip=True``
the map gathers p - d instead: the alternative orientation the lato.2_mrp_mlx
README ("Correctness") leaves open and builds behind its --flip-kernel switch.

The resampling ops around the convolution (``downsample``, ``downsample_amax``,
``upsample``, ``subdivide``) follow the lato.2_mrp_mlx README ("Status":
SparseDownsample is max pooling with the "amax" reduction; the table of upstream
equivalents: SparseSubdivide expands the coordinates x8) and the pixal3d_mrp_mlx
README ("Scope, measured against the shared core": SparseUpsample(2) is the
inverse of a downsample that reuses its pairing).  Readings where the pages are
silent: a voxel p falls in the coarse voxel floor(p / factor) of the same batch;
the coarse voxels are listed in increasing lexicographic (b, x, y, z) order; the
coarse grid is ceil(extent / factor); "amax" of a block is the largest value,
with +0 above -0 (the IEEE 754 total order); subdivision lists the children of
voxel i as rows 8 i + c, c = 4 ox + 2 oy + oz, each carrying voxel i's features.

The fused decoder epilogue (``epilogue``, ``channel_stats``): the pixal3d_mrp_mlx
README ("Correction to the earlier scope") lists SparseConvNeXtBlock3d and
SparseResBlockC2S3d among the decoder blocks around the convolution, and the
lato.2_mrp_mlx README ("Status") lists the activations, norms and SparseResBlock
of the shared core.  Reading: the convolution's store may apply, in this order,
an activation to conv + bias (ReLU, SiLU, or GELU with the exact erf), then add a
residual of the output's shape, and may report per output channel the sum and
the sum of squares of the stored (rounded) output over all rows, which a
following LayerNorm / GroupNorm needs.

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
dense brute force, torch's CPU conv3d, closed forms and invariants; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "subm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, INVALID_ARG, COORD_RANGE, DUPLICATE, OOM = 0, 1, 3, 4, 6


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle error code {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile subm_oracle.c into liboracle.so with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_neighbor_map.restype = ctypes.c_int
        lib.oracle_neighbor_map.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                            ctypes.c_int32, ctypes.c_void_p]
        lib.oracle_neighbor_map_oriented.restype = ctypes.c_int
        lib.oracle_neighbor_map_oriented.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
        lib.oracle_forward_f64.restype = ctypes.c_int
        lib.oracle_forward_f64.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_int64, ctypes.c_void_p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None) -> int | None:
    return None if a is None else a.ctypes.data


def neighbor_map(coords: np.ndarray, extent, kernel_size: int = 3, flip: bool = False) -> np.ndarray:
    """int32 [N, K^3]: row index of the active voxel at p_i + d_k (p_i - d_k with
    ``flip``), or -1."""
    coords = np.ascontiguousarray(coords, dtype=np.int32).reshape(-1, 4)
    ext = np.ascontiguousarray(extent, dtype=np.int32).reshape(3)
    kvol = kernel_size ** 3
    nbr = np.empty((coords.shape[0], kvol), dtype=np.int32)
    rc = _load().oracle_neighbor_map_oriented(_ptr(coords), coords.shape[0], _ptr(ext), kernel_size,
                                              1 if flip else 0, _ptr(nbr))
    if rc != OK:
        raise OracleError(rc)
    return nbr


def forward(nbr: np.ndarray, x: np.ndarray, w: np.ndarray, bias: np.ndarray | None = None,
            rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 output rows ``rows`` (all rows when None) of the convolution over ``nbr``."""
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    kvol, cin, cout = w.shape
    n = x.shape[0]
    assert nbr.shape == (n, kvol) and x.shape[1] == cin
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64).reshape(cout)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    nrows = n if r is None else r.shape[0]
    out = np.empty((nrows, cout), dtype=np.float64)
    rc = _load().oracle_forward_f64(_ptr(nbr), n, kvol, _ptr(x), cin, _ptr(w), _ptr(b), cout,
                                    _ptr(r), nrows, _ptr(out))
    if rc != OK:
        raise OracleError(rc)
    return out


def subm_conv3d(coords, extent, x, w, bias=None, rows=None):
    """Convenience: neighbour map then forward (kernel size from w.shape[0])."""
    ks = {1: 1, 27: 3}[int(np.shape(w)[0])]
    return forward(neighbor_map(coords, extent, ks), x, w, bias, rows)


# ---------------------------------------------------------------------------
# Pure-Python twin (dict lookup, per-voxel loop) for tiny inputs.
# ---------------------------------------------------------------------------

def _offsets(kernel_size: int):
    r = kernel_size // 2
    return [(dx, dy, dz) for dx in range(-r, r + 1) for dy in range(-r, r + 1) for dz in range(-r, r + 1)]


def neighbor_map_py(coords, extent, kernel_size: int = 3, flip: bool = False) -> np.ndarray:
    coords = np.asarray(coords).reshape(-1, 4).tolist()
    ex, ey, ez = (int(v) for v in extent)
    table = {}
    for i, (b, x, y, z) in enumerate(coords):
        if not (0 <= b <= 65535 and 0 <= x < ex and 0 <= y < ey and 0 <= z < ez):
            raise OracleError(COORD_RANGE)
        if (b, x, y, z) in table:
            raise OracleError(DUPLICATE)
        table[(b, x, y, z)] = i
    offs = _offsets(kernel_size)
    s = -1 if flip else 1
    nbr = np.full((len(coords), len(offs)), -1, dtype=np.int32)
    for i, (b, x, y, z) in enumerate(coords):
        for k, (dx, dy, dz) in enumerate(offs):
            nbr[i, k] = table.get((b, x + s * dx, y + s * dy, z + s * dz), -1)
    return nbr


def forward_py(nbr, x, w, bias=None) -> np.ndarray:
    nbr = np.asarray(nbr)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    kvol, cin, cout = w.shape
    out = np.zeros((x.shape[0], cout), dtype=np.float64)
    for i in range(x.shape[0]):
        acc = [0.0] * cout if bias is None else [float(v) for v in np.asarray(bias, dtype=np.float64)]
        for k in range(kvol):
            j = int(nbr[i, k])
            if j < 0:
                continue
            for ci in range(cin):
                xv = float(x[j, ci])
                for co in range(cout):
                    acc[co] += xv * float(w[k, ci, co])
        out[i] = acc
    return out


# ---------------------------------------------------------------------------
# Resampling around the convolution: SparseDownsample (amax), SparseUpsample
# (paired with a downsample), SparseSubdivide.
# ---------------------------------------------------------------------------

def _check_coords(coords: np.ndarray, extent) -> None:
    ext = np.asarray(extent, dtype=np.int64).reshape(3)
    c = coords.astype(np.int64)
    if c.size and ((c[:, 0] < 0).any() or (c[:, 0] > 65535).any() or (c[:, 1:] < 0).any()
                   or (c[:, 1:] >= ext).any()):
        raise OracleError(COORD_RANGE)


def downsample(coords, extent, factor: int = 2):
    """Coarse voxel set of SparseDownsample(factor): returns (coarse int32 [M, 4]
    in increasing lexicographic (b, x, y, z) order, parent int32 [N] = coarse row
    of each input row, coarse extent ceil(extent / factor))."""
    coords = np.asarray(coords, dtype=np.int32).reshape(-1, 4)
    _check_coords(coords, extent)
    cells = coords.astype(np.int64).copy()
    cells[:, 1:] //= int(factor)
    # np.unique over rows sorts them lexicographically: one library sort as a step
    coarse, parent = np.unique(cells, axis=0, return_inverse=True)
    coarse_extent = tuple(-(-int(e) // int(factor)) for e in extent)
    return coarse.astype(np.int32).reshape(-1, 4), parent.astype(np.int32).reshape(-1), coarse_extent


def downsample_amax(parent, n_coarse: int, x) -> np.ndarray:
    """out[g] = element-wise max of x[i] over the rows i with parent[i] = g, where
    +0 counts as larger than -0.  Returns x's dtype (the max is one of the inputs)."""
    parent = np.asarray(parent, dtype=np.int64).reshape(-1)
    x = np.asarray(x)
    xf = x.astype(np.float64)
    out = np.full((int(n_coarse), x.shape[1]), -np.inf)
    np.maximum.at(out, parent, xf)
    # signed zero: a zero maximum is +0 when any element of its block is +0
    pos_zero = np.zeros(out.shape, dtype=bool)
    np.logical_or.at(pos_zero, parent, (xf == 0) & ~np.signbit(xf))
    zero = out == 0
    out[zero & pos_zero] = 0.0
    out[zero & ~pos_zero] = -0.0
    return out


def upsample(parent, x_coarse) -> np.ndarray:
    """SparseUpsample paired with a downsample: row i gets x_coarse[parent[i]]."""
    return np.asarray(x_coarse)[np.asarray(parent, dtype=np.int64)]


def subdivide(coords, extent, x=None):
    """SparseSubdivide: row 8 i + c (c = 4 ox + 2 oy + oz) is (b, 2x + ox, 2y + oy,
    2z + oz) with voxel i's features.  Returns (coords [8N, 4], features or None)."""
    coords = np.asarray(coords, dtype=np.int32).reshape(-1, 4)
    _check_coords(coords, extent)
    out = np.empty((8 * coords.shape[0], 4), dtype=np.int32)
    for c in range(8):
        ox, oy, oz = c >> 2, (c >> 1) & 1, c & 1
        out[c::8, 0] = coords[:, 0]
        out[c::8, 1] = 2 * coords[:, 1] + ox
        out[c::8, 2] = 2 * coords[:, 2] + oy
        out[c::8, 3] = 2 * coords[:, 3] + oz
    xo = None if x is None else np.repeat(np.asarray(x), 8, axis=0)
    return out, xo


def downsample_py(coords, factor: int = 2):
    """Pure-Python twin of ``downsample`` (dict of blocks, sorted keys), tiny inputs."""
    blocks = {}
    for i, (b, x, y, z) in enumerate(np.asarray(coords).reshape(-1, 4).tolist()):
        blocks.setdefault((b, x // factor, y // factor, z // factor), []).append(i)
    keys = sorted(blocks)
    parent = [0] * sum(len(v) for v in blocks.values())
    for g, key in enumerate(keys):
        for i in blocks[key]:
            parent[i] = g
    return np.array(keys, dtype=np.int32).reshape(-1, 4), np.array(parent, dtype=np.int32)


# ---------------------------------------------------------------------------
# Fused decoder epilogue: activation, residual add, per-channel statistics.
# ---------------------------------------------------------------------------

ACTIVATIONS = ("none", "relu", "silu", "gelu")


def activation(name: str, y) -> np.ndarray:
    """The activation applied to conv + bias, in fp64: ReLU max(y, 0); SiLU
    y * sigmoid(y) = y / (1 + exp(-y)); GELU 0.5 y (1 + erf(y / sqrt 2))."""
    y = np.asarray(y, dtype=np.float64)
    if name == "none":
        return y.copy()
    if name == "relu":
        return np.maximum(y, 0.0)
    if name == "silu":
        with np.errstate(over="ignore"):
            return y / (1.0 + np.exp(-y))
    if name == "gelu":
        from scipy.special import erf  # a library routine as one step
        return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))
    raise ValueError(f"unknown activation {name!r}")


def epilogue(conv, act: str = "none", residual=None) -> np.ndarray:
    """The stored value before rounding: act(conv) (+ residual), where conv is the
    convolution output with its bias (fp64, e.g. from ``forward``)."""
    y = activation(act, conv)
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    return y


def channel_stats(out) -> np.ndarray:
    """[2, C]: per channel the sum and the sum of squares of the stored output over
    all rows, in fp64 (out holds the stored, rounded values)."""
    o = np.asarray(out, dtype=np.float64)
    return np.stack([o.sum(axis=0), (o * o).sum(axis=0)])
