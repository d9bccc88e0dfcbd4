"""Seeded synthetic inputs for SubMConv3d: coordinates, features, weights, bias.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It holds no convolution arithmetic: it only draws inputs.

Workloads (shapes and value distributions follow the pages' benchmark and the
TRELLIS.2-family decoders they describe):

* ``tiny``     -- 16^3 grid, 410 voxels uniform without replacement, fp32, 16->16.
* ``uniform``  -- 128^3 grid, 209,715 voxels (~10 %) uniform without replacement,
                  bf16, 128->128, ten layers on one map.  This is the workload of the
                  "Fleet benchmark" table of the lato.2_mrp_mlx README.
* ``shells``   -- 256^3 grid, 1-voxel-thick shells of 6 ellipsoids, bf16, 64->64.
* ``batched``  -- 4 independent 64^3 shell shapes (3-8 ellipsoids each), bf16,
                  512->512, a k=3 layer then a k=1 layer.
* ``large``    -- 512^3 grid, shells of 12 ellipsoids, bf16, 32->64.

Draw order within one workload: coordinates, features, weights, bias (one numpy
``default_rng(seed)`` stream).  Weight variance reads "N(0, 1/(27*C))" as a
variance, so the standard deviation is (27*Cin)^-1/2 (Cin^-1/2 for k=1); bias
variance is 0.01.  bf16 inputs are drawn in fp32 and rounded to the nearest bf16
(ties to even), so every side sees the same exactly representable values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Layer", "Workload", "round_to_bf16", "uniform_coords", "shell_coords",
    "make_workload", "WORKLOADS",
]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding them.

    Inputs here are finite normal draws, so no NaN/Inf handling is needed.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def uniform_coords(rng: np.random.Generator, grid: int, n: int, batch: int = 0) -> np.ndarray:
    """n distinct voxels of a grid^3 cube, uniform without replacement, in draw order.

    The flat index unflattens as x = idx // grid^2, y = (idx // grid) % grid,
    z = idx % grid.  Returns int32 [n, 4] = (batch, x, y, z).
    """
    idx = rng.choice(grid ** 3, n, replace=False).astype(np.int64)
    out = np.empty((n, 4), dtype=np.int32)
    out[:, 0] = batch
    out[:, 1] = idx // (grid * grid)
    out[:, 2] = (idx // grid) % grid
    out[:, 3] = idx % grid
    return out


def _ellipsoid_shell(grid: int, c: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Voxels v in [0, grid)^3 with f(v) <= 1 and some 6-neighbour with f > 1.

    f(v) = sum_a ((v_a - c_a) / r_a)^2, evaluated in fp64 for every voxel and
    every neighbour (neighbours outside the grid are evaluated too: the shell
    is a property of the ellipsoid, then clipped to the grid).
    """
    lo = np.maximum(np.floor(c - r).astype(np.int64) - 1, 0)
    hi = np.minimum(np.ceil(c + r).astype(np.int64) + 1, grid - 1)
    if np.any(hi < lo):
        return np.zeros((0, 3), dtype=np.int32)
    ys = np.arange(lo[1] - 1, hi[1] + 2, dtype=np.float64)
    zs = np.arange(lo[2] - 1, hi[2] + 2, dtype=np.float64)
    gy = ((ys - c[1]) / r[1]) ** 2
    gz = ((zs - c[2]) / r[2]) ** 2
    plane_yz = gy[:, None] + gz[None, :]  # includes a 1-voxel margin in y and z

    def fx(x: int) -> np.ndarray:
        return ((x - c[0]) / r[0]) ** 2 + plane_yz

    pts = []
    f_prev = fx(lo[0] - 1)
    f_cur = fx(lo[0])
    for x in range(lo[0], hi[0] + 1):
        f_next = fx(x + 1)
        core = f_cur[1:-1, 1:-1]
        inside = core <= 1.0
        if inside.any():
            out_nb = ((f_prev[1:-1, 1:-1] > 1.0) | (f_next[1:-1, 1:-1] > 1.0)
                      | (f_cur[:-2, 1:-1] > 1.0) | (f_cur[2:, 1:-1] > 1.0)
                      | (f_cur[1:-1, :-2] > 1.0) | (f_cur[1:-1, 2:] > 1.0))
            yy, zz = np.nonzero(inside & out_nb)
            if yy.size:
                p = np.empty((yy.size, 3), dtype=np.int32)
                p[:, 0] = x
                p[:, 1] = yy + lo[1]
                p[:, 2] = zz + lo[2]
                pts.append(p)
        f_prev, f_cur = f_cur, f_next
    if not pts:
        return np.zeros((0, 3), dtype=np.int32)
    p = np.concatenate(pts)
    keep = np.all((p >= 0) & (p < grid), axis=1)
    return p[keep]


def shell_coords(rng: np.random.Generator, grid: int, n_ellipsoids: int,
                 axis_lo: float, axis_hi: float, batch: int = 0) -> np.ndarray:
    """Union of 1-voxel-thick axis-aligned ellipsoid shells, deduplicated, sorted.

    Centres are uniform (real valued) in [grid/4, 3*grid/4)^3 and semi-axes
    uniform in [axis_lo, axis_hi] per axis; each ellipsoid draws its centre then
    its three semi-axes.  Returns int32 [n, 4] = (batch, x, y, z), sorted
    lexicographically.
    """
    shells = []
    for _ in range(n_ellipsoids):
        c = rng.uniform(grid / 4, 3 * grid / 4, size=3)
        r = rng.uniform(axis_lo, axis_hi, size=3)
        shells.append(_ellipsoid_shell(grid, c, r))
    xyz = np.unique(np.concatenate(shells), axis=0)  # sorts lexicographically
    out = np.empty((xyz.shape[0], 4), dtype=np.int32)
    out[:, 0] = batch
    out[:, 1:] = xyz
    return out


@dataclass
class Layer:
    """One SubMConv3d layer's parameters: w [K^3, Cin, Cout], bias [Cout] or None."""
    kernel_size: int
    w: np.ndarray
    bias: np.ndarray | None


@dataclass
class Workload:
    name: str
    grid: tuple[int, int, int]
    coords: np.ndarray          # int32 [N, 4]
    x: np.ndarray               # fp32 [N, Cin] (bf16-exact values when dtype == "bf16")
    dtype: str                  # "f32" or "bf16"
    layers: list[Layer] = field(default_factory=list)
    chained: bool = False       # layer i+1 consumes layer i's output

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])


def _weights(rng, kvol, cin, cout, dtype):
    w = rng.standard_normal((kvol, cin, cout), dtype=np.float32) * np.float32((kvol * cin) ** -0.5)
    return round_to_bf16(w) if dtype == "bf16" else w


def _bias(rng, cout, dtype):
    b = rng.standard_normal(cout, dtype=np.float32) * np.float32(0.1)
    return round_to_bf16(b) if dtype == "bf16" else b


def _features(rng, n, c, dtype):
    x = rng.standard_normal((n, c), dtype=np.float32)
    return round_to_bf16(x) if dtype == "bf16" else x


def make_workload(name: str, seed: int = 0, n_layers: int | None = None) -> Workload:
    """Build one named workload from ``seed`` (see the module docstring)."""
    rng = np.random.default_rng(seed)
    if name == "tiny":
        coords = uniform_coords(rng, 16, 410)
        x = _features(rng, coords.shape[0], 16, "f32")
        w3 = _weights(rng, 27, 16, 16, "f32")
        b = _bias(rng, 16, "f32")
        w1 = _weights(rng, 1, 16, 16, "f32")
        return Workload(name, (16, 16, 16), coords, x, "f32",
                        [Layer(3, w3, b), Layer(1, w1, b)], chained=False)
    if name == "uniform":
        coords = uniform_coords(rng, 128, 209715)
        x = _features(rng, coords.shape[0], 128, "bf16")
        layers = []
        for _ in range(10 if n_layers is None else n_layers):
            w = _weights(rng, 27, 128, 128, "bf16")
            layers.append(Layer(3, w, _bias(rng, 128, "bf16")))
        return Workload(name, (128, 128, 128), coords, x, "bf16", layers, chained=True)
    if name == "shells":
        coords = shell_coords(rng, 256, 6, 20.0, 100.0)
        x = _features(rng, coords.shape[0], 64, "bf16")
        w = _weights(rng, 27, 64, 64, "bf16")
        return Workload(name, (256, 256, 256), coords, x, "bf16", [Layer(3, w, _bias(rng, 64, "bf16"))])
    if name == "batched":
        items = []
        for b in range(4):
            k = int(rng.integers(3, 9))
            items.append(shell_coords(rng, 64, k, 5.0, 25.0, batch=b))
        coords = np.concatenate(items)
        x = _features(rng, coords.shape[0], 512, "bf16")
        w3 = _weights(rng, 27, 512, 512, "bf16")
        b3 = _bias(rng, 512, "bf16")
        w1 = _weights(rng, 1, 512, 512, "bf16")
        b1 = _bias(rng, 512, "bf16")
        return Workload(name, (64, 64, 64), coords, x, "bf16",
                        [Layer(3, w3, b3), Layer(1, w1, b1)], chained=True)
    if name == "large":
        coords = shell_coords(rng, 512, 12, 40.0, 220.0)
        x = _features(rng, coords.shape[0], 32, "bf16")
        w = _weights(rng, 27, 32, 64, "bf16")
        return Workload(name, (512, 512, 512), coords, x, "bf16", [Layer(3, w, _bias(rng, 64, "bf16"))])
    raise ValueError(f"unknown workload {name!r}")


WORKLOADS = ("tiny", "uniform", "shells", "batched", "large")
