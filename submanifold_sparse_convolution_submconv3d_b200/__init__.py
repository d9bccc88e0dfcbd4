"""Python binding of the B200 SubMConv3d library (``include/spconv.h``).

Argument marshalling only: every step of the hot path (map build, gather, GEMM,
store) runs in the CUDA library ``libspconv_b200.so``.  PyTorch supplies device
memory and the current stream.  Importing this package fails loudly if the
library has not been built (``python -m submanifold_sparse_convolution_submconv3d_b200.build``).

The functions carry the C names:

* ``spconv_build_map(coords, extent, kernel_size=3, flip_kernel=False, sorted_keys=False)``
  -> ``SubmMap`` (``spconv_build_map_ex`` when an option is set)
* ``spconv_subm_forward(map, x, w, bias=None, out=None)`` -> ``out``
* ``spconv_free(map)``
* ``spconv_downsample_build(coords, extent, factor=2)`` -> ``Downsample``;
  ``spconv_downsample_amax(ds, x)``, ``spconv_upsample(ds, x_coarse)``
* ``spconv_subdivide(coords, extent, x=None)`` -> ``(coords_out, x_out)``
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspconv_b200.so")

OK, INVALID_ARG, UNSUPPORTED, COORD_RANGE, DUPLICATE, TABLE_FULL, OOM, CUDA_ERROR, TIMEOUT = range(9)
MAP_DEFAULT, MAP_FLIP_KERNEL, MAP_SORTED_KEYS, MAP_HASH_TABLE, MAP_SHORT_TILES = 0, 1, 2, 4, 8
ALGO_AUTO, ALGO_SIMT, ALGO_TCGEN05 = 0, 1, 2
KERNEL_SIMT, KERNEL_TCGEN05, KERNEL_TCGEN05_GEMM = 0, 1, 2
KERNEL_NAMES = ("simt", "tcgen05", "tcgen05_gemm")
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}

EXPORTED = ("spconv_build_map", "spconv_subm_forward", "spconv_free", "spconv_map_info", "spconv_map_check",
            "spconv_map_tile_rows",
            "spconv_last_error", "spconv_subm_forward_algo", "spconv_debug_set_table_slots",
            "spconv_debug_set_tile_rows", "spconv_build_neighbor_map_noalloc", "spconv_map_launch_counts",
            "spconv_map_stats", "spconv_debug_set_ring_depths", "spconv_build_map_ex", "spconv_downsample_build",
            "spconv_downsample_info", "spconv_downsample_amax", "spconv_upsample", "spconv_downsample_free",
            "spconv_subdivide", "spconv_subm_forward_ex")


class _MapStats(ctypes.Structure):
    _fields_ = [("tiles", ctypes.c_int64), ("rows_per_tile", ctypes.c_int32), ("job_stride", ctypes.c_int32),
                ("spans", ctypes.c_int64), ("span_cols", ctypes.c_int64), ("perm_dev", ctypes.c_void_p),
                ("nbr_t_dev", ctypes.c_void_p), ("jobs_dev", ctypes.c_void_p), ("order_dev", ctypes.c_void_p)]


class _Epilogue(ctypes.Structure):
    _fields_ = [("act", ctypes.c_int), ("residual", ctypes.c_void_p), ("stats", ctypes.c_void_p)]


ACTIVATIONS = {None: 0, "none": 0, "relu": 1, "silu": 2, "gelu": 3}


class SpconvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"spconv status {status}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run python -m submanifold_sparse_convolution_submconv3d_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.spconv_build_map.argtypes = [vp, i64, vp, i32, vp, ctypes.POINTER(vp)]
    lib.spconv_subm_forward.argtypes = [vp, ctypes.c_int, vp, i32, vp, vp, vp, i32, vp]
    lib.spconv_subm_forward_algo.argtypes = [vp, ctypes.c_int, vp, i32, vp, vp, vp, i32, ctypes.c_int, vp]
    lib.spconv_free.argtypes = [vp]
    lib.spconv_map_info.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(i32), ctypes.POINTER(i64),
                                    ctypes.POINTER(vp)]
    lib.spconv_map_check.argtypes = [vp, vp]
    lib.spconv_map_tile_rows.argtypes = [vp, ctypes.POINTER(i32)]
    lib.spconv_debug_set_table_slots.argtypes = [i64]
    lib.spconv_debug_set_tile_rows.argtypes = [i32]
    lib.spconv_build_neighbor_map_noalloc.argtypes = [vp, i64, vp, vp, ctypes.POINTER(i64), vp]
    lib.spconv_map_launch_counts.argtypes = [vp, ctypes.POINTER(i64), i32]
    lib.spconv_map_stats.argtypes = [vp, ctypes.POINTER(_MapStats)]
    lib.spconv_debug_set_ring_depths.argtypes = [i32, i32]
    lib.spconv_build_map_ex.argtypes = [vp, i64, vp, i32, ctypes.c_uint32, vp, ctypes.POINTER(vp)]
    lib.spconv_downsample_build.argtypes = [vp, i64, vp, i32, vp, ctypes.POINTER(vp)]
    lib.spconv_downsample_info.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), vp, ctypes.POINTER(vp),
                                           ctypes.POINTER(vp)]
    lib.spconv_downsample_amax.argtypes = [vp, ctypes.c_int, vp, i32, vp, vp]
    lib.spconv_upsample.argtypes = [vp, ctypes.c_int, vp, i32, vp, vp]
    lib.spconv_downsample_free.argtypes = [vp]
    lib.spconv_subdivide.argtypes = [vp, i64, vp, ctypes.c_int, vp, i32, vp, vp, vp]
    lib.spconv_subm_forward_ex.argtypes = [vp, ctypes.c_int, vp, i32, vp, vp, vp, i32, ctypes.POINTER(_Epilogue),
                                           ctypes.c_int, vp]
    lib.spconv_last_error.restype = ctypes.c_char_p
    for name in ("spconv_build_map", "spconv_subm_forward", "spconv_subm_forward_algo", "spconv_free",
                 "spconv_map_info", "spconv_map_check", "spconv_map_tile_rows", "spconv_debug_set_table_slots",
                 "spconv_debug_set_tile_rows", "spconv_build_neighbor_map_noalloc", "spconv_map_launch_counts",
                 "spconv_map_stats", "spconv_debug_set_ring_depths", "spconv_build_map_ex",
                 "spconv_downsample_build", "spconv_downsample_info", "spconv_downsample_amax", "spconv_upsample",
                 "spconv_downsample_free", "spconv_subdivide", "spconv_subm_forward_ex"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


try:
    lib = _load()
    _LOAD_ERROR = None
except (OSError, AttributeError, ImportError) as _exc:  # missing or stale library
    lib = None
    _LOAD_ERROR = _exc


def _require() -> None:
    """Raise if the CUDA library could not be loaded: there is no fallback path."""
    if lib is None:
        raise ImportError(f"the CUDA library {LIB_PATH} is unavailable ({_LOAD_ERROR}); build it with "
                          "python -m submanifold_sparse_convolution_submconv3d_b200.build")


def _check(status: int) -> None:
    if status != OK:
        raise SpconvError(status, lib.spconv_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class SubmMap:
    """Owns a neighbour-map handle; freed by ``free()`` or garbage collection."""

    def __init__(self, handle: int, device: torch.device):
        self.handle = handle
        self.device = device
        n, ks, pairs, ptr = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int64(), ctypes.c_void_p()
        _check(lib.spconv_map_info(handle, ctypes.byref(n), ctypes.byref(ks), ctypes.byref(pairs), ctypes.byref(ptr)))
        self.n, self.kernel_size, self.pairs = n.value, ks.value, pairs.value
        self._nbr_ptr = ptr.value
        rows = ctypes.c_int32()
        _check(lib.spconv_map_tile_rows(handle, ctypes.byref(rows)))
        self.tile_rows = rows.value  # rows per forward tile (<= 384)

    def _copy_device(self, ptr: int, shape: tuple, typestr: str, dtype) -> torch.Tensor:
        """Copy of a library-owned device buffer, viewed through the CUDA array interface."""
        out = torch.empty(shape, dtype=dtype, device=self.device)
        if out.numel():
            class _View:
                __cuda_array_interface__ = {"shape": shape, "typestr": typestr, "data": (ptr, False), "version": 3}
            out.copy_(torch.as_tensor(_View(), device=self.device))
        return out

    def neighbor_map(self) -> torch.Tensor:
        """Copy of the dense int32 [n, 27] map (identity column for kernel size 1)."""
        if self.kernel_size == 1:
            return torch.arange(self.n, dtype=torch.int32, device=self.device).view(-1, 1)
        return self._copy_device(self._nbr_ptr, (self.n, 27), "<i4", torch.int32)

    def stats(self, copy_arrays: bool = False) -> dict:
        """The tensor-core forward's metadata (spconv_map_stats): tiling, span counts
        and, with copy_arrays, copies of perm [n], nbr_t [27, tiles * rows_per_tile],
        jobs [tiles, job_stride] (uint32 words as int64) and order [tiles]."""
        st = _MapStats()
        _check(lib.spconv_map_stats(self.handle, ctypes.byref(st)))
        d = {"tiles": st.tiles, "rows_per_tile": st.rows_per_tile, "job_stride": st.job_stride, "spans": st.spans,
             "span_cols": st.span_cols}
        if copy_arrays and st.perm_dev:
            npad = st.tiles * st.rows_per_tile
            d["perm"] = self._copy_device(st.perm_dev, (self.n,), "<i4", torch.int32)
            d["nbr_t"] = self._copy_device(st.nbr_t_dev, (27, npad), "<i4", torch.int32)
            d["jobs"] = self._copy_device(st.jobs_dev, (st.tiles, st.job_stride), "<i4",
                                          torch.int32).to(torch.int64) & 0xFFFFFFFF
            d["order"] = self._copy_device(st.order_dev, (st.tiles,), "<i4", torch.int32)
        return d

    def launch_counts(self) -> dict:
        """Forward launches on this map per kernel family, e.g. {"simt": 0, "tcgen05": 3}."""
        counts = (ctypes.c_int64 * len(KERNEL_NAMES))()
        _check(lib.spconv_map_launch_counts(self.handle, counts, len(KERNEL_NAMES)))
        return dict(zip(KERNEL_NAMES, counts))

    def check(self, stream=None) -> None:
        """Synchronise and raise if a forward kernel's bounded wait gave up.  The
        default stream is the current stream of the map's device."""
        with torch.cuda.device(self.device):
            _check(lib.spconv_map_check(self.handle, _stream(stream)))

    def free(self) -> None:
        if self.handle:
            lib.spconv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def _coords_arg(coords: torch.Tensor) -> torch.Tensor:
    if coords.dtype != torch.int32 or not coords.is_cuda or coords.dim() != 2 or coords.shape[1] != 4:
        raise ValueError("coords must be a CUDA int32 tensor of shape [N, 4]")
    return coords.contiguous()


def spconv_build_map(coords: torch.Tensor, extent, kernel_size: int = 3, stream=None, flip_kernel: bool = False,
                     sorted_keys: bool | None = None, short_tiles: bool = False) -> SubmMap:
    """Build the neighbour map of int32 [N, 4] (b, x, y, z) CUDA coordinates.
    ``flip_kernel`` gathers p - d_k; ``sorted_keys`` True builds the dictionary from
    sorted keys instead of the hash table (same map; None and False: the hash table);
    ``short_tiles`` cuts the forward's tiles at 128 rows (faster for layers with 128
    or more input channels)."""
    _require()
    coords = _coords_arg(coords)
    ext = (ctypes.c_int32 * 3)(*[int(v) for v in extent])
    handle = ctypes.c_void_p()
    flags = (MAP_FLIP_KERNEL if flip_kernel else 0) | (MAP_SHORT_TILES if short_tiles else 0) | \
        {None: 0, True: MAP_SORTED_KEYS, False: MAP_HASH_TABLE}[sorted_keys]
    with torch.cuda.device(coords.device):
        ptr = coords.data_ptr() if coords.numel() else None
        if flags:
            _check(lib.spconv_build_map_ex(ptr, coords.shape[0], ext, kernel_size, flags, _stream(stream),
                                           ctypes.byref(handle)))
        else:
            _check(lib.spconv_build_map(ptr, coords.shape[0], ext, kernel_size, _stream(stream),
                                        ctypes.byref(handle)))
    return SubmMap(handle.value, coords.device)


def spconv_subm_forward(m: SubmMap, x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None = None,
                        out: torch.Tensor | None = None, algo: int = ALGO_AUTO, stream=None, act: str | None = None,
                        residual: torch.Tensor | None = None, stats: torch.Tensor | None = None) -> torch.Tensor:
    """One SubMConv3d layer: x [N, Cin], w [K^3, Cin, Cout], bias [Cout] -> out [N, Cout].
    Fused epilogue (spconv_subm_forward_ex): out = act(conv + bias) (+ residual [N, Cout],
    which may be ``out`` itself); ``stats``, a float32 CUDA tensor [2, Cout], receives the
    per-channel sum and sum of squares of out."""
    _require()
    if x.dtype not in _DTYPES:
        raise ValueError("x must be float32 or bfloat16")
    for t in (w,) + (() if bias is None else (bias,)):
        if t.dtype != x.dtype or t.device != x.device:
            raise ValueError("w and bias must match x in dtype and device")
    if x.dim() != 2 or w.dim() != 3:
        raise ValueError(f"x must be [N, Cin] and w [K^3, Cin, Cout]; got x {tuple(x.shape)}, w {tuple(w.shape)}")
    cin, cout = int(w.shape[1]), int(w.shape[2])
    if x.shape != (m.n, cin) or w.shape[0] != m.kernel_size ** 3:
        raise ValueError(f"shape mismatch: x {tuple(x.shape)}, w {tuple(w.shape)}, map n={m.n} k={m.kernel_size}")
    if bias is not None and bias.shape != (cout,):
        raise ValueError(f"bias must be [Cout] = [{cout}]; got {tuple(bias.shape)}")
    if out is not None and (out.shape != (m.n, cout) or out.dtype != x.dtype or not out.is_contiguous()):
        raise ValueError("out must be a contiguous [N, Cout] tensor of x's dtype")
    # The library reads and writes these through raw device pointers: a host
    # tensor, or one on another GPU than the map, must never reach it.
    if not x.is_cuda or x.device != m.device or (out is not None and out.device != x.device):
        raise ValueError(f"x, w, bias and out must be CUDA tensors on the map's device {m.device}")
    if act not in ACTIVATIONS:
        raise ValueError(f"act must be one of {sorted(k for k in ACTIVATIONS if k)} or None")
    if residual is not None and (residual.shape != (m.n, cout) or residual.dtype != x.dtype
                                 or residual.device != x.device or not residual.is_contiguous()):
        raise ValueError("residual must be a contiguous [N, Cout] tensor of x's dtype on x's device")
    if stats is not None and (stats.shape != (2, cout) or stats.dtype != torch.float32
                              or stats.device != x.device or not stats.is_contiguous()):
        raise ValueError("stats must be a contiguous float32 [2, Cout] tensor on x's device")
    x, w = x.contiguous(), w.contiguous()
    bias = None if bias is None else bias.contiguous()
    if out is None:
        out = torch.empty((m.n, cout), dtype=x.dtype, device=x.device)
    if m.n == 0:
        if stats is not None:
            stats.zero_()
        return out
    with torch.cuda.device(x.device):
        if ACTIVATIONS[act] or residual is not None or stats is not None:
            epi = _Epilogue(ACTIVATIONS[act], None if residual is None else residual.data_ptr(),
                            None if stats is None else stats.data_ptr())
            _check(lib.spconv_subm_forward_ex(m.handle, _DTYPES[x.dtype], x.data_ptr(), cin, w.data_ptr(),
                                              None if bias is None else bias.data_ptr(), out.data_ptr(), cout,
                                              ctypes.byref(epi), algo, _stream(stream)))
        else:
            _check(lib.spconv_subm_forward_algo(m.handle, _DTYPES[x.dtype], x.data_ptr(), cin, w.data_ptr(),
                                                None if bias is None else bias.data_ptr(), out.data_ptr(), cout,
                                                algo, _stream(stream)))
    return out


def spconv_free(m: SubmMap) -> None:
    m.free()


def spconv_build_neighbor_map_noalloc(coords: torch.Tensor, extent, out: torch.Tensor | None = None,
                                      stream=None) -> tuple[torch.Tensor, int]:
    """Dense int32 [N, 27] neighbour map built without any device allocation by
    the library (scratch in a static device array; N <= 524288).  The caller may
    pass ``out``; otherwise the binding allocates it with torch before the call.
    Returns (map, pairs)."""
    _require()
    if coords.dtype != torch.int32 or not coords.is_cuda or coords.dim() != 2 or coords.shape[1] != 4:
        raise ValueError("coords must be a CUDA int32 tensor of shape [N, 4]")
    coords = coords.contiguous()
    n = coords.shape[0]
    if out is None:
        out = torch.empty((n, 27), dtype=torch.int32, device=coords.device)
    elif out.shape != (n, 27) or out.dtype != torch.int32 or not out.is_contiguous() or out.device != coords.device:
        raise ValueError("out must be a contiguous int32 [N, 27] tensor on the device of coords")
    ext = (ctypes.c_int32 * 3)(*[int(v) for v in extent])
    pairs = ctypes.c_int64()
    with torch.cuda.device(coords.device):
        _check(lib.spconv_build_neighbor_map_noalloc(coords.data_ptr() if n else None, n, ext,
                                                     out.data_ptr() if n else None, ctypes.byref(pairs),
                                                     _stream(stream)))
    return out, pairs.value


class Downsample:
    """Owns a downsample handle (spconv_downsample_build): the coarse voxel set and
    the pairing of input voxels with coarse voxels."""

    def __init__(self, handle: int, device: torch.device):
        self.handle = handle
        self.device = device
        nf, nc, ext = ctypes.c_int64(), ctypes.c_int64(), (ctypes.c_int32 * 3)()
        cptr, pptr = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib.spconv_downsample_info(handle, ctypes.byref(nf), ctypes.byref(nc), ext, ctypes.byref(cptr),
                                          ctypes.byref(pptr)))
        self.n, self.n_coarse, self.coarse_extent = nf.value, nc.value, tuple(ext)
        self._coarse_ptr, self._parent_ptr = cptr.value, pptr.value

    def _copy(self, ptr, shape) -> torch.Tensor:
        out = torch.empty(shape, dtype=torch.int32, device=self.device)
        if out.numel():
            class _View:
                __cuda_array_interface__ = {"shape": shape, "typestr": "<i4", "data": (ptr, False), "version": 3}
            out.copy_(torch.as_tensor(_View(), device=self.device))
        return out

    def coarse_coords(self) -> torch.Tensor:
        """Copy of the coarse coordinates, int32 [n_coarse, 4], sorted."""
        return self._copy(self._coarse_ptr, (self.n_coarse, 4))

    def parent(self) -> torch.Tensor:
        """Copy of the coarse row of every input row, int32 [n]."""
        return self._copy(self._parent_ptr, (self.n,))

    def free(self) -> None:
        if self.handle:
            lib.spconv_downsample_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def spconv_downsample_build(coords: torch.Tensor, extent, factor: int = 2, stream=None) -> Downsample:
    """SparseDownsample(factor) coordinates of int32 [N, 4] CUDA coordinates."""
    _require()
    coords = _coords_arg(coords)
    ext = (ctypes.c_int32 * 3)(*[int(v) for v in extent])
    handle = ctypes.c_void_p()
    with torch.cuda.device(coords.device):
        _check(lib.spconv_downsample_build(coords.data_ptr() if coords.numel() else None, coords.shape[0], ext,
                                           int(factor), _stream(stream), ctypes.byref(handle)))
    return Downsample(handle.value, coords.device)


def _rows_arg(x: torch.Tensor, rows: int, device, what: str) -> torch.Tensor:
    if x.dtype not in _DTYPES or not x.is_cuda or x.device != device or x.dim() != 2 or x.shape[0] != rows:
        raise ValueError(f"{what} must be a float32 or bfloat16 CUDA tensor [{rows}, C] on {device}")
    return x.contiguous()


def spconv_downsample_amax(ds: Downsample, x: torch.Tensor, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """Max pooling of x [n, C] onto the coarse voxels -> [n_coarse, C]."""
    _require()
    x = _rows_arg(x, ds.n, ds.device, "x")
    if out is None:
        out = torch.empty((ds.n_coarse, x.shape[1]), dtype=x.dtype, device=x.device)
    elif out.shape != (ds.n_coarse, x.shape[1]) or out.dtype != x.dtype or not out.is_contiguous() \
            or out.device != x.device:
        raise ValueError("out must be a contiguous [n_coarse, C] tensor like x")
    if ds.n:
        with torch.cuda.device(x.device):
            _check(lib.spconv_downsample_amax(ds.handle, _DTYPES[x.dtype], x.data_ptr(), x.shape[1], out.data_ptr(),
                                              _stream(stream)))
    return out


def spconv_upsample(ds: Downsample, x_coarse: torch.Tensor, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Coarse features [n_coarse, C] back onto the downsample's input voxels -> [n, C]."""
    _require()
    x_coarse = _rows_arg(x_coarse, ds.n_coarse, ds.device, "x_coarse")
    if out is None:
        out = torch.empty((ds.n, x_coarse.shape[1]), dtype=x_coarse.dtype, device=x_coarse.device)
    elif out.shape != (ds.n, x_coarse.shape[1]) or out.dtype != x_coarse.dtype or not out.is_contiguous() \
            or out.device != x_coarse.device:
        raise ValueError("out must be a contiguous [n, C] tensor like x_coarse")
    if ds.n:
        with torch.cuda.device(x_coarse.device):
            _check(lib.spconv_upsample(ds.handle, _DTYPES[x_coarse.dtype], x_coarse.data_ptr(), x_coarse.shape[1],
                                       out.data_ptr(), _stream(stream)))
    return out


def spconv_subdivide(coords: torch.Tensor, extent, x: torch.Tensor | None = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
    """SparseSubdivide: int32 [N, 4] coordinates (and optional features [N, C]) ->
    the 8 N children (coordinates [8N, 4], features [8N, C]) on the grid 2 * extent."""
    _require()
    coords = _coords_arg(coords)
    n = coords.shape[0]
    ext = (ctypes.c_int32 * 3)(*[int(v) for v in extent])
    coords_out = torch.empty((8 * n, 4), dtype=torch.int32, device=coords.device)
    x_out = None
    if x is not None:
        x = _rows_arg(x, n, coords.device, "x")
        x_out = torch.empty((8 * n, x.shape[1]), dtype=x.dtype, device=x.device)
    with torch.cuda.device(coords.device):
        _check(lib.spconv_subdivide(coords.data_ptr() if n else None, n, ext,
                                    _DTYPES[x.dtype] if x is not None else 0,
                                    x.data_ptr() if x is not None and n else None,
                                    x.shape[1] if x is not None else 0, coords_out.data_ptr() if n else None,
                                    x_out.data_ptr() if x_out is not None and n else None, _stream(stream)))
    return coords_out, x_out


def spconv_debug_set_table_slots(slots: int) -> None:
    _require()
    _check(lib.spconv_debug_set_table_slots(int(slots)))


def spconv_debug_set_tile_rows(rows: int) -> None:
    _require()
    _check(lib.spconv_debug_set_tile_rows(int(rows)))


def spconv_debug_set_ring_depths(a_slots: int, b_units: int) -> None:
    _require()
    _check(lib.spconv_debug_set_ring_depths(int(a_slots), int(b_units)))


__all__ = ["OK", "INVALID_ARG", "UNSUPPORTED", "COORD_RANGE", "DUPLICATE", "TABLE_FULL", "OOM", "CUDA_ERROR",
           "TIMEOUT", "SubmMap", "SpconvError", "spconv_build_map", "spconv_subm_forward", "spconv_free",
           "spconv_debug_set_table_slots", "spconv_debug_set_tile_rows", "spconv_debug_set_ring_depths",
           "spconv_build_neighbor_map_noalloc", "lib", "Downsample", "spconv_downsample_build",
           "spconv_downsample_amax", "spconv_upsample", "spconv_subdivide", "MAP_DEFAULT", "MAP_FLIP_KERNEL",
           "MAP_SORTED_KEYS", "MAP_HASH_TABLE", "MAP_SHORT_TILES", "ACTIVATIONS",
           "LIB_PATH", "EXPORTED",
           "ALGO_AUTO", "ALGO_SIMT", "ALGO_TCGEN05", "KERNEL_SIMT", "KERNEL_TCGEN05", "KERNEL_TCGEN05_GEMM",
           "KERNEL_NAMES"]
