"""Helpers shared by the GPU parity tests: tensors on cuda:0, the tolerance check,
and a row-parallel driver for the CPU oracle.

Tolerances are on max |out - ref| relative to the RMS of the reference output
(fp64 oracle): 1e-5 for fp32 results and 2e-2 for bf16 results.  fp32
accumulation gives ~1e-6 relative error over the few hundred to few thousand
terms per output.

bf16 outputs: the result is rounded to the output type (round to nearest even),
which alone moves a value v by up to half a bf16 ulp of v.  bf16 keeps 8
significant bits, so half an ulp is 2^-8 = 0.0039 for |v| in [1, 2) and
2^-7 = 0.0078 for |v| in [2, 4).  On the 128^3 workload the output RMS is about
0.38, so 2e-2 * RMS is about 0.0076: the rounding of an output in [2, 4) alone
can exceed the bar, and the first full-output check met such an output among
27 M.  The bf16 bound is therefore applied to the error beyond that final
rounding:

    max_i ( |out_i - ref_i| - half_ulp_bf16(max(|out_i|, |ref_i|)) ) <= 2e-2 * RMS(ref).

Every check also records the raw max |out - ref| / RMS; the tests' terminal
summary lists both figures for every comparison (``tests/conftest.py``).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

TOL = {"f32": 1e-5, "bf16": 2e-2}

# (test id, label, dtype, raw error / rms, error beyond output rounding / rms, rows compared)
RECORDS: list[tuple[str, str, str, float, float, int]] = []


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device="cuda", dtype=torch.float32 if dtype == "f32" else torch.bfloat16)


def coords_dev(coords: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).cuda()


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at magnitude |v| (8 significand bits)."""
    a = np.abs(v.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def errors(out: np.ndarray, ref: np.ndarray, dtype: str, rms: float) -> tuple[float, float]:
    """(max |out-ref| / rms, max error beyond the output rounding / rms)."""
    if out.size == 0:
        return 0.0, 0.0
    d = np.abs(out.astype(np.float64) - ref)
    raw = float(d.max() / max(rms, 1e-30))
    if dtype != "bf16":
        return raw, raw
    excess = d - half_ulp_bf16(np.maximum(np.abs(out.astype(np.float64)), np.abs(ref)))
    return raw, float(max(excess.max(), 0.0) / max(rms, 1e-30))


def assert_close(out, ref: np.ndarray, dtype: str, rms: float | None = None, label: str = ""):
    out_np = out.float().cpu().numpy() if isinstance(out, torch.Tensor) else out
    if rms is None:
        rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 1.0
    raw, err = errors(out_np, ref, dtype, rms)
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    RECORDS.append((test, label, dtype, raw, err, int(ref.shape[0]) if ref.ndim else 0))
    assert err <= TOL[dtype], f"error/rms = {err:.3e} (raw {raw:.3e}) > {TOL[dtype]:.0e}"
    return err


def oracle_forward_rows(oracle, nbr, x, w, bias, rows=None, chunk: int = 4096) -> np.ndarray:
    """oracle.forward over ``rows`` (all rows when None), split into chunks that run
    on host threads.  The oracle is called unchanged on each chunk: its C entry point
    releases the GIL, so the chunks run in parallel, and each output row is computed
    exactly as a single call would compute it."""
    n = x.shape[0]
    rows = np.arange(n, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    if rows.size <= chunk:
        return oracle.forward(nbr, x, w, bias, rows=rows)
    nbr = np.ascontiguousarray(nbr, dtype=np.int32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    parts = [rows[i:i + chunk] for i in range(0, rows.size, chunk)]
    workers = max(1, min(len(parts), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        outs = list(ex.map(lambda r: oracle.forward(nbr, x, w, bias, rows=r), parts))
    return np.concatenate(outs)
