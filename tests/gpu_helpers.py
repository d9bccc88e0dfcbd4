"""Helpers shared by the GPU parity tests: tensors on cuda:0 and the tolerance check."""
import numpy as np
import torch

# Tolerances on max |out - ref| relative to the RMS of the reference output (fp64
# oracle).  fp32 accumulation gives ~1e-6 relative error over the few hundred to
# few thousand terms per output.
#
# bf16 outputs: the result is rounded to the output type (round to nearest
# even), which alone moves a value v by up to half a bf16 ulp of v -- for the rare
# outputs with |v| >= 2 at unit-scale data that is 2^-8, above 2e-2 * RMS.  The
# bf16 bound is therefore applied to the error beyond that final rounding:
#     max_i ( |out_i - ref_i| - half_ulp_bf16(max(|out_i|, |ref_i|)) ) <= 2e-2 * RMS(ref).
TOL = {"f32": 1e-5, "bf16": 2e-2}


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


def assert_close(out, ref: np.ndarray, dtype: str, rms: float | None = None):
    out_np = out.float().cpu().numpy() if isinstance(out, torch.Tensor) else out
    if rms is None:
        rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 1.0
    raw, err = errors(out_np, ref, dtype, rms)
    assert err <= TOL[dtype], f"error/rms = {err:.3e} (raw {raw:.3e}) > {TOL[dtype]:.0e}"
    return err
