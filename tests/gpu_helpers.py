"""Helpers shared by the GPU parity tests: tensors on cuda:0 and the tolerance check."""
import numpy as np
import torch

# Tolerances on max |out - ref| relative to the RMS of the whole reference output
# (fp64 oracle): fp32 accumulation gives ~1e-6 relative error over the few hundred
# to few thousand terms per output; the bf16 bound also covers the final rounding
# of the output to bf16 (2^-9 relative).
TOL = {"f32": 1e-5, "bf16": 2e-2}


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device="cuda", dtype=torch.float32 if dtype == "f32" else torch.bfloat16)


def coords_dev(coords: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).cuda()


def rel_err(out: np.ndarray, ref: np.ndarray, rms: float) -> float:
    return float(np.max(np.abs(out.astype(np.float64) - ref)) / max(rms, 1e-30)) if out.size else 0.0


def assert_close(out, ref: np.ndarray, dtype: str, rms: float | None = None):
    out_np = out.float().cpu().numpy() if isinstance(out, torch.Tensor) else out
    if rms is None:
        rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 1.0
    err = rel_err(out_np, ref, rms)
    assert err <= TOL[dtype], f"max|out-ref|/rms = {err:.3e} > {TOL[dtype]:.0e}"
    return err
