"""Pins of the bf16 tolerance helper that every bf16 parity test uses, against
torch's own bf16 format (CPU only).

The parity reading for bf16 outputs is: the error beyond the output's own
rounding to bf16 (half a bf16 spacing at the value) must stay within 2e-2 of the
output RMS.  These tests check that half_ulp_bf16 is exactly that half spacing,
so the tolerance is neither looser nor tighter than the format."""
import numpy as np
import torch

from gpu_helpers import TOL, errors, half_ulp_bf16


def _bf16_values(rng, count):
    """Positive normal bf16 numbers spread over many binades, as float64."""
    mags = np.ldexp(rng.uniform(1.0, 2.0, count), rng.integers(-100, 100, count))
    return torch.from_numpy(mags).to(torch.bfloat16).double().numpy()


def test_half_ulp_is_half_the_spacing_of_adjacent_bf16_numbers():
    r = _bf16_values(np.random.default_rng(0), 20000)
    t = torch.from_numpy(r).to(torch.bfloat16)
    nxt = (t.view(torch.int16) + 1).view(torch.bfloat16).double().numpy()  # next bf16 upwards
    spacing = nxt - r
    # in the binade [2^e, 2^(e+1)) bf16 numbers are 2^(e-7) apart (8 significand bits)
    assert np.array_equal(spacing, 2.0 * half_ulp_bf16(r))
    assert np.array_equal(half_ulp_bf16(-r), half_ulp_bf16(r))


def test_round_to_nearest_error_is_within_half_ulp_and_reaches_it():
    rng = np.random.default_rng(1)
    v = np.ldexp(rng.uniform(-2.0, 2.0, 200000), rng.integers(-60, 60, 200000))
    r = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    bound = half_ulp_bf16(np.maximum(np.abs(r), np.abs(v)))
    assert np.all(np.abs(r - v) <= bound)
    # ties (exact midpoints) reach the bound: the helper is not looser than needed
    lo = _bf16_values(rng, 1000)
    mid = lo + half_ulp_bf16(lo)
    rm = torch.from_numpy(mid).to(torch.bfloat16).double().numpy()
    assert np.array_equal(np.abs(rm - mid), half_ulp_bf16(lo))


def test_errors_discounts_exactly_the_output_rounding():
    """A result that is the exact value rounded to bf16 has no excess error; one
    bf16 step further off has an excess of one half spacing."""
    rng = np.random.default_rng(2)
    ref = rng.standard_normal(5000) * 3.0
    out = torch.from_numpy(ref).to(torch.bfloat16)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    raw, excess = errors(out.float().numpy(), ref, "bf16", rms)
    assert excess == 0.0 and raw > 0.0
    off = (out.view(torch.int16) + 1).view(torch.bfloat16).float().numpy()  # one step away from |ref|'s rounding
    _, excess2 = errors(off, ref, "bf16", rms)
    assert excess2 > 0.0
    assert TOL["bf16"] == 2e-2 and TOL["f32"] == 1e-5
