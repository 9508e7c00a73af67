"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (written here, applied element by element over every output):
  float32:        max |gpu - ref| <= 1e-5 * max |ref|
  float16/bf16:   max |gpu - ref| <= 1e-2 * max |ref|
The reference `ref` is the float64 oracle on the same dtype-rounded inputs.

A second, tighter check catches small systematic errors that the 16-bit
tolerance would let through: every 16-bit output must equal the reference
rounded to the dtype, or be its neighbour (float32 accumulation can land on
the other side of a rounding boundary); at most 1% of outputs may be
neighbours.  Outputs below 1e-2 * max |ref| (cancellation) are left to the
absolute bound.  For float32 outputs the elementwise bound above already is
tight.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}


def _ordered(bits16):
    """Map 16-bit float bit patterns to integers that preserve order."""
    b = bits16.to(torch.int32) & 0xFFFF
    neg = b >= 0x8000
    return torch.where(neg, -(b & 0x7FFF), b)


def compare(gpu, ref, label=""):
    """Assert parity of a GPU output tensor with a float64 oracle array."""
    got = gpu.detach().cpu()
    ref_t = torch.from_numpy(np.ascontiguousarray(ref))
    assert tuple(got.shape) == tuple(ref_t.shape), f"{label}: shape {got.shape} vs {ref_t.shape}"
    assert torch.isfinite(got).all(), f"{label}: non-finite outputs"
    scale = float(ref_t.abs().max()) if ref_t.numel() else 0.0
    err = (got.double() - ref_t).abs()
    max_err = float(err.max()) if err.numel() else 0.0
    tol = TOL[got.dtype]
    assert max_err <= tol * max(scale, 1e-30), (
        f"{label}: max|gpu-ref| = {max_err:.3e} > {tol:g} * max|ref| ({scale:.3e})")
    stats = {"max_abs_err": max_err, "max_abs_ref": scale,
             "rel": max_err / scale if scale else 0.0}
    if got.dtype in (torch.float16, torch.bfloat16) and got.numel():
        rounded = ref_t.to(got.dtype)
        d = (_ordered(got.view(torch.int16)) - _ordered(rounded.view(torch.int16))).abs()
        # outputs far below the largest one come from cancellation; there the
        # float32 accumulation error can exceed one 16-bit ulp, and the
        # absolute tolerance above is the check
        d = torch.where(ref_t.abs() >= 1e-2 * scale, d, torch.zeros_like(d))
        assert int(d.max()) <= 1, f"{label}: an output is {int(d.max())} ulps from the rounded ref"
        frac = float((d == 1).double().mean())
        assert frac <= 0.01, f"{label}: {frac:.2%} of outputs are one ulp off"
        stats["one_ulp_frac"] = frac
    return stats
