"""Parity helpers shared by the GPU tests: tolerances and tensor plumbing.

Tolerances (stated for the whole suite):
  * fp32 inputs:  max|gpu - ref| / max|ref| <= 1e-4       (max relative error)
  * bf16 inputs:  max|gpu - ref| / rms(ref) <= 2e-2       (max-abs normalised by the RMS)
The reference is the fp64 CPU oracle evaluated on exactly the values the GPU received.
"""
import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_cuda(d):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in d.items()}


def npf(x):
    if torch.is_tensor(x):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def rel_error(gpu, ref, kind: str) -> float:
    g, r = npf(gpu), npf(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    diff = np.max(np.abs(g - r)) if g.size else 0.0
    if kind == "f32":
        den = np.max(np.abs(r)) if r.size else 1.0
    else:
        den = np.sqrt(np.mean(r * r)) if r.size else 1.0
    return float(diff / max(den, 1e-30))


def assert_parity(gpu, ref, kind: str, name: str = ""):
    e = rel_error(gpu, ref, kind)
    assert e <= TOL[kind], f"{name}: error {e:.3e} > {TOL[kind]:.0e} ({kind})"
    return e


def kind_of(t: torch.Tensor) -> str:
    return "f32" if t.dtype == torch.float32 else "bf16"


def assert_bf16_is_rounding(out_bf16: torch.Tensor, out_f32: torch.Tensor, name: str = ""):
    """A bf16 output must be exactly the round-to-nearest-even of the same call's fp32 output.
    (The parity bound is checked on the fp32 output: a bf16 store alone costs up to 2^-8 of
    the largest entry, which on heavy-tailed outputs exceeds 2e-2 of the RMS by itself.)"""
    assert out_bf16.dtype == torch.bfloat16 and out_f32.dtype == torch.float32
    assert torch.equal(out_bf16, out_f32.to(torch.bfloat16)), f"{name}: bf16 output is not the rounded fp32 output"
