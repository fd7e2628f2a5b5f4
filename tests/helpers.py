"""Shared test helpers: tolerances and comparisons against the fp64 oracle.

Tolerances (stated for the KDA entry points):
  fp32 inputs: max |x - ref| <= 1e-3 on the outputs and on every final state.
  bf16 inputs: ||x - ref||_inf / ||ref||_inf <= 2e-2, tensor-wise, on the
               outputs and on each final state (fp32 state).
"""
import torch

F32_ABS_TOL = 1e-3
BF16_REL_TOL = 2e-2


def max_abs(x, ref) -> float:
    return float((x.double().cpu() - ref.double().cpu()).abs().max())


def rel_inf(x, ref) -> float:
    ref = ref.double().cpu()
    den = float(ref.abs().max())
    num = float((x.double().cpu() - ref).abs().max())
    return num / den if den > 0 else num


def rms_rel(x, ref) -> float:
    ref = ref.double().cpu()
    d = (x.double().cpu() - ref)
    den = float(ref.pow(2).mean().sqrt())
    return float(d.pow(2).mean().sqrt()) / den if den > 0 else float(d.pow(2).mean().sqrt())


def assert_close(x, ref, dtype, what=""):
    """Apply the stated tolerance for the input dtype."""
    assert torch.isfinite(x.double()).all(), f"{what}: non-finite values"
    if dtype == torch.float32:
        e = max_abs(x, ref)
        assert e <= F32_ABS_TOL, f"{what}: max-abs error {e:.3e} > {F32_ABS_TOL}"
        return e
    e = rel_inf(x, ref)
    assert e <= BF16_REL_TOL, f"{what}: relative inf-norm error {e:.3e} > {BF16_REL_TOL}"
    return e
