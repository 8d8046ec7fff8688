"""Shared test helpers: error metrics and the tolerances the GPU path must meet.

Tolerances (fixed by the target of this library, stated once here):
  forward O      max |err| <= 1e-2 and relative RMS <= 5e-3
  LSE            max |err| <= 1e-4
  dQ, dK, dV     relative RMS <= 1e-2
  FP8 forward O  relative RMS <= 5e-2 (vs the fp64 oracle on unquantised inputs)
relative RMS = sqrt(mean((x - ref)^2)) / sqrt(mean(ref^2)); for gradients the
denominator is floored at 1e-3 (absolute), because some exact gradients are
identically zero (N = 1: P = 1, so dS = 0 and dQ = dK = 0) and a relative
error against zero is undefined.
"""
import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-4
GRAD_REL_RMS = 1e-2
FP8_REL_RMS = 5e-2


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_rms(x, ref, floor: float = 1e-300) -> float:
    x, ref = f64(x), f64(ref)
    den = np.sqrt(np.mean(ref ** 2))
    return float(np.sqrt(np.mean((x - ref) ** 2)) / max(den, floor))


GRAD_RMS_FLOOR = 1e-3


def max_abs(x, ref) -> float:
    return float(np.max(np.abs(f64(x) - f64(ref)))) if np.size(ref) else 0.0


def max_scaled_err(o, o_ref) -> float:
    """max |err| / max(1, |ref|) elementwise: the forward bound for masks
    (sliding window, ALiBi) that average few keys per row, where |O| grows
    past 1 and one bf16 half-ulp of O alone approaches 1e-2 (the same
    reading as the large-magnitude forward test)."""
    o, o_ref = f64(o), f64(o_ref)
    return float(np.max(np.abs(o - o_ref) / np.maximum(1.0, np.abs(o_ref)))) if o_ref.size else 0.0


def assert_fwd_close(o, lse, o_ref, lse_ref, tag=""):
    o, lse = f64(o), f64(lse)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), f"{tag}: non-finite output"
    ea, er, el = max_abs(o, o_ref), rel_rms(o, o_ref), max_abs(lse, lse_ref)
    assert ea <= O_MAX_ABS and er <= O_REL_RMS and el <= LSE_MAX_ABS, (
        f"{tag}: O max abs {ea:.3e} (<= {O_MAX_ABS}), O rel RMS {er:.3e} (<= {O_REL_RMS}), "
        f"LSE max abs {el:.3e} (<= {LSE_MAX_ABS})")
    return ea, er, el
