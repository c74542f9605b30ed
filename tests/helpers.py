"""Shared test helpers: moving seeded inputs to the GPU and comparing results."""
from __future__ import annotations

import numpy as np
import torch

ATTN_MAX_ABS = 2e-2     # attention outputs, h and y: max-abs error
ATTN_MEAN_ABS = 2e-3    # and mean-abs error
W_TOL = 1e-5            # router probabilities and renormalised weights
NEAR_TIE = 1e-4         # logit margin below which both TopK choices are correct


def bf16_dev(u16: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch bf16 tensor on the device."""
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_attn(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def assert_close_proj(got, ref, what=""):
    """bf16-rounded projection: |err| <= 2^-8 |ref| + 1e-3."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.abs(got - ref) > (2.0 ** -8) * np.abs(ref) + 1e-3
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, worst {np.abs(got - ref).max():.3e}"


BF16_U = 2.0 ** -8      # relative half-ulp of bf16 (8 significant bits)
GRAD_MEAN_REL = 2e-3    # gradients: mean-abs error <= 2e-3 rms(ref)


def assert_close_grad(got, ref, bound, what="", floor=1e-6):
    """Gradients computed with bf16 MMA operands and fp32 accumulation, stored
    as bf16.  Per element |err| <= 2^-8 |ref| + bound + floor, where ``bound``
    is the worst-case error of the arithmetic before the final rounding (the
    oracle's *_error_bound functions) and 2^-8 |ref| that rounding; on top,
    mean-abs <= 2e-3 rms(ref)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = np.asarray(bound, dtype=np.float64)
    assert got.shape == ref.shape == bound.shape, (what, got.shape, ref.shape, bound.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = BF16_U * np.abs(ref) + bound + floor
    worst = float((err / tol).max())
    s = max(float(np.sqrt(np.mean(ref * ref))), 1e-3)
    mean = float(err.mean()) / s
    assert worst <= 1.0 and mean <= GRAD_MEAN_REL, f"{what}: worst err/bound {worst:.3f}, mean-abs/rms {mean:.3e}"
    return worst, mean
