"""Shared helpers for the GPU parity tests: tolerances and comparisons of
the CUDA path against the fp64 oracle.

Tolerances (outputs from bf16 inputs with fp32 accumulation against the fp64
oracle run on the same bf16 values):
  O:   max |dO| <= 2e-2 and mean |dO| <= 2e-3;
  LSE: |dLSE| <= 1e-3 * max(1, |LSE|);
  RoPE: at most 1 bf16 ulp from the fp64 rotation rounded to nearest even;
  cutoff tables and tile classes: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_REL = 1e-3


def widen(t: torch.Tensor) -> np.ndarray:
    """bf16/fp32 tensor (any device) -> fp64 numpy (exact)."""
    return t.detach().to("cpu").double().numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns."""
    a = a_bits.astype(np.int64)
    b = b_bits.astype(np.int64)
    # map sign-magnitude to a monotone integer line
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)


def assert_attention_close(o_gpu, lse_gpu, o_ref, lse_ref, tag: str = ""):
    o = widen(o_gpu).reshape(o_ref.shape)
    err = np.abs(o - o_ref)
    assert np.all(np.isfinite(o)), f"{tag}: non-finite output"
    assert err.max() <= O_MAX_ABS, f"{tag}: max |dO| {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{tag}: mean |dO| {err.mean():.3e}"
    if lse_gpu is not None and lse_ref is not None:
        lse = widen(lse_gpu).reshape(lse_ref.shape)
        tol = LSE_REL * np.maximum(1.0, np.abs(lse_ref))
        bad = np.abs(lse - lse_ref) > tol
        assert not bad.any(), f"{tag}: LSE off at {np.argwhere(bad)[:5].tolist()} " \
                              f"max {np.abs(lse - lse_ref).max():.3e}"
    return float(err.max()), float(err.mean())


# Gradients (wp_prefill_backward) against the fp64 oracle's: the kernel rounds
# P and dS to bf16 (relative rounding 2^-9) before the dV, dQ and dK products
# and takes D from the forward's bf16 O, so each entry carries a relative error
# of a few 2^-9 of the terms it sums. The bounds are relative to the size of
# the reference gradient, max |dG| <= 2e-2 max |G| + 1e-4 and
# mean |dG| <= 1e-2 mean |G| + 1e-5; the small absolute terms cover gradients
# that are exactly 0 (one key: dS = dP - D = 0), where the kernel leaves the
# fp32 rounding of dP - D.
GRAD_MAX_REL = 2e-2
GRAD_MEAN_REL = 1e-2
GRAD_MAX_ABS = 1e-4
GRAD_MEAN_ABS = 1e-5


def assert_grad_close(g_gpu, g_ref, tag: str = "", mean_rel: float = GRAD_MEAN_REL):
    g = widen(g_gpu).reshape(g_ref.shape)
    err = np.abs(g - g_ref)
    assert np.all(np.isfinite(g)), f"{tag}: non-finite gradient"
    ref_max, ref_mean = float(np.abs(g_ref).max()), float(np.abs(g_ref).mean())
    assert err.max() <= GRAD_MAX_REL * ref_max + GRAD_MAX_ABS, \
        f"{tag}: max |dG| {err.max():.3e} vs max |G| {ref_max:.3e}"
    assert err.mean() <= mean_rel * ref_mean + GRAD_MEAN_ABS, \
        f"{tag}: mean |dG| {err.mean():.3e} vs mean |G| {ref_mean:.3e}"
    print(f"{tag}: max |dG|/max |G| {err.max() / max(ref_max, 1e-30):.2e}, "
          f"mean |dG|/mean |G| {err.mean() / max(ref_mean, 1e-30):.2e}")
    return float(err.max() / max(ref_max, 1e-30)), float(err.mean() / max(ref_mean, 1e-30))
