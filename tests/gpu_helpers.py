"""Shared helpers for the GPU parity tests: tolerances and comparison against the oracle.

Tolerances (bf16 inputs, fp32 accumulation, compared with the fp64 oracle):
  forward   max|O - O_ref| <= 2e-2, mean|O - O_ref| <= 2e-3, max|lse - lse_ref| <= 1e-3
  backward  max|X - X_ref| <= 5e-2 * max|X_ref| for X in dQ, dK, dV
"""
import numpy as np
import torch

O_MAX = 2e-2
O_MEAN = 2e-3
LSE_MAX = 1e-3
GRAD_REL = 5e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_fwd_close(O, lse, O_ref, lse_ref, what=""):
    O, lse = np.asarray(O, np.float64), np.asarray(lse, np.float64)
    err = np.abs(O - O_ref)
    assert np.isfinite(O).all(), f"{what}: non-finite O"
    assert err.max() <= O_MAX, f"{what}: max|O-O_ref| = {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: mean|O-O_ref| = {err.mean():.3e}"
    lerr = np.abs(lse - lse_ref)
    assert lerr.max() <= LSE_MAX, f"{what}: max|lse-lse_ref| = {lerr.max():.3e}"
    return err.max(), err.mean(), lerr.max()


def assert_grad_close(X, X_ref, name, what=""):
    X = np.asarray(X, np.float64)
    assert np.isfinite(X).all(), f"{what}: non-finite {name}"
    ref = max(np.abs(X_ref).max(), 1e-30)
    err = np.abs(X - X_ref).max()
    assert err <= GRAD_REL * ref, f"{what}: max|{name}-ref| = {err:.3e} > {GRAD_REL} * {ref:.3e}"
    return err / ref
