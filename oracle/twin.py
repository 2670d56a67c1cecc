"""Second, independently written fp64 implementation of exact attention (numpy).  TEST ONLY.

Whole-matrix expressions of the same definition that ``oracle.c`` writes out row by row
(FlashAttention (DE), "Problematik der Standard-Attention": softmax(Q K^T / sqrt(d_k)) V),
plus the ordinary derivative for the backward pass.  It exists so that the pin tests can
compare two implementations that were written separately; tiny shapes only (it forms N x N).
"""
from __future__ import annotations

import numpy as np


def visible_mask(N: int, causal: bool, L: int) -> np.ndarray:
    """Boolean [N, N]: key j is visible to query i (j < L, and j <= i when causal)."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    m = j < L
    if causal:
        m = m & (j <= i)
    return m


def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, causal: bool, L=None):
    """One head -> (O, lse, P), all fp64."""
    N = q.shape[0]
    L = N if L is None else L
    vis = visible_mask(N, causal, L)
    S = scale * (q @ k.T)
    S = np.where(vis, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe)
    l = E.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(l > 0, E / np.where(l > 0, l, 1.0), 0.0)
        lse = np.where(l[:, 0] > 0, m_safe[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)), -np.inf)
    return P @ v, lse, P


def backward(q, k, v, do, scale: float, causal: bool, L=None):
    """One head -> dict(dq, dk, dv, o, lse)."""
    O, lse, P = forward(q, k, v, scale, causal, L)
    dP = do @ v.T
    D = (do * O).sum(axis=1, keepdims=True)
    dS = P * (dP - D)
    return {"dq": scale * dS @ k, "dk": scale * dS.T @ q, "dv": P.T @ do, "o": O, "lse": lse}
