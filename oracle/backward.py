"""Gradients of the block-masked softmax attention (DynamicRad Sec. 3.3,
Eqs. 12-13 with eps -> 0): dQ, dK, dV of a scalar loss given dO.

Test infrastructure only (see the package docstring).

The paper fine-tunes its mask-aware LoRA "under the selected sparse mask"
(Sec. 3.3), which needs the gradient of exactly the attention the forward
computes.  Written out from the definition, per (batch, head), with the token
mask M of the kept blocks:
  S = scale * Q K^T,  P = softmax over the kept keys of each row (0 elsewhere),
  O = P V;
  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dP * P)),
  dQ = scale * dS K,  dK = scale * dS^T Q.
Rows with no kept key have P = 0 and contribute nothing.  float64.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import token_mask


def masked_softmax(s: np.ndarray, mask: np.ndarray) -> np.ndarray:
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(s - m), 0.0)
    z = e.sum(axis=1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def sparse_attention_backward(q, k, v, do, block: int, row_ptr, col, scale=None):
    """(dq, dk, dv, o) for one (batch, head): float64 [N, D] each."""
    n, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    mask = token_mask(block, n, row_ptr, col)
    p = masked_softmax(scale * (q @ k.T), mask)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv, o
