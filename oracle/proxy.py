"""Objective of the offline parameter search (DynamicRad, Appendix C.2-C.4,
Eq. 22) on the feature-drift proxy (Eq. 20).

Test infrastructure only (see the package docstring).

* The proxy attention is A_ij proportional to exp(h_i . h_j / sqrt(D)) (Q = K =
  the drifting features), row-normalized: the dense softmax matrix.
* A_sparse(x) is the softmax restricted to the blocks the mask keeps (the
  candidate set of Sec. 3.1 for x = (gamma, lambda, theta_m, theta_c)), zero
  elsewhere.
* L(x) = ||A_dense - A_sparse||_F^2 / ||A_dense||_F^2 + alpha * ReLU(tau_s - S),
  S the fraction of (query block, key block) pairs the mask drops, tau_s = 0.8,
  alpha = 10 (Eq. 22).
Computed here from the dense matrices in float64.
"""
from __future__ import annotations

import math

import numpy as np


def dense_attention_matrix(h: np.ndarray) -> np.ndarray:
    """Row-softmax of h h^T / sqrt(D), float64 [N, N]."""
    s = (h @ h.T) / math.sqrt(h.shape[1])
    s -= s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def sparse_attention_matrix(h: np.ndarray, block: int, row_ptr, col) -> np.ndarray:
    """Softmax restricted to the kept blocks (token mask from the block CSR)."""
    n, d = h.shape
    nb = -(-n // block)
    keep = np.zeros((nb, nb), dtype=bool)
    for r in range(nb):
        keep[r, col[row_ptr[r]:row_ptr[r + 1]]] = True
    tok = np.repeat(np.repeat(keep, block, axis=0), block, axis=1)[:n, :n]
    s = (h @ h.T) / math.sqrt(d)
    s = np.where(tok, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(tok, np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
    z = e.sum(axis=1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def block_sparsity(n_blocks: int, kept_blocks: int) -> float:
    """S(x): the fraction of the n_blocks^2 block pairs the mask drops."""
    return 1.0 - kept_blocks / float(n_blocks * n_blocks)


def objective(h: np.ndarray, block: int, row_ptr, col, tau_s: float = 0.8, alpha: float = 10.0):
    """(L, normalized MSE, sparsity) of Eq. 22."""
    a = dense_attention_matrix(h)
    b = sparse_attention_matrix(h, block, row_ptr, col)
    nmse = float(((a - b) ** 2).sum() / (a ** 2).sum())
    nb = -(-h.shape[0] // block)
    s = block_sparsity(nb, int(row_ptr[-1]))
    return nmse + alpha * max(0.0, tau_s - s), nmse, s
