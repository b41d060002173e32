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


def _block_tokens(block: int, n: int, blocks) -> np.ndarray:
    parts = [np.arange(b * block, min((b + 1) * block, n), dtype=np.int64) for b in blocks]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def query_block_backward(q, k, v, do, block: int, kept, i: int, scale=None):
    """The same gradients restricted to the query tokens of block i, whose kept
    key blocks are `kept` (for sampled checks at sizes where the [N, N] mask
    does not fit).  Returns (rows, keys, p, ds, dq_rows): the query and key
    token indices, P and dS over [rows, keys], and dQ of the rows."""
    n, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rows = np.arange(i * block, min((i + 1) * block, n), dtype=np.int64)
    keys = _block_tokens(block, n, kept)
    if len(keys) == 0:
        z = np.zeros((len(rows), 0))
        return rows, keys, z, z, np.zeros((len(rows), d))
    p = masked_softmax(scale * (q[rows] @ k[keys].T), np.ones((len(rows), len(keys)), dtype=bool))
    dp = do[rows] @ v[keys].T
    ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
    return rows, keys, p, ds, scale * (ds @ k[keys])


def key_block_backward(q, k, v, do, block: int, row_ptr, col, j: int, scale=None):
    """dK, dV of the key tokens of block j: the sum over every query block that
    keeps j of that block's P^T dO and scale dS^T Q on j's keys, each query
    row normalised over its own kept keys.  Returns (keys_j, dk_j, dv_j)."""
    n, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    keys_j = _block_tokens(block, n, [j])
    dk = np.zeros((len(keys_j), d))
    dv = np.zeros((len(keys_j), d))
    nb = -(-n // block)
    for i in range(nb):
        kept = np.asarray(col[int(row_ptr[i]):int(row_ptr[i + 1])], dtype=np.int64)
        if not np.any(kept == j):
            continue
        rows, keys, p, ds, _ = query_block_backward(q, k, v, do, block, kept, i, scale)
        sel = np.searchsorted(keys, keys_j)
        dv += p[:, sel].T @ do[rows]
        dk += scale * (ds[:, sel].T @ q[rows])
    return keys_j, dk, dv
