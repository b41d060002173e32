"""Block-masked softmax attention (DynamicRad, Sec. 3.3, Eqs. 12-13).

Test infrastructure only (see the package docstring).

Eq. 13 computes Softmax(A + log(M~ + eps)) V with A = Q K^T / sqrt(d_k) (Eq. 12)
and M~ the block mask broadcast to tokens.  The block-sparse kernel skips the
masked blocks outright, which is Eq. 13 in the limit eps -> 0: every query row
takes a plain softmax over the keys of its kept blocks.  Padded key positions
(beyond the sequence) are never keys; padded query rows have no output.

``sparse_attention_rows`` is that limit written out per query block;
``eq13_dense`` evaluates Eq. 13 literally with a finite eps on small inputs, and
the tests show the two agree as eps shrinks.
"""
from __future__ import annotations

import math

import numpy as np


def block_key_tokens(block: int, n: int, kept_blocks) -> np.ndarray:
    """Valid key token indices covered by the kept blocks (ascending blocks)."""
    parts = [np.arange(j * block, min((j + 1) * block, n), dtype=np.int64) for j in kept_blocks]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def attend_block(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, keys: np.ndarray,
                 scale: float):
    """Softmax attention of the given query rows over the given key tokens (float64).

    Returns (o [r, D], lse [r]) with lse the natural log of sum exp(logit)."""
    if len(keys) == 0:
        return (np.zeros((q_rows.shape[0], v.shape[1])),
                np.full(q_rows.shape[0], -math.inf))
    a = (q_rows @ k[keys].T) * scale                 # Eq. 12 restricted to the kept keys
    m = a.max(axis=1, keepdims=True)
    p = np.exp(a - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v[keys]) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def sparse_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int,
                          row_ptr, col, rows=None, scale=None, token_rows=None):
    """Eq. 13 with eps -> 0 for one (batch, head) slice.

    q, k, v: float64 [N, D].  (row_ptr, col): kept-block CSR over all query
    blocks.  rows: query blocks to evaluate (default all).  token_rows: optional
    dict block -> array of in-block row offsets to evaluate (sampling).

    Returns dict block -> (token indices, o, lse)."""
    n, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nb = -(-n // block)
    rows = range(nb) if rows is None else rows
    out = {}
    for r in rows:
        kept = col[int(row_ptr[r]):int(row_ptr[r + 1])]
        keys = block_key_tokens(block, n, kept)
        toks = np.arange(r * block, min((r + 1) * block, n), dtype=np.int64)
        if token_rows is not None and r in token_rows:
            toks = toks[np.asarray(token_rows[r], dtype=np.int64)]
        o, lse = attend_block(q[toks], k, v, keys, scale)
        out[r] = (toks, o, lse)
    return out


def sparse_attention(q, k, v, block, row_ptr, col, scale=None):
    """Full [N, D] output and [N] LSE of one slice (small inputs)."""
    n, d = q.shape
    o = np.zeros((n, d))
    lse = np.zeros(n)
    for _, (toks, ob, lb) in sparse_attention_rows(q, k, v, block, row_ptr, col, scale=scale).items():
        o[toks] = ob
        lse[toks] = lb
    return o, lse


def token_mask(block: int, n: int, row_ptr, col) -> np.ndarray:
    """M~ of Eq. 13: the block mask broadcast to a boolean [N, N] token mask."""
    nb = -(-n // block)
    m = np.zeros((n, n), dtype=bool)
    for r in range(nb):
        q0, q1 = r * block, min((r + 1) * block, n)
        for j in col[int(row_ptr[r]):int(row_ptr[r + 1])]:
            m[q0:q1, j * block:min((j + 1) * block, n)] = True
    return m


def eq13_dense(q, k, v, mask: np.ndarray, eps: float, scale=None):
    """Eq. 13 evaluated literally: Softmax(A + log(M~ + eps)) V, float64, dense."""
    n, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    a = (q @ k.T) * scale + np.log(mask.astype(np.float64) + eps)
    m = a.max(axis=1, keepdims=True)
    p = np.exp(a - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v) / l, (m + np.log(l))[:, 0]
