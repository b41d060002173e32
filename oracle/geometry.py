"""Radial candidate block set (DynamicRad, Sec. 3.1, Eqs. 1-7; Algorithm 1, candidate
construction and block aggregation).

Test infrastructure only (see the package docstring).

Readings where the paper is silent or loose:

* Blocks are contiguous runs of ``block`` tokens over the flattened (frame, h, w)
  order; the sequence tail is padded (Sec. 3.1 "Notation").  A block may straddle
  two or more frames: its tokens keep their own frame and in-frame index.
* ``u`` and ``v`` are the flattened in-frame indices h * W + w, and the spatial
  distance is |u - v| exactly as Eq. 7 writes it.
* The rounding bracket of Eq. 3 is round-half-up, floor(x + 0.5).
* Eq. 5's epsilon is a parameter (default 1e-6).
* t = 0 pairs are always retained with w = N_t (Eq. 3 and Algorithm 1, intra-frame case);
  Eq. 6's split rule applies to t >= 1.
* "Density control": a key token (column) of block J is active for query block I
  when the number of tokens of I linked to it exceeds theta_c * n_I; J is a
  candidate when its active columns exceed theta_m * n_J (strict inequalities,
  n counts valid tokens).  With theta_c = theta_m = 0 this is "some token pair
  of (I, J) lies in P".
* The always-kept (forced) set F_I: blocks holding a token whose frame is within
  ``force_t`` (0 or 1) of a frame of I, over frame pairs the split rule retains.
  These are the pairs Eq. 8 gives rho = 1 and Eq. 11 gives tau = -inf.  The
  candidate set of row I is the aggregated set united with F_I.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------- Eq. 1 -----
def log_group(t: int) -> int:
    """B(t) = floor(log2 t) + 1 for t >= 1 (Eq. 1), evaluated exactly: the bit length of t."""
    if t < 1:
        raise ValueError("B(t) is defined for t >= 1")
    return int(t).bit_length()


def base_span(tokens_per_frame: int) -> int:
    """L0 = 2^ceil(log2 N_t) (Eq. 1): the smallest power of two >= N_t."""
    if tokens_per_frame < 1:
        raise ValueError("N_t must be positive")
    return 1 << (tokens_per_frame - 1).bit_length()


# ---------------------------------------------------------------- Eq. 2-3 ---
def decay_length(t: int, l0: int, gamma: float) -> float:
    """L(t) = L0 / 2^B(t) * gamma (Eq. 2).  The power-of-two division is exact."""
    return (l0 / 2.0 ** log_group(t)) * gamma


def window(t: int, tokens_per_frame: int, l0: int, block: int, gamma: float) -> int:
    """w(i, j) of Eq. 3: N_t for t <= 1, else max(B_s, round(L(t)))."""
    if t <= 1:
        return tokens_per_frame
    return max(block, math.floor(decay_length(t, l0, gamma) + 0.5))


# ---------------------------------------------------------------- Eq. 4-6 ---
def split_length(t: int, l0: int, lam: float) -> float:
    """L_split(t) = L0 / 2^B(t) * lambda (Eq. 4)."""
    return (l0 / 2.0 ** log_group(t)) * lam


def split_factor(t: int, l0: int, block: int, lam: float, eps: float) -> int:
    """sf(t) = max(1, floor(B_s / (L_split(t) + eps))) (Eq. 5)."""
    return max(1, math.floor(block / (split_length(t, l0, lam) + eps)))


def frame_pair_retained(t: int, l0: int, block: int, lam: float, eps: float) -> bool:
    """Eq. 6: a pair at distance t >= 1 survives iff t mod sf(t) = 0; t = 0 always does."""
    if t == 0:
        return True
    return t % split_factor(t, l0, block, lam, eps) == 0


def frame_tables(geom):
    """Per temporal distance t in [0, F-1]: (w(t), retained(t)) as numpy arrays."""
    nt = geom.height * geom.width
    l0 = base_span(nt)
    w = np.array([window(t, nt, l0, geom.block, geom.gamma) for t in range(geom.frames)],
                 dtype=np.int64)
    r = np.array([frame_pair_retained(t, l0, geom.block, geom.lam, geom.eps)
                  for t in range(geom.frames)], dtype=bool)
    return w, r


# ---------------------------------------------------------------- Eq. 7 -----
def token_pair_allowed(geom, q: int, k: int) -> bool:
    """(q, k) in P(frame(q), frame(k)) of Eq. 7, with the split rule of Eq. 6."""
    nt = geom.height * geom.width
    l0 = base_span(nt)
    i, u = divmod(q, nt)
    j, v = divmod(k, nt)
    t = abs(i - j)
    if not frame_pair_retained(t, l0, geom.block, geom.lam, geom.eps):
        return False
    return abs(u - v) <= window(t, nt, l0, geom.block, geom.gamma)


def _block_tokens(geom, blk: int) -> np.ndarray:
    n = geom.frames * geom.height * geom.width
    return np.arange(blk * geom.block, min((blk + 1) * geom.block, n), dtype=np.int64)


def candidate_row(geom, row: int):
    """Candidate blocks of query block ``row`` and its forced subset.

    Returns (cand, forced): sorted int64 arrays of block indices, forced a subset
    of cand.  Token-level evaluation of Eq. 7 for every (query token of the
    block, key token), then the (theta_c, theta_m) aggregation."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    nb = -(-n // geom.block)
    w_t, r_t = frame_tables(geom)
    q = _block_tokens(geom, row)
    qi, qu = q // nt, q % nt
    keys = np.arange(n, dtype=np.int64)
    kj, kv = keys // nt, keys % nt
    tt = np.abs(qi[:, None] - kj[None, :])
    allowed = r_t[tt] & (np.abs(qu[:, None] - kv[None, :]) <= w_t[tt])
    col_count = allowed.sum(axis=0)                      # linked queries per key token
    active = col_count > geom.theta_c * len(q)           # column activity
    blk_of_key = keys // geom.block
    n_active = np.bincount(blk_of_key, weights=active, minlength=nb)
    n_valid = np.bincount(blk_of_key, minlength=nb)
    aggregated = n_active > geom.theta_m * n_valid
    # forced: key tokens whose frame is within force_t of a frame of the row,
    # over retained frame pairs
    near = (tt <= geom.force_t) & r_t[tt]
    forced_tok = near.any(axis=0)
    forced = np.bincount(blk_of_key, weights=forced_tok, minlength=nb) > 0
    cand = aggregated | forced
    return np.flatnonzero(cand), np.flatnonzero(forced)


def candidate_csr(geom, rows=None):
    """Candidate CSR over all (or the given) rows.

    Returns dict with row_ptr (int64 [R+1]), col (int64), forced_lo, forced_hi
    (int64 [R]) -- the forced set of a row is the contiguous range
    [forced_lo, forced_hi] (asserted)."""
    nb = geom.n_blocks
    rows = range(nb) if rows is None else rows
    ptr, cols, flo, fhi = [0], [], [], []
    for r in rows:
        c, f = candidate_row(geom, r)
        if len(f) == 0 or f[-1] - f[0] + 1 != len(f):
            raise AssertionError("forced set is not a contiguous block range")
        cols.append(c)
        ptr.append(ptr[-1] + len(c))
        flo.append(int(f[0]))
        fhi.append(int(f[-1]))
    return {
        "row_ptr": np.array(ptr, dtype=np.int64),
        "col": np.concatenate(cols) if cols else np.zeros(0, np.int64),
        "forced_lo": np.array(flo, dtype=np.int64),
        "forced_hi": np.array(fhi, dtype=np.int64),
    }
