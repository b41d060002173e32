"""Block pooling, block proxy scores and the two selection modes.

Test infrastructure only (see the package docstring).

DynamicRad (arXiv 2604.20470) Sec. 3.2 and Algorithm 1 select, inside the
candidate set of each query block, either a fixed fraction (static-ratio) or the
pairs whose score clears a threshold (dynamic-threshold).  This oracle follows
the block-pooled form of those two modes:

* block proxy score s_IJ = qbar_I . kbar_J / sqrt(d), with qbar, kbar the means
  of Q and K over the valid tokens of each block (the scale of Eq. 9, one head);
* static-ratio: keep the forced set F_I and the top k of the other candidates
  N_I = C_I minus F_I by (score descending, block index ascending), with
  k = max(1, floor(rho * |N_I|)) as in Eq. 8 (0 when N_I is empty); the floor
  is taken of rho * n + 1e-9 so that products such as 0.15 * 20 that are
  mathematically integral do not round down;
* dynamic-threshold: p_J = softmax over C_I of s_IJ (float64); keep F_I and the
  shortest prefix of N_I in the same order whose mass, added to the forced
  mass, reaches tau.  tau >= 1 keeps all of C_I.

Forced blocks cover frame distance t <= 1, where Eq. 8 sets rho = 1 and Eq. 11
sets tau = -inf; they always contain the diagonal block, so the "keep the top
pair if nothing passes" fallback of Sec. 3.2 never has to fire.
"""
from __future__ import annotations

import math

import numpy as np


def block_means(x: np.ndarray, block: int) -> np.ndarray:
    """Mean over the valid tokens of each block: x [N, D] -> [ceil(N / block), D] (float64)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    nb = -(-n // block)
    out = np.empty((nb, x.shape[1]), dtype=np.float64)
    for b in range(nb):
        seg = x[b * block:min((b + 1) * block, n)]
        out[b] = seg.sum(axis=0) / seg.shape[0]
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray, row: int, cols, scale=None) -> np.ndarray:
    """s_IJ = qbar_I . kbar_J * scale for J in cols; scale defaults to 1/sqrt(d)."""
    d = qbar.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    cols = np.asarray(cols, dtype=np.int64)
    return (kbar[cols] @ qbar[row]) * scale


def static_k(rho: float, n: int) -> int:
    """k = max(1, floor(rho * n)) of Eq. 8 for n > 0 candidates, 0 for none."""
    if n == 0:
        return 0
    return max(1, math.floor(rho * n + 1e-9))


def rank_order(cols, scores) -> list:
    """Positions of cols sorted by (score descending, block index ascending).

    Scores compare as numbers, so -0.0 and +0.0 tie and the lower index wins."""
    return sorted(range(len(cols)), key=lambda i: (-float(scores[i]), int(cols[i])))


def select_static(cols, scores, forced_lo: int, forced_hi: int, rho: float) -> np.ndarray:
    """Kept blocks of one row in static-ratio mode, ascending."""
    cols = np.asarray(cols, dtype=np.int64)
    is_forced = (cols >= forced_lo) & (cols <= forced_hi)
    free = np.flatnonzero(~is_forced)
    k = static_k(rho, len(free))
    order = rank_order(cols[free], np.asarray(scores)[free])
    keep = set(cols[is_forced].tolist()) | {int(cols[free[i]]) for i in order[:k]}
    return np.array(sorted(keep), dtype=np.int64)


def softmax_mass(scores) -> tuple:
    """(e, Z): e_J = exp(s_J - max s) in float64 and Z = sum of e (exactly rounded sum)."""
    s = np.asarray(scores, dtype=np.float64)
    e = np.exp(s - s.max())
    return e, math.fsum(e.tolist())


def dynamic_cut(cols, scores, forced_lo: int, forced_hi: int, tau: float):
    """Dynamic-threshold selection of one row.

    Returns (kept ascending, info) where info holds the forced mass, Z, the
    prefix masses at the cut and one step before it (for ambiguity checks)."""
    cols = np.asarray(cols, dtype=np.int64)
    if tau >= 1.0:
        return cols.copy(), {"ambiguous_gap": math.inf}
    is_forced = (cols >= forced_lo) & (cols <= forced_hi)
    e, z = softmax_mass(scores)
    m_f = math.fsum(e[is_forced].tolist())
    free = np.flatnonzero(~is_forced)
    order = rank_order(cols[free], np.asarray(scores)[free])
    target = tau * z
    taken = []
    gaps = [abs(m_f - target)]
    while True:
        mass = math.fsum([m_f] + [e[free[i]] for i in taken])
        gaps.append(abs(mass - target))
        if mass >= target or len(taken) == len(order):
            break
        taken.append(order[len(taken)])
    keep = set(cols[is_forced].tolist()) | {int(cols[free[i]]) for i in taken}
    # distance of the decision from the threshold, relative to Z, at the
    # cut and one step before it
    info = {"forced_mass": m_f, "z": z, "n_taken": len(taken),
            "ambiguous_gap": min(gaps[-2:]) / z}
    return np.array(sorted(keep), dtype=np.int64), info


def select_dynamic(cols, scores, forced_lo: int, forced_hi: int, tau: float) -> np.ndarray:
    """Kept blocks of one row in dynamic-threshold mode, ascending."""
    return dynamic_cut(cols, scores, forced_lo, forced_hi, tau)[0]


def kept_mass(cols, scores, kept) -> float:
    """Softmax block mass (over the row's candidates) of the kept subset."""
    cols = np.asarray(cols, dtype=np.int64)
    e, z = softmax_mass(scores)
    sel = np.isin(cols, np.asarray(kept, dtype=np.int64))
    return math.fsum(e[sel].tolist()) / z


def select_row(mode: str, cols, scores, forced_lo, forced_hi, value):
    if mode == "static":
        return select_static(cols, scores, forced_lo, forced_hi, value)
    if mode == "dynamic":
        return select_dynamic(cols, scores, forced_lo, forced_hi, value)
    raise ValueError(mode)


def select_head(q: np.ndarray, k: np.ndarray, block: int, cand: dict, mode: str,
                value: float, rows=None, scores_override=None):
    """Selection for one (batch, head) slice: q, k float64 [N, D].

    cand is the candidate CSR (row_ptr, col, forced_lo, forced_hi) over all
    rows.  scores_override, if given, is the flat float32 score array in
    candidate order (e.g. scores exported by another implementation); the
    selection is then made from those exact values.

    Returns (kept CSR as dict(row_ptr, col) over the given rows, scores per row)."""
    qbar = block_means(q, block)
    kbar = block_means(k, block)
    nb = qbar.shape[0]
    rows = range(nb) if rows is None else rows
    ptr, out, all_scores = [0], [], {}
    for r in rows:
        a, b = int(cand["row_ptr"][r]), int(cand["row_ptr"][r + 1])
        cols = cand["col"][a:b]
        if scores_override is None:
            s = block_scores(qbar, kbar, r, cols)
        else:
            s = np.asarray(scores_override[a:b], dtype=np.float64)
        kept = select_row(mode, cols, s, int(cand["forced_lo"][r]), int(cand["forced_hi"][r]), value)
        out.append(kept)
        ptr.append(ptr[-1] + len(kept))
        all_scores[r] = s
    return {"row_ptr": np.array(ptr, dtype=np.int64),
            "col": np.concatenate(out) if out else np.zeros(0, np.int64)}, all_scores
