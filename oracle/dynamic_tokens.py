"""Paper-exact dynamic-threshold mode: token-level proxy logits on the
candidate pairs (DynamicRad, Sec. 3.2 "Dynamic-threshold mode", Eqs. 9-11, with
the fused-head proxy of Appendix B, Eq. 19), then the block aggregation of Sec.
3.1.

Test infrastructure only (see the package docstring).

What the mode computes, in the paper's notation:

* for each candidate token pair (u, v) in P(i, j) (Eq. 7), the proxy score
  s(u, v) = (1/H_f) sum_{h < H_f} Q_u^(h) . K_v^(h) / sqrt(d) over the FIRST
  H_f heads (Eq. 9 / Eq. 19, H_f = 2 in the paper);
* per candidate set P(i, j), the z-score s~ = (s - mu_ij) / (sigma_ij + eps)
  (Eq. 10);
* keep the pairs with s~ > tau(i, j), tau = -inf for t <= 1, tau_1 when
  L(t) >= B_s and tau_2 when L(t) < B_s (Eq. 11); if no pair of P(i, j)
  passes, keep the highest-scoring pair (the paper's fallback);
* aggregate the kept token links to blocks with (theta_c, theta_m) and add
  F_I, as for the candidate set (Sec. 3.1); the mask is shared by every head
  (it is computed from the fused heads) and is per batch element.

Readings where the paper leaves a step open:

* sigma is the population standard deviation over P(i, j) (divide by |P|);
  eps = 1e-6.
* "exceeds" is strict: s~ > tau.  With sigma + eps > 0 this is
  s > mu + tau * (sigma + eps), the form both sides evaluate.  The pages
  disagree here: the sentence that introduces Eq. 11 says "exceeds", while
  Algorithm 1's dynamic-threshold step writes s~ >= tau.  The sentence beside
  the equation is taken as the definition and the algorithm as its summary;
  the two readings differ only on pairs whose z-score equals tau exactly,
  which continuous scores hit with probability zero, and the GPU parity test
  (a row between the masks at tau + 1e-3 and tau - 1e-3) accepts either.
* The fallback pair is the one with the largest s; among equal scores the one
  with the smaller in-pair counter u * N_t + v.
* The fallback applies per ordered frame pair (i, j), the unit the threshold
  and the normalization are defined on.
"""
from __future__ import annotations

import math

import numpy as np

from . import geometry as G
from .sampling import aggregate_links, candidate_pairs

EPS_Z = 1e-6


def threshold(geom, t: int, tau1: float, tau2: float) -> float:
    """tau(i, j) of Eq. 11."""
    if t <= 1:
        return -math.inf
    nt = geom.height * geom.width
    return tau1 if G.decay_length(t, G.base_span(nt), geom.gamma) >= geom.block else tau2


def proxy_scores(qf: np.ndarray, kf: np.ndarray, i: int, j: int, u: np.ndarray, v: np.ndarray, nt: int):
    """s(u, v) of Eq. 9 for token pairs of frame pair (i, j).  qf, kf: float64
    [H_f, N, d] (the fused heads).  Returns float64 [len(u)]."""
    hf, _, d = qf.shape
    qs = qf[:, i * nt + u, :]
    ks = kf[:, j * nt + v, :]
    return (qs * ks).sum(axis=2).mean(axis=0) / math.sqrt(d)


def frame_pair_stats(geom, qf, kf, i: int, j: int):
    """(n, mu, sigma, s_max, argmax counter u * N_t + v, s) over P(i, j); n = 0
    when the split rule drops the pair."""
    nt = geom.height * geom.width
    u, v = candidate_pairs(geom, abs(i - j))
    if len(u) == 0:
        return 0, 0.0, 0.0, -math.inf, -1, np.zeros(0)
    s = proxy_scores(qf, kf, i, j, u, v, nt)
    mu = float(s.mean())
    sigma = float(np.sqrt(((s - mu) ** 2).mean()))
    best = int(np.argmax(s))            # first maximum = smallest counter (u, v ascending)
    return len(u), mu, sigma, float(s[best]), int(u[best] * nt + v[best]), s


def kept_pairs(geom, qf, kf, i: int, j: int, tau1: float, tau2: float):
    """Boolean mask over P(i, j) (in candidate_pairs order) of the kept pairs."""
    t = abs(i - j)
    n, mu, sigma, _, _, s = frame_pair_stats(geom, qf, kf, i, j)
    if n == 0:
        return np.zeros(0, dtype=bool)
    tau = threshold(geom, t, tau1, tau2)
    if tau == -math.inf:
        return np.ones(n, dtype=bool)
    keep = (s - mu) / (sigma + EPS_Z) > tau
    if not keep.any():
        keep[int(np.argmax(s))] = True
    return keep


def dynamic_links(geom, qf, kf, tau1: float, tau2: float):
    """Boolean [N, N] token-link matrix of the kept pairs (small geometries)."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    links = np.zeros((n, n), dtype=bool)
    for i in range(geom.frames):
        for j in range(geom.frames):
            u, v = candidate_pairs(geom, abs(i - j))
            if len(u) == 0:
                continue
            keep = kept_pairs(geom, qf, kf, i, j, tau1, tau2)
            links[i * nt + u[keep], j * nt + v[keep]] = True
    return links


def dynamic_mask_csr(geom, qf, kf, tau1: float, tau2: float):
    """The paper-exact dynamic-threshold block mask of one batch element."""
    return aggregate_links(geom, dynamic_links(geom, qf, kf, tau1, tau2))


def frame_pair_logits(qf, kf, i: int, j: int, nt: int):
    """Dense [N_t, N_t] proxy logits of frame pair (i, j) (Eq. 9), float64."""
    hf, _, d = qf.shape
    acc = np.zeros((nt, nt))
    for h in range(hf):
        acc += qf[h, i * nt:(i + 1) * nt] @ kf[h, j * nt:(j + 1) * nt].T
    return acc / hf / math.sqrt(d)


def dynamic_mask_rows(geom, qf, kf, tau1: float, tau2: float, rows, tau_shift: float = 0.0):
    """Mask rows for the given query blocks (large geometries): per frame pair the
    logits over P from a dense product, the z-rule at tau + tau_shift, the
    fallback, then the aggregation restricted to each row's query tokens."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    nb = -(-n // geom.block)
    w_t, r_t = G.frame_tables(geom)
    blk_of_key = np.arange(n, dtype=np.int64) // geom.block
    n_valid = np.bincount(blk_of_key, minlength=nb)
    uu = np.arange(nt)
    cache = {}

    def kept_matrix(i, j):
        if (i, j) in cache:
            return cache[(i, j)]
        t = abs(i - j)
        if not r_t[t]:
            m = np.zeros((nt, nt), dtype=bool)
        else:
            w = w_t[t]
            inb = np.abs(uu[:, None] - uu[None, :]) <= w
            tau = threshold(geom, t, tau1, tau2)
            if tau == -math.inf:
                m = inb
            else:
                s = frame_pair_logits(qf, kf, i, j, nt)
                sv = s[inb]
                mu = float(sv.mean())
                sigma = float(np.sqrt(((sv - mu) ** 2).mean()))
                m = inb & ((s - mu) / (sigma + EPS_Z) > tau + tau_shift)
                if not m.any():
                    flat = np.where(inb, s, -np.inf)
                    best = int(np.argmax(flat))          # first maximum in (u, v) order
                    m = np.zeros((nt, nt), dtype=bool)
                    m.flat[best] = True
        cache[(i, j)] = m
        return m

    out = []
    for row in rows:
        q = np.arange(row * geom.block, min((row + 1) * geom.block, n), dtype=np.int64)
        col_count = np.zeros(n, dtype=np.int64)
        near = np.zeros(n, dtype=bool)
        for qq in q:
            i, u = divmod(int(qq), nt)
            for j in range(geom.frames):
                m = kept_matrix(i, j)
                col_count[j * nt:(j + 1) * nt] += m[u]
                t = abs(i - j)
                if t <= geom.force_t and r_t[t]:
                    near[j * nt:(j + 1) * nt] = True
        active = col_count > geom.theta_c * len(q)
        n_active = np.bincount(blk_of_key, weights=active, minlength=nb)
        agg = n_active > geom.theta_m * n_valid
        forced = np.bincount(blk_of_key, weights=near, minlength=nb) > 0
        out.append(np.flatnonzero(agg | forced))
    return out
