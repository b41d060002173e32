"""Paper-exact static-ratio mode: seeded token-pair sampling per frame pair
(DynamicRad, Sec. 3.2 "Static-ratio mode", Eq. 8), then the block aggregation
of Sec. 3.1 "Density control within blocks".

Test infrastructure only (see the package docstring).

What the mode computes, in the paper's notation:

* for an (ordered) frame pair (i, j) at distance t = |i - j| that the split rule
  retains, the retention ratio rho(i, j) of Eq. 8 is 1 for t <= 1, rho_1 when
  L(t) >= B_s ("near field") and rho_2 when L(t) < B_s ("far field");
* k = max(1, floor(|P(i, j)| * rho(i, j))) token pairs are sampled uniformly
  from the candidate set P(i, j) of Eq. 7 "using a deterministic seed";
* the sampled token links are aggregated to a block mask with (theta_c,
  theta_m) as in Sec. 3.1, and the always-kept near-frame blocks F_I are added
  (the pairs Eq. 8 gives rho = 1; the same union the candidate set takes).

Readings where the paper leaves a step open:

* The uniform k-subset: each token pair (u, v) of frame pair (i, j) gets the
  counter c = ((i * F + j) * N_t + u) * N_t + v and the key SplitMix64(seed)
  output number c + 1, i.e. mix(seed + (c + 1) * 0x9E3779B97F4A7C15 mod 2^64)
  with the SplitMix64 finaliser of Steele, Lea and Flood (OOPSLA 2014).  The
  sample is the k pairs with the smallest keys.  mix is a bijection of 64-bit
  words and the states of distinct counters are distinct, so keys never tie
  and the sample is unique.
* floor(|P| * rho) is taken in float64 with a 1e-9 guard (0.3 * 10 must give
  3), as for the block-pooled static mode.
* The sample is drawn independently for (i, j) and (j, i).
"""
from __future__ import annotations

import numpy as np

from . import geometry as G

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15


# ------------------------------------------------------ SplitMix64 ----------
def splitmix64_mix(z: int) -> int:
    """The SplitMix64 output function on one 64-bit state (Python ints)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64_sequence(seed: int, count: int) -> list:
    """The first ``count`` outputs of the SplitMix64 generator seeded with ``seed``:
    the state advances by the golden gamma before each output."""
    out, s = [], seed & MASK64
    for _ in range(count):
        s = (s + GOLDEN_GAMMA) & MASK64
        out.append(splitmix64_mix(s))
    return out


def splitmix64_mix_np(z: np.ndarray) -> np.ndarray:
    """splitmix64_mix over a uint64 array (numpy's uint64 products wrap mod 2^64)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def pair_keys(seed: int, frames: int, nt: int, i: int, j: int, u: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Keys of token pairs (u, v) of frame pair (i, j) (uint64 arrays)."""
    c = ((np.uint64(i * frames + j) * np.uint64(nt) + u.astype(np.uint64)) * np.uint64(nt)
         + v.astype(np.uint64))
    with np.errstate(over="ignore"):
        state = np.uint64(seed & MASK64) + (c + np.uint64(1)) * np.uint64(GOLDEN_GAMMA)
    return splitmix64_mix_np(state)


# ------------------------------------------------------ Eq. 8 ---------------
def retention_ratio(geom, t: int, rho1: float, rho2: float) -> float:
    """rho(i, j) of Eq. 8."""
    if t <= 1:
        return 1.0
    nt = geom.height * geom.width
    return rho1 if G.decay_length(t, G.base_span(nt), geom.gamma) >= geom.block else rho2


def candidate_pairs(geom, t: int):
    """(u, v) arrays of P(i, j) for a frame pair at distance t (Eq. 7), empty if the
    split rule drops the pair.  Ordered by u, then v."""
    nt = geom.height * geom.width
    l0 = G.base_span(nt)
    if not G.frame_pair_retained(t, l0, geom.block, geom.lam, geom.eps):
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    w = G.window(t, nt, l0, geom.block, geom.gamma)
    u = np.arange(nt, dtype=np.int64)
    lo = np.maximum(u - w, 0)
    hi = np.minimum(u + w, nt - 1)
    cnt = hi - lo + 1
    uu = np.repeat(u, cnt)
    start = np.repeat(lo, cnt)
    off = np.arange(len(uu), dtype=np.int64) - np.repeat(np.cumsum(cnt) - cnt, cnt)
    return uu, start + off


def sample_size(n_pairs: int, rho: float) -> int:
    """k = max(1, floor(|P| * rho)) of Sec. 3.2 (0 for an empty P)."""
    if n_pairs == 0:
        return 0
    return max(1, int(np.floor(n_pairs * rho + 1e-9)))


def frame_pair_threshold(geom, i: int, j: int, rho1: float, rho2: float, seed: int):
    """(k, |P|, T): the sample of frame pair (i, j) is the pairs whose key is <= T,
    T the k-th smallest key (None when nothing is sampled by key: t <= 1 keeps
    all of P, an empty P keeps nothing)."""
    t = abs(i - j)
    u, v = candidate_pairs(geom, t)
    n = len(u)
    rho = retention_ratio(geom, t, rho1, rho2)
    k = sample_size(n, rho)
    if t <= 1 or n == 0:
        return k, n, None
    keys = pair_keys(seed, geom.frames, geom.height * geom.width, i, j, u, v)
    return k, n, int(np.partition(keys, k - 1)[k - 1])


def sampled_links(geom, rho1: float, rho2: float, seed: int, thresholds=None):
    """Boolean [N, N] token-link matrix of the sample (small geometries only)."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    links = np.zeros((n, n), dtype=bool)
    for i in range(geom.frames):
        for j in range(geom.frames):
            t = abs(i - j)
            u, v = candidate_pairs(geom, t)
            if len(u) == 0:
                continue
            if t <= 1:
                keep = np.ones(len(u), dtype=bool)
            else:
                T = (thresholds[(i, j)] if thresholds is not None
                     else frame_pair_threshold(geom, i, j, rho1, rho2, seed)[2])
                keep = pair_keys(seed, geom.frames, nt, i, j, u, v) <= np.uint64(T)
            links[i * nt + u[keep], j * nt + v[keep]] = True
    return links


def aggregate_links(geom, links: np.ndarray):
    """Block CSR from a token-link matrix: the (theta_c, theta_m) aggregation of
    Sec. 3.1 united with the near-frame set F_I (geometry.candidate_row's
    aggregation, applied to the given links)."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    nb = -(-n // geom.block)
    _, r_t = G.frame_tables(geom)
    keys = np.arange(n, dtype=np.int64)
    kj = keys // nt
    blk_of_key = keys // geom.block
    n_valid = np.bincount(blk_of_key, minlength=nb)
    ptr, cols = [0], []
    for row in range(nb):
        q = np.arange(row * geom.block, min((row + 1) * geom.block, n), dtype=np.int64)
        col_count = links[q].sum(axis=0)
        active = col_count > geom.theta_c * len(q)
        n_active = np.bincount(blk_of_key, weights=active, minlength=nb)
        agg = n_active > geom.theta_m * n_valid
        tt = np.abs((q // nt)[:, None] - kj[None, :])
        near = ((tt <= geom.force_t) & r_t[tt]).any(axis=0)
        forced = np.bincount(blk_of_key, weights=near, minlength=nb) > 0
        c = np.flatnonzero(agg | forced)
        cols.append(c)
        ptr.append(ptr[-1] + len(c))
    return {"row_ptr": np.array(ptr, dtype=np.int64),
            "col": np.concatenate(cols) if cols else np.zeros(0, np.int64)}


def sampled_mask_csr(geom, rho1: float, rho2: float, seed: int):
    """The paper-exact static-ratio block mask (all rows; small geometries)."""
    return aggregate_links(geom, sampled_links(geom, rho1, rho2, seed))


def sampled_mask_rows(geom, rho1: float, rho2: float, seed: int, rows, thresholds=None):
    """Block-mask rows for the given query blocks, by token-level evaluation of
    the sample restricted to each row's query tokens (large geometries).
    ``thresholds``: optional dict (i, j) -> T, else computed here.  Returns a
    list of sorted int64 arrays."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    nb = -(-n // geom.block)
    l0 = G.base_span(nt)
    w_t, r_t = G.frame_tables(geom)
    keys_all = np.arange(n, dtype=np.int64)
    kj, kv = keys_all // nt, keys_all % nt
    blk_of_key = keys_all // geom.block
    n_valid = np.bincount(blk_of_key, minlength=nb)
    thr = {} if thresholds is None else dict(thresholds)
    out = []
    for row in rows:
        q = np.arange(row * geom.block, min((row + 1) * geom.block, n), dtype=np.int64)
        col_count = np.zeros(n, dtype=np.int64)
        near = np.zeros(n, dtype=bool)
        for qq in q:
            i, u = divmod(int(qq), nt)
            t = np.abs(i - kj)
            in_p = r_t[t] & (np.abs(u - kv) <= w_t[t])
            sampled = in_p.copy()
            far = in_p & (t >= 2)
            for j in np.unique(kj[far]):
                j = int(j)
                if (i, j) not in thr:
                    thr[(i, j)] = frame_pair_threshold(geom, i, j, rho1, rho2, seed)[2]
                sel = far & (kj == j)
                ks = pair_keys(seed, geom.frames, nt, i, j, np.full(int(sel.sum()), u), kv[sel])
                sampled[np.flatnonzero(sel)] = ks <= np.uint64(thr[(i, j)])
            col_count += sampled
            near |= (t <= geom.force_t) & r_t[t]
        active = col_count > geom.theta_c * len(q)
        n_active = np.bincount(blk_of_key, weights=active, minlength=nb)
        agg = n_active > geom.theta_m * n_valid
        forced = np.bincount(blk_of_key, weights=near, minlength=nb) > 0
        out.append(np.flatnonzero(agg | forced))
    return out
