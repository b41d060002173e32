"""Pins of the oracle's pooling, block scores and the two selection modes."""
import itertools
import math

import numpy as np
import pytest

from oracle import selection as S
from oracle import geometry as G
from block_sparse_attention_candidate_b200.workloads import (
    WORKLOADS, Geometry, bf16_bits_to_f64, make_qkv_bf16)


def test_block_means_hand_example_with_ragged_tail():
    x = np.arange(10, dtype=np.float64).reshape(5, 2)     # rows (0,1) (2,3) (4,5) (6,7) (8,9)
    m = S.block_means(x, 2)
    assert m.tolist() == [[1.0, 2.0], [5.0, 6.0], [8.0, 9.0]]   # last block has one valid row


def test_block_means_of_constant_blocks():
    rng = np.random.default_rng(3)
    rows = rng.standard_normal((7, 16))
    x = np.repeat(rows, 5, axis=0)[:33]                     # blocks of 5 identical rows, tail of 3
    np.testing.assert_allclose(S.block_means(x, 5), rows, rtol=0, atol=1e-15)


def test_block_scores_closed_forms():
    d = 64
    qbar = np.zeros((2, d))
    kbar = np.zeros((3, d))
    qbar[0, 0] = 2.0
    kbar[0, 0] = 3.0          # parallel: 6 / 8
    kbar[1, 1] = 5.0          # orthogonal: 0
    kbar[2, 0] = -1.0         # anti-parallel: -2 / 8
    s = S.block_scores(qbar, kbar, 0, [0, 1, 2])
    assert s.tolist() == [0.75, 0.0, -0.25]


@pytest.mark.parametrize("rho,n,k", [(0.15, 20, 3), (0.2, 1, 1), (0.25, 7, 1), (0.25, 8, 2),
                                     (0.2, 10, 2), (0.3, 10, 3), (1.0, 9, 9), (0.5, 0, 0),
                                     (0.01, 50, 1)])
def test_static_k_eq8(rho, n, k):
    # k = max(1, floor(|P| * rho)); products that are integers in exact
    # arithmetic (0.15 * 20 = 3, 0.3 * 10 = 3) must not floor to one less
    assert S.static_k(rho, n) == k


def _rank_key(cols, scores, i):
    return (-float(scores[i]), int(cols[i]))


def _random_row(rng, n, n_forced_lo=2, n_forced=3, ties=False):
    cols = np.sort(rng.choice(4 * n + 10, size=n, replace=False))
    if ties:
        scores = rng.integers(-3, 3, size=n).astype(np.float64) * 0.5
    else:
        scores = rng.standard_normal(n)
    lo = int(cols[min(n_forced_lo, n - 1)])
    hi = int(cols[min(n_forced_lo + n_forced - 1, n - 1)])
    return cols, scores, lo, hi


@pytest.mark.parametrize("seed", range(30))
def test_static_selection_is_the_top_k_by_score_then_index(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    cols, scores, lo, hi = _random_row(rng, n, ties=seed % 2 == 0)
    rho = float(rng.choice([0.1, 0.15, 0.2, 0.25, 0.5, 0.9]))
    kept = S.select_static(cols, scores, lo, hi, rho)
    forced = [(c >= lo and c <= hi) for c in cols]
    free = [i for i in range(n) if not forced[i]]
    kept_free = [i for i in free if cols[i] in set(kept.tolist())]
    # forced blocks always kept; exactly k others
    assert all(cols[i] in kept for i in range(n) if forced[i])
    assert len(kept_free) == S.static_k(rho, len(free))
    # exchange argument: every kept one ranks above every dropped one
    dropped = [i for i in free if i not in kept_free]
    for a in kept_free:
        for b in dropped:
            assert _rank_key(cols, scores, a) < _rank_key(cols, scores, b)
    assert np.all(np.diff(kept) > 0)


def test_static_ties_lower_index_wins_and_signed_zero_ties():
    cols = np.array([3, 5, 8, 9, 12])
    scores = np.array([0.0, -0.0, 1.0, 0.0, -0.0])
    # forced = [8, 8]; free = 3, 5, 9, 12 all tied at zero; rho 0.5 -> k = 2
    kept = S.select_static(cols, scores, 8, 8, 0.5)
    assert kept.tolist() == [3, 5, 8]


def _exhaustive_min_cut(cols, scores, lo, hi, tau):
    """Brute force: smallest number of non-forced blocks whose addition to the
    forced set reaches softmax mass tau, and every subset of that size that does."""
    e = np.exp(np.asarray(scores) - np.max(scores))
    z = math.fsum(e.tolist())
    forced = [i for i in range(len(cols)) if lo <= cols[i] <= hi]
    free = [i for i in range(len(cols)) if not (lo <= cols[i] <= hi)]
    mf = math.fsum(e[forced].tolist())
    for size in range(0, len(free) + 1):
        hits = [sub for sub in itertools.combinations(free, size)
                if math.fsum([mf] + [e[i] for i in sub]) >= tau * z]
        if hits:
            return size, hits
    return len(free), [tuple(free)]


@pytest.mark.parametrize("seed", range(40))
def test_dynamic_selection_is_minimal_and_reaches_tau(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 13))
    cols, scores, lo, hi = _random_row(rng, n, n_forced_lo=int(rng.integers(0, n)),
                                       n_forced=int(rng.integers(1, 3)))
    scores = scores * rng.choice([0.5, 2.0, 4.0])
    tau = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.97]))
    kept, info = S.dynamic_cut(cols, scores, lo, hi, tau)
    size, hits = _exhaustive_min_cut(cols, scores, lo, hi, tau)
    free_kept = [i for i in range(n) if cols[i] in set(kept.tolist()) and not (lo <= cols[i] <= hi)]
    assert len(free_kept) == size
    assert tuple(free_kept) in hits
    assert S.kept_mass(cols, scores, kept) >= tau - 1e-12
    # among the minimal sets it takes the highest-ranked blocks
    free = [i for i in range(n) if not (lo <= cols[i] <= hi)]
    order = sorted(free, key=lambda i: _rank_key(cols, scores, i))
    assert sorted(free_kept) == sorted(order[:size])


def test_dynamic_tau_one_keeps_everything():
    rng = np.random.default_rng(7)
    cols, scores, lo, hi = _random_row(rng, 30)
    assert S.select_dynamic(cols, scores, lo, hi, 1.0).tolist() == cols.tolist()


def test_static_rho_one_keeps_everything():
    rng = np.random.default_rng(8)
    cols, scores, lo, hi = _random_row(rng, 30)
    assert S.select_static(cols, scores, lo, hi, 1.0).tolist() == cols.tolist()


@pytest.mark.parametrize("seed", range(10))
def test_selection_is_monotone_in_rho_and_tau(seed):
    rng = np.random.default_rng(200 + seed)
    cols, scores, lo, hi = _random_row(rng, int(rng.integers(5, 60)))
    prev = set()
    for rho in [0.05, 0.1, 0.15, 0.2, 0.3, 0.5, 0.75, 1.0]:
        cur = set(S.select_static(cols, scores, lo, hi, rho).tolist())
        assert prev <= cur
        prev = cur
    prev = set()
    for tau in [0.1, 0.3, 0.5, 0.7, 0.8, 0.9, 0.95, 0.99, 1.0]:
        cur = set(S.select_dynamic(cols, scores, lo, hi, tau).tolist())
        assert prev <= cur
        prev = cur


def test_tiny_workload_selection_invariants():
    wl = WORKLOADS["tiny"]
    g = wl.geom
    cand = G.candidate_csr(g)
    qkv = make_qkv_bf16(wl)
    for h in range(wl.heads):
        q = bf16_bits_to_f64(qkv["q"][0, h])
        k = bf16_bits_to_f64(qkv["k"][0, h])
        kept_s, scores = S.select_head(q, k, g.block, cand, "static", 0.25)
        kept_d, _ = S.select_head(q, k, g.block, cand, "dynamic", 0.8)
        for r in range(g.n_blocks):
            cols = cand["col"][cand["row_ptr"][r]:cand["row_ptr"][r + 1]]
            ks = kept_s["col"][kept_s["row_ptr"][r]:kept_s["row_ptr"][r + 1]]
            kd = kept_d["col"][kept_d["row_ptr"][r]:kept_d["row_ptr"][r + 1]]
            assert r in ks and r in kd                               # diagonal kept
            assert set(ks) <= set(cols) and set(kd) <= set(cols)
            assert S.kept_mass(cols, scores[r], kd) >= 0.8 - 1e-12    # kept mass >= tau
