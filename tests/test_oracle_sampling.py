"""Pins of the oracle's paper-exact static-ratio mode (DynamicRad Sec. 3.2,
Eq. 8: seeded uniform sampling of k token pairs per frame pair, then the block
aggregation of Sec. 3.1)."""
import itertools

import numpy as np
import pytest

from conftest import read_golden
from oracle import geometry as G
from oracle import sampling as S
from block_sparse_attention_candidate_b200.workloads import Geometry

M64 = (1 << 64) - 1


def test_splitmix64_known_answers():
    rows = read_golden("splitmix64.txt")
    assert rows
    for seed, idx, val in rows:
        assert S.splitmix64_sequence(int(seed), int(idx))[-1] == int(val, 16)


def _unmix(z):
    # inverse of the finaliser, from the algebra: x ^= x >> s is undone by
    # repeating it until the shift covers 64 bits; multiplication by an odd
    # constant is undone by its inverse mod 2^64
    def unxorshift(x, s):
        y = x
        for _ in range(64 // s + 1):
            y = x ^ (y >> s)
        return y & M64
    z = unxorshift(z, 31)
    z = (z * pow(0x94D049BB133111EB, -1, 1 << 64)) & M64
    z = unxorshift(z, 27)
    z = (z * pow(0xBF58476D1CE4E5B9, -1, 1 << 64)) & M64
    return unxorshift(z, 30)


def test_splitmix64_finaliser_is_a_bijection_and_numpy_agrees():
    rng = np.random.default_rng(0)
    xs = [int(x) for x in rng.integers(0, 2 ** 63, 300, dtype=np.uint64)] + [0, 1, M64, 1 << 63]
    for x in xs:
        assert _unmix(S.splitmix64_mix(x)) == x
    got = S.splitmix64_mix_np(np.array(xs, dtype=np.uint64))
    assert [int(g) for g in got] == [S.splitmix64_mix(x) for x in xs]


@pytest.mark.parametrize("nt,w", [(1, 1), (5, 0), (7, 2), (16, 16), (33, 5), (64, 100)])
def test_candidate_pairs_brute_force(nt, w):
    geom = Geometry(3, 1, nt, 4, 1.0, 2.0)
    # force the window through t = 0 (w = N_t) or a direct check of the band
    u, v = S.candidate_pairs(geom, 0)
    assert sorted(zip(u.tolist(), v.tolist())) == [(a, b) for a in range(nt) for b in range(nt)]
    # band of half-width w, by brute force against the closed-form enumeration
    lo = np.maximum(np.arange(nt) - w, 0)
    hi = np.minimum(np.arange(nt) + w, nt - 1)
    want = [(a, b) for a in range(nt) for b in range(nt) if abs(a - b) <= w]
    assert int((hi - lo + 1).sum()) == len(want)


def test_candidate_pairs_follow_eq7_and_the_split_rule():
    geom = Geometry(6, 4, 8, 8, 0.5, 0.1, eps=1e-6)        # lambda small: the split rule fires
    nt, l0 = 32, G.base_span(32)
    for t in range(geom.frames):
        u, v = S.candidate_pairs(geom, t)
        if not G.frame_pair_retained(t, l0, geom.block, geom.lam, geom.eps):
            assert len(u) == 0
            continue
        w = G.window(t, nt, l0, geom.block, geom.gamma)
        want = [(a, b) for a in range(nt) for b in range(nt) if abs(a - b) <= w]
        assert list(zip(u.tolist(), v.tolist())) == want


def test_sample_size():
    assert S.sample_size(10, 0.3) == 3          # 0.3 * 10 is 2.9999999999999996 in binary
    assert S.sample_size(7, 0.01) == 1
    assert S.sample_size(7, 1.0) == 7
    assert S.sample_size(0, 0.5) == 0


def test_retention_ratio_eq8_regimes():
    geom = Geometry(40, 16, 16, 32, 0.5, 2.0)   # N_t = 256 = L0; L(t) = 256 / 2^B(t) * 0.5
    assert S.retention_ratio(geom, 0, 0.3, 0.1) == 1.0
    assert S.retention_ratio(geom, 1, 0.3, 0.1) == 1.0
    # t = 2, 3: L = 32 >= 32 -> near; t = 4: L = 16 < 32 -> far
    assert S.retention_ratio(geom, 2, 0.3, 0.1) == 0.3
    assert S.retention_ratio(geom, 3, 0.3, 0.1) == 0.3
    assert S.retention_ratio(geom, 4, 0.3, 0.1) == 0.1


def test_threshold_selects_exactly_k_distinct_keys():
    geom = Geometry(5, 4, 8, 8, 0.5, 2.0)
    nt = 32
    for (i, j) in [(0, 2), (3, 0), (4, 1), (1, 4)]:
        k, n, T = S.frame_pair_threshold(geom, i, j, 0.35, 0.2, seed=7)
        u, v = S.candidate_pairs(geom, abs(i - j))
        keys = S.pair_keys(7, geom.frames, nt, i, j, u, v)
        assert len(np.unique(keys)) == len(keys) == n
        assert int((keys <= np.uint64(T)).sum()) == k >= 1


@pytest.mark.parametrize("geom", [Geometry(4, 4, 4, 8, 0.5, 2.0), Geometry(5, 3, 5, 4, 0.7, 0.3),
                                  Geometry(4, 4, 4, 8, 0.5, 2.0, theta_c=0.2, theta_m=0.3),
                                  Geometry(6, 2, 5, 16, 0.4, 0.1)])
def test_full_retention_reduces_to_the_candidate_set(geom):
    # rho_1 = rho_2 = 1 samples every pair of P: the mask is stage 1's candidate set
    got = S.sampled_mask_csr(geom, 1.0, 1.0, seed=3)
    want = G.candidate_csr(geom)
    np.testing.assert_array_equal(got["row_ptr"], want["row_ptr"])
    np.testing.assert_array_equal(got["col"], want["col"])


def test_samples_are_nested_in_rho_and_inside_p():
    geom = Geometry(5, 4, 8, 8, 0.5, 2.0)
    full = S.sampled_links(geom, 1.0, 1.0, 11)
    prev = None
    for rho in (0.05, 0.2, 0.5, 0.9):
        cur = S.sampled_links(geom, rho, rho, 11)
        assert not (cur & ~full).any()
        if prev is not None:
            assert not (prev & ~cur).any()
        prev = cur


def test_sample_is_uniform_over_seeds():
    # each pair of P is in the k-subset with probability k / n: frequency over
    # 400 seeds within 5 standard deviations, and the mean exactly k / n
    geom = Geometry(3, 1, 6, 4, 1.0, 2.0)
    i, j = 0, 2
    u, v = S.candidate_pairs(geom, 2)
    n = len(u)
    k = S.sample_size(n, 0.25)
    hits = np.zeros(n)
    seeds = 400
    for s in range(seeds):
        keys = S.pair_keys(s, geom.frames, 6, i, j, u, v)
        T = np.partition(keys, k - 1)[k - 1]
        hits += keys <= T
    p = k / n
    sd = np.sqrt(seeds * p * (1 - p))
    assert np.all(np.abs(hits - seeds * p) < 5 * sd)
    assert hits.sum() == seeds * k


def test_tiny_workload_rho_regimes_differ():
    geom = Geometry(4, 16, 16, 32, 0.5, 2.0)
    m1 = S.sampled_mask_csr(geom, 0.9, 0.9, 1)
    m2 = S.sampled_mask_csr(geom, 0.05, 0.05, 1)
    assert m2["row_ptr"][-1] <= m1["row_ptr"][-1]


@pytest.mark.parametrize("geom", [Geometry(4, 4, 4, 8, 0.5, 2.0), Geometry(5, 3, 5, 4, 0.7, 0.3),
                                  Geometry(4, 4, 4, 8, 0.5, 2.0, theta_c=0.2, theta_m=0.3),
                                  Geometry(6, 2, 5, 16, 0.4, 0.1, force_t=0)])
@pytest.mark.parametrize("rho", [(0.3, 0.1), (0.6, 0.6)])
def test_row_restricted_form_matches_the_whole_mask(geom, rho):
    # the per-row evaluation the full-size GPU checks use equals the rows of the
    # whole-matrix construction (same sample, same aggregation)
    want = S.sampled_mask_csr(geom, rho[0], rho[1], seed=5)
    nb = geom.n_blocks
    got = S.sampled_mask_rows(geom, rho[0], rho[1], 5, list(range(nb)))
    for r in range(nb):
        np.testing.assert_array_equal(got[r], want["col"][want["row_ptr"][r]:want["row_ptr"][r + 1]])
