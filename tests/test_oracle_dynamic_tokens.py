"""Pins of the oracle's paper-exact dynamic-threshold mode (DynamicRad Sec. 3.2,
Eqs. 9-11 and Eq. 19: fused-head proxy logits on candidate token pairs,
per-frame-pair z-scores, tau_1 / tau_2 thresholds with the top-pair fallback)."""
import math

import numpy as np
import pytest

from oracle import dynamic_tokens as DT
from oracle import geometry as G
from oracle import sampling as S
from block_sparse_attention_candidate_b200.workloads import Geometry


def _qk(geom, hf=2, d=8, seed=0):
    rng = np.random.default_rng(seed)
    n = geom.frames * geom.height * geom.width
    return rng.standard_normal((hf, n, d)), rng.standard_normal((hf, n, d))


def test_proxy_scores_brute_force():
    geom = Geometry(3, 2, 3, 4, 0.5, 2.0)
    qf, kf = _qk(geom, hf=3, d=5)
    nt = 6
    u, v = S.candidate_pairs(geom, 2)
    s = DT.proxy_scores(qf, kf, 0, 2, u, v, nt)
    for x, (a, b) in enumerate(zip(u, v)):
        want = sum(float(np.dot(qf[h, a], kf[h, 2 * nt + b])) for h in range(3)) / 3 / math.sqrt(5)
        assert abs(s[x] - want) < 1e-12


def test_z_scores_have_zero_mean_unit_std():
    geom = Geometry(4, 3, 5, 4, 0.5, 2.0)
    qf, kf = _qk(geom)
    for i, j in [(0, 2), (3, 0), (1, 1)]:
        n, mu, sigma, smax, arg, s = DT.frame_pair_stats(geom, qf, kf, i, j)
        z = (s - mu) / (sigma + DT.EPS_Z)
        assert abs(z.mean()) < 1e-9 and abs(z.std() - sigma / (sigma + DT.EPS_Z)) < 1e-9
        u, v = S.candidate_pairs(geom, abs(i - j))
        first = int(np.flatnonzero(s == s.max())[0])
        assert smax == s.max() and arg == int(u[first] * 15 + v[first])


def test_threshold_eq11_regimes():
    geom = Geometry(40, 16, 16, 32, 0.5, 2.0)      # L(2), L(3) = 32 >= 32; L(4) = 16 < 32
    assert DT.threshold(geom, 0, 1.0, 2.0) == -math.inf
    assert DT.threshold(geom, 1, 1.0, 2.0) == -math.inf
    assert DT.threshold(geom, 2, 1.0, 2.0) == 1.0
    assert DT.threshold(geom, 4, 1.0, 2.0) == 2.0


def test_high_threshold_keeps_only_the_argmax_pair():
    geom = Geometry(4, 3, 5, 4, 0.5, 2.0)
    qf, kf = _qk(geom, seed=3)
    nt = 15
    for i, j in [(0, 2), (3, 1), (0, 3)]:
        keep = DT.kept_pairs(geom, qf, kf, i, j, 1e9, 1e9)
        u, v = S.candidate_pairs(geom, abs(i - j))
        s = DT.proxy_scores(qf, kf, i, j, u, v, nt)
        assert keep.sum() == 1 and s[keep][0] == s.max()


def test_minus_infinity_thresholds_reduce_to_the_candidate_set():
    for geom in [Geometry(4, 4, 4, 8, 0.5, 2.0), Geometry(5, 3, 5, 4, 0.7, 0.3, theta_c=0.2, theta_m=0.3)]:
        qf, kf = _qk(geom, seed=1)
        got = DT.dynamic_mask_csr(geom, qf, kf, -math.inf, -math.inf)
        want = G.candidate_csr(geom)
        np.testing.assert_array_equal(got["row_ptr"], want["row_ptr"])
        np.testing.assert_array_equal(got["col"], want["col"])


def test_kept_sets_are_nested_in_tau_and_counts_match_the_z_rule():
    geom = Geometry(5, 4, 4, 8, 0.5, 2.0)
    qf, kf = _qk(geom, seed=2)
    prev = None
    for tau in (2.0, 1.0, 0.0, -1.0):
        cur = DT.dynamic_links(geom, qf, kf, tau, tau)
        if prev is not None:
            assert not (prev & ~cur).any()
        prev = cur
    # count for one frame pair: #{z > tau}, or 1 through the fallback
    n, mu, sigma, _, _, s = DT.frame_pair_stats(geom, qf, kf, 0, 3)
    z = (s - mu) / (sigma + DT.EPS_Z)
    for tau in (-0.5, 0.7, 5.0):
        assert DT.kept_pairs(geom, qf, kf, 0, 3, tau, tau).sum() == max(1, int((z > tau).sum()))


@pytest.mark.parametrize("geom", [Geometry(4, 4, 4, 8, 0.5, 2.0), Geometry(5, 3, 5, 4, 0.7, 0.3, theta_c=0.2, theta_m=0.3),
                                  Geometry(5, 4, 4, 8, 0.5, 2.0, force_t=0)])
@pytest.mark.parametrize("taus", [(0.5, 1.5), (2.5, 0.0), (9.0, 9.0)])
def test_row_restricted_form_matches_the_whole_mask(geom, taus):
    # the dense-logit per-row evaluation the full-size GPU checks use equals the
    # rows of the pair-list construction (including the top-pair fallback)
    qf, kf = _qk(geom, seed=4)
    want = DT.dynamic_mask_csr(geom, qf, kf, *taus)
    nb = geom.n_blocks
    got = DT.dynamic_mask_rows(geom, qf, kf, taus[0], taus[1], list(range(nb)))
    for r in range(nb):
        np.testing.assert_array_equal(got[r], want["col"][want["row_ptr"][r]:want["row_ptr"][r + 1]])
