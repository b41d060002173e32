"""Pins of the oracle's radial candidate geometry (DynamicRad Sec. 3.1, Eqs. 1-7)."""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden
from oracle import geometry as G
from block_sparse_attention_candidate_b200.workloads import Geometry, WORKLOADS


def test_log_group_matches_eq1_formula():
    # Eq. 1 writes B(t) = floor(log2 t) + 1; the oracle evaluates it exactly as
    # the bit length.  Compare with the floating formula where it is exact
    # (powers of two and their neighbours are the risky points).
    for t in list(range(1, 5000)) + [2 ** e + d for e in range(13, 46) for d in (-1, 0, 1)]:
        assert G.log_group(t) == math.floor(math.log2(t)) + 1, t
    with pytest.raises(ValueError):
        G.log_group(0)


@pytest.mark.parametrize("nt,l0", [(1, 1), (2, 2), (3, 4), (256, 256), (257, 512),
                                   (1560, 2048), (3600, 4096), (4096, 4096)])
def test_base_span_next_power_of_two(nt, l0):
    assert G.base_span(nt) == l0


def test_window_widths_golden():
    rows = read_golden("window_widths.txt")
    assert len(rows) > 20
    for nt, bs, gamma, t, w in rows:
        nt, bs, t, w = int(nt), int(bs), int(t), int(w)
        assert G.window(t, nt, G.base_span(nt), bs, float(gamma)) == w, (nt, bs, gamma, t)


def test_split_rule_golden():
    for nt, bs, lam, eps, t, sf, kept in read_golden("split_retention.txt"):
        nt, bs, t, sf, kept = int(nt), int(bs), int(t), int(sf), int(kept)
        l0 = G.base_span(nt)
        assert G.split_factor(t, l0, bs, float(lam), float(eps)) == sf, (nt, bs, lam, t)
        assert G.frame_pair_retained(t, l0, bs, float(lam), float(eps)) == bool(kept)


def test_split_rule_is_noop_at_every_workload():
    # with lambda >= 2 the split length stays >= B_s for every distance in range
    for wl in WORKLOADS.values():
        g = wl.geom
        w, r = G.frame_tables(g)
        assert r.all(), wl.name


def _brute_candidates(geom):
    """Pure-Python enumeration of Eq. 7 over every token pair + the aggregation rule."""
    nt = geom.height * geom.width
    n = geom.frames * nt
    bs = geom.block
    nb = -(-n // bs)
    l0 = G.base_span(nt)
    cand = [[False] * nb for _ in range(nb)]
    forced = [[False] * nb for _ in range(nb)]
    for bi in range(nb):
        qs = range(bi * bs, min((bi + 1) * bs, n))
        for bj in range(nb):
            ks = range(bj * bs, min((bj + 1) * bs, n))
            active = 0
            for kk in ks:
                linked = sum(1 for qq in qs if G.token_pair_allowed(geom, qq, kk))
                if linked > geom.theta_c * len(qs):
                    active += 1
                for qq in qs:
                    t = abs(qq // nt - kk // nt)
                    if t <= geom.force_t and G.frame_pair_retained(t, l0, bs, geom.lam, geom.eps):
                        forced[bi][bj] = True
            cand[bi][bj] = active > geom.theta_m * len(ks) or forced[bi][bj]
    return cand, forced


TINY_GRIDS = [
    Geometry(4, 4, 4, 8, 0.5, 2.0),
    Geometry(5, 3, 5, 8, 0.3, 2.0),            # blocks straddle frames, ragged tail
    Geometry(6, 4, 4, 4, 0.2, 0.5),            # split rule fires (retained t: 0,1,2,3)
    Geometry(6, 8, 8, 16, 0.05, 0.5),          # split rule fires, w clipped at B_s
    Geometry(3, 5, 7, 32, 0.5, 1.0),           # a block spans all frames
    Geometry(6, 4, 4, 4, 0.2, 0.1),            # adjacent frames dropped by the split rule
    Geometry(5, 4, 6, 8, 0.4, 2.0, theta_c=0.25, theta_m=0.3),
    Geometry(4, 4, 4, 8, 0.3, 2.0, theta_c=0.5, theta_m=0.5, force_t=0),
]


@pytest.mark.parametrize("geom", TINY_GRIDS)
def test_candidates_match_token_level_brute_force(geom):
    cand, forced = _brute_candidates(geom)
    nb = geom.n_blocks
    for r in range(nb):
        c, f = G.candidate_row(geom, r)
        assert c.tolist() == [j for j in range(nb) if cand[r][j]], (geom, r)
        assert f.tolist() == [j for j in range(nb) if forced[r][j]], (geom, r)


@pytest.mark.parametrize("geom", TINY_GRIDS)
def test_forced_set_contains_diagonal_and_is_contiguous(geom):
    csr = G.candidate_csr(geom)  # asserts contiguity
    for r in range(geom.n_blocks):
        assert csr["forced_lo"][r] <= r <= csr["forced_hi"][r]
        row = csr["col"][csr["row_ptr"][r]:csr["row_ptr"][r + 1]]
        assert set(range(csr["forced_lo"][r], csr["forced_hi"][r] + 1)) <= set(row.tolist())
        assert np.all(np.diff(row) > 0)


def test_symmetry_with_zero_thresholds():
    # |i - j| and |u - v| are symmetric, so with theta = 0 and no ragged tail the
    # block candidate relation is symmetric
    for geom in [Geometry(6, 4, 4, 8, 0.3, 2.0), Geometry(6, 4, 4, 4, 0.2, 0.5),
                 Geometry(4, 6, 8, 16, 0.4, 1.0)]:
        assert geom.n_tokens % geom.block == 0
        nb = geom.n_blocks
        m = np.zeros((nb, nb), dtype=bool)
        for r in range(nb):
            m[r, G.candidate_row(geom, r)[0]] = True
        assert (m == m.T).all()


def test_wide_window_gives_full_candidate_set():
    geom = Geometry(6, 4, 6, 8, 100.0, 100.0)
    for r in range(geom.n_blocks):
        assert len(G.candidate_row(geom, r)[0]) == geom.n_blocks


def test_dropped_frame_pairs_leave_no_candidates():
    # N_t = 64, B_s = 16, lambda = 0.5: retained distances are 0, 1, 2, 3 and
    # 4, 5 are dropped (golden split file); with a window wider than the frame,
    # the candidates of a block are exactly the blocks of frames within 3
    geom = Geometry(6, 8, 8, 16, 10.0, 0.5)
    l0 = G.base_span(64)
    assert [G.frame_pair_retained(t, l0, 16, 0.5, 1e-6) for t in range(6)] == \
        [True, True, True, True, False, False]
    for r in range(geom.n_blocks):
        c, _ = G.candidate_row(geom, r)
        assert set(c.tolist()) == {j for j in range(geom.n_blocks) if abs(j // 4 - r // 4) <= 3}


def test_radial_window_widths_enter_the_candidate_set():
    # one frame per block row of 1 token: block = 1 token, so the candidate set of
    # token (i, u) is exactly {(j, v): retained, |u - v| <= w(|i - j|)}
    geom = Geometry(5, 2, 16, 1, 0.25, 4.0)
    nt = 32
    l0 = G.base_span(nt)
    for q in [0, 17, 40, 100, 159]:
        c, _ = G.candidate_row(geom, q)
        i, u = divmod(q, nt)
        expect = [k for k in range(geom.n_tokens)
                  if abs((k % nt) - u) <= G.window(abs(k // nt - i), nt, l0, 1, 0.25)]
        assert c.tolist() == expect
