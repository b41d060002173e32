"""Pins of the oracle's masked attention (DynamicRad Sec. 3.3, Eqs. 12-13)."""
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import attention as A
from oracle import geometry as G
from oracle import selection as S
from block_sparse_attention_candidate_b200.workloads import (
    WORKLOADS, Geometry, bf16_bits_to_f64, make_qkv_bf16)


def _full_csr(nb):
    return np.arange(nb + 1) * nb, np.tile(np.arange(nb), nb)


def _rand(seed, n, d, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((n, d)) * scale for _ in range(3)]


@pytest.mark.parametrize("n,d,bs", [(96, 16, 32), (70, 8, 16), (33, 64, 32), (5, 4, 8)])
def test_full_mask_equals_library_dense_attention(n, d, bs):
    q, k, v = _rand(n * d, n, d, 1.5)
    rp, col = _full_csr(-(-n // bs))
    o, lse = A.sparse_attention(q, k, v, bs, rp, col)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None])[0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(q @ k.T / math.sqrt(d), axis=1),
                               rtol=1e-13, atol=1e-13)


def test_eq13_literal_with_vanishing_eps_equals_block_skipping():
    geom = Geometry(4, 4, 4, 8, 0.3, 2.0)
    n, d = geom.n_tokens, 16
    q, k, v = _rand(5, n, d)
    cand = G.candidate_csr(geom)
    kept, _ = S.select_head(q, k, geom.block, cand, "static", 0.3)
    o, lse = A.sparse_attention(q, k, v, geom.block, kept["row_ptr"], kept["col"])
    mask = A.token_mask(geom.block, n, kept["row_ptr"], kept["col"])
    assert 0 < mask.mean() < 1
    o13, lse13 = A.eq13_dense(q, k, v, mask, eps=1e-300)
    np.testing.assert_allclose(o, o13, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse13, rtol=1e-12, atol=1e-12)
    # a finite eps leaks mass into the masked blocks: visibly different
    o_leak, _ = A.eq13_dense(q, k, v, mask, eps=1e-2)
    assert np.abs(o_leak - o).max() > 1e-3


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(11)
    n, d, bs = 64, 8, 16
    q = rng.standard_normal((n, d))
    k = np.tile(rng.standard_normal(d), (n, 1))
    v = rng.standard_normal((n, d))
    rp = np.array([0, 1, 3, 4, 6])
    col = np.array([0, 0, 1, 2, 1, 3])
    o, lse = A.sparse_attention(q, k, v, bs, rp, col)
    np.testing.assert_allclose(o[0], v[0:16].mean(axis=0), atol=1e-13)
    np.testing.assert_allclose(o[20], v[0:32].mean(axis=0), atol=1e-13)
    np.testing.assert_allclose(o[63], np.concatenate([v[16:32], v[48:64]]).mean(axis=0), atol=1e-13)
    # lse of uniform logits a over m keys is a + ln m
    np.testing.assert_allclose(lse[20], q[20] @ k[0] / math.sqrt(d) + math.log(32), atol=1e-13)


def test_single_key_block():
    # one kept block holding one valid key (ragged tail): o = v_key, lse = logit
    rng = np.random.default_rng(12)
    n, d, bs = 33, 8, 16
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    rp = np.array([0, 1, 2, 3])
    col = np.array([2, 2, 2])
    o, lse = A.sparse_attention(q, k, v, bs, rp, col)
    np.testing.assert_allclose(o, np.tile(v[32], (n, 1)), atol=1e-14)
    np.testing.assert_allclose(lse, q @ k[32] / math.sqrt(d), atol=1e-13)


def test_output_in_convex_hull_and_discarded_mass_bound():
    # App. C.3: the error is bounded by the attention mass the mask discards.
    # With m_q = exp(lse_sparse - lse_dense) the kept mass of row q, the
    # definitions give |o_sparse - o_dense|_inf <= 2 (1 - m_q) max |V|.
    wl = WORKLOADS["tiny"]
    g = wl.geom
    qkv = make_qkv_bf16(wl)
    q, k, v = (bf16_bits_to_f64(qkv[t][0, 1]) for t in "qkv")
    cand = G.candidate_csr(g)
    kept, _ = S.select_head(q, k, g.block, cand, "static", 0.25)
    o, lse = A.sparse_attention(q, k, v, g.block, kept["row_ptr"], kept["col"])
    od, lsed = A.sparse_attention(q, k, v, g.block, *_full_csr(g.n_blocks))
    m = np.exp(lse - lsed)
    assert np.all(m > 0) and np.all(m <= 1 + 1e-12)
    bound = 2 * (1 - m) * np.abs(v).max()
    assert np.all(np.abs(o - od).max(axis=1) <= bound + 1e-12)
    assert np.all(o <= v.max(axis=0) + 1e-12) and np.all(o >= v.min(axis=0) - 1e-12)
    assert m.mean() < 0.999          # the mask does drop something


def test_row_sampling_matches_full_evaluation():
    q, k, v = _rand(21, 100, 8)
    rp, col = np.array([0, 2, 3, 5, 7]), np.array([0, 3, 1, 1, 2, 0, 3])
    o, lse = A.sparse_attention(q, k, v, 32, rp, col)
    part = A.sparse_attention_rows(q, k, v, 32, rp, col, rows=[1, 3], token_rows={1: [0, 5], 3: [2]})
    toks, ob, lb = part[1]
    np.testing.assert_array_equal(toks, [32, 37])
    np.testing.assert_allclose(ob, o[[32, 37]], atol=0)
    toks, ob, lb = part[3]
    np.testing.assert_array_equal(toks, [98])
    np.testing.assert_allclose(lb, lse[[98]], atol=0)
