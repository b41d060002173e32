"""Stage 2 on the GPU vs the oracle: pooled block scores within fp32 tolerance,
kept-block CSR bit-exact given the GPU's exported fp32 scores."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (
    WORKLOADS, Geometry, Workload, bf16_bits_to_f64, make_qkv_bf16, random_qkv_bf16)
from gpu_util import (SCORE_REL, cand_to_numpy, check_device_status, compare_selection, csr_rows,
                      gpu_inputs)
from oracle import selection as OS

pytestmark = pytest.mark.gpu


def _run(wl: Workload, qkv_bits, mode, value):
    geom = wl.geom
    q, k, _ = gpu_inputs(qkv_bits)
    cand = abi.dynrad_build_candidates(geom)
    row_ptr, col_idx, scores = abi.dynrad_select_blocks(q, k, geom, cand, mode, value, scores=True)
    torch.cuda.synchronize()
    check_device_status()
    return cand, row_ptr.cpu().numpy().astype(np.int64), col_idx.cpu().numpy().astype(np.int64), \
        scores.cpu().numpy()


def _check_scores(wl, qkv_bits, cand_np, scores, b, h, rows):
    nb = wl.geom.n_blocks
    bh = b * wl.heads + h
    q = bf16_bits_to_f64(qkv_bits["q"][b, h])
    k = bf16_bits_to_f64(qkv_bits["k"][b, h])
    qbar = OS.block_means(q, wl.geom.block)
    kbar = OS.block_means(k, wl.geom.block)
    nnz = len(cand_np["col"])
    for r in rows:
        a, e = cand_np["row_ptr"][r], cand_np["row_ptr"][r + 1]
        cols = cand_np["col"][a:e]
        want = OS.block_scores(qbar, kbar, r, cols)
        got = scores[bh * nnz + a: bh * nnz + e].astype(np.float64)
        scale = np.linalg.norm(qbar[r]) * np.linalg.norm(kbar[cols], axis=1) / math.sqrt(q.shape[1])
        assert np.all(np.abs(got - want) <= SCORE_REL * scale + 1e-7), (b, h, r)


@pytest.mark.parametrize("mode,value", [("static", 0.25), ("dynamic", 0.8), ("static", 1.0),
                                        ("dynamic", 1.0), ("static", 0.05), ("dynamic", 0.3)])
def test_tiny_selection_parity(mode, value):
    wl = WORKLOADS["tiny"]
    bits = make_qkv_bf16(wl)
    cand, rp, col, scores = _run(wl, bits, mode, value)
    cand_np = cand_to_numpy(cand)
    nb = wl.geom.n_blocks
    for h in range(wl.heads):
        _check_scores(wl, bits, cand_np, scores, 0, h, range(nb))
        kept = csr_rows(rp, col, h, nb)
        assert compare_selection(mode, value, cand_np, kept, scores, h, nb, cand["nnz"]) == 0
        # and against the oracle's own scores: only near-ties may differ
        q = bf16_bits_to_f64(bits["q"][0, h])
        k = bf16_bits_to_f64(bits["k"][0, h])
        ref, _ = OS.select_head(q, k, wl.geom.block, cand_np, mode, value)
        same = sum(np.array_equal(ref["col"][ref["row_ptr"][r]:ref["row_ptr"][r + 1]], kept[r])
                   for r in range(nb))
        assert same >= nb - 2
    if value == 1.0:
        assert rp[-1] == wl.heads * cand["nnz"]


@pytest.mark.parametrize("geom,D", [(Geometry(5, 3, 5, 8, 0.3, 2.0), 64),
                                    (Geometry(6, 8, 8, 16, 0.05, 0.5), 128),
                                    (Geometry(7, 6, 10, 32, 0.3, 0.2), 128),
                                    (Geometry(9, 12, 12, 64, 0.4, 0.05, theta_c=0.1, theta_m=0.2), 64),
                                    (Geometry(12, 10, 13, 128, 0.6, 3.0), 128)])
@pytest.mark.parametrize("mode,value", [("static", 0.2), ("dynamic", 0.9)])
def test_ragged_grids_random_inputs(geom, D, mode, value):
    wl = Workload("adhoc", 2, 3, D, geom, seed=5)
    bits = random_qkv_bf16(1234 + geom.block + D, 2, 3, geom.n_tokens, D, scale=2.0)
    cand, rp, col, scores = _run(wl, bits, mode, value)
    cand_np = cand_to_numpy(cand)
    nb = geom.n_blocks
    for b in range(2):
        for h in range(3):
            bh = b * 3 + h
            _check_scores(wl, bits, cand_np, scores, b, h, range(nb))
            kept = csr_rows(rp, col, bh, nb)
            assert compare_selection(mode, value, cand_np, kept, scores, bh, nb, cand["nnz"]) == 0


def test_ties_lower_index_wins_on_gpu():
    # identical K rows everywhere -> identical block scores within each row:
    # static selection must keep the lowest-index free candidates
    geom = Geometry(6, 4, 8, 8, 0.3, 2.0)
    D = 64
    n = geom.n_tokens
    rng = np.random.default_rng(3)
    kb = np.tile(rng.standard_normal(D).astype(np.float32), (n, 1))
    bits = random_qkv_bf16(9, 1, 1, n, D)
    from block_sparse_attention_candidate_b200.workloads import round_to_bf16_bits
    bits["k"] = round_to_bf16_bits(kb)[None, None]
    wl = Workload("ties", 1, 1, D, geom, seed=0)
    cand, rp, col, scores = _run(wl, bits, "static", 0.3)
    cand_np = cand_to_numpy(cand)
    nb = geom.n_blocks
    kept = csr_rows(rp, col, 0, nb)
    assert compare_selection("static", 0.3, cand_np, kept, scores, 0, nb, cand["nnz"]) == 0
    for r in range(nb):
        a, e = cand_np["row_ptr"][r], cand_np["row_ptr"][r + 1]
        cols = cand_np["col"][a:e]
        free = [c for c in cols if not cand_np["forced_lo"][r] <= c <= cand_np["forced_hi"][r]]
        kfree = [c for c in kept[r] if not cand_np["forced_lo"][r] <= c <= cand_np["forced_hi"][r]]
        assert kfree == free[:len(kfree)]


def test_monotone_in_rho_and_tau_on_gpu():
    wl = WORKLOADS["tiny"]
    bits = make_qkv_bf16(wl)
    nb = wl.geom.n_blocks
    for mode, values in (("static", [0.1, 0.25, 0.5, 1.0]), ("dynamic", [0.5, 0.8, 0.95, 1.0])):
        prev = None
        for v in values:
            _, rp, col, _ = _run(wl, bits, mode, v)
            cur = [set(x.tolist()) for h in range(wl.heads) for x in csr_rows(rp, col, h, nb)]
            if prev is not None:
                assert all(a <= b for a, b in zip(prev, cur))
            prev = cur


@pytest.mark.parametrize("name,gamma", [("tiny", None), ("wan13b_480p", None)])
@pytest.mark.parametrize("mode,value", [("static", 0.2), ("dynamic", 0.8)])
def test_selection_without_score_export_matches(name, gamma, mode, value):
    # the bench path calls selection without exporting scores; static mode then
    # skips scoring the forced blocks -- the kept CSR must not change
    wl = WORKLOADS[name]
    bits = make_qkv_bf16(wl, heads=range(min(wl.heads, 4)))
    wl = Workload(wl.name, wl.batch, min(wl.heads, 4), wl.head_dim, wl.geom, wl.seed)
    q, k, _ = gpu_inputs(bits)
    cand = abi.dynrad_build_candidates(wl.geom)
    rp1, col1, _ = abi.dynrad_select_blocks(q, k, wl.geom, cand, mode, value, scores=True)
    rp1, col1 = rp1.clone(), col1.clone()
    rp2, col2, _ = abi.dynrad_select_blocks(q, k, wl.geom, cand, mode, value, scores=False)
    torch.cuda.synchronize()
    check_device_status()
    assert torch.equal(rp1, rp2)
    n = int(rp1[-1])
    assert torch.equal(col1[:n], col2[:n])


@pytest.mark.parametrize("mode,value", [("static", 0.2), ("dynamic", 0.85)])
def test_every_selection_width_gives_the_same_csr(mode, value):
    # The selection kernel is instantiated for 4, 8, 16 or 32 candidates per
    # lane, picked from the declared longest candidate row; declaring a longer
    # bound (clamped to Nb) picks a wider instance over the same data, which
    # must keep exactly the same blocks.  Rows of at most 128 candidates and
    # Nb = 576 let the same data run all four widths.
    geom = Geometry(36, 4, 32, 8, 0.05, 0.2)
    D = 64
    bits = random_qkv_bf16(77, 1, 2, geom.n_tokens, D, scale=2.0)
    q, k, _ = gpu_inputs(bits)
    cand = abi.dynrad_build_candidates(geom)
    nb = geom.n_blocks
    assert nb > 512
    real = cand["max_row"]
    assert real <= 128
    results = []
    for bound in sorted({real, max(real, 129), max(real, 257), max(real, 513), nb}):
        rp, col, scores = abi.dynrad_select_blocks(q, k, geom, dict(cand, max_row=bound), mode, value, scores=True)
        torch.cuda.synchronize()
        check_device_status()
        results.append((bound, rp.cpu().numpy().astype(np.int64), col.cpu().numpy().astype(np.int64),
                        scores.cpu().numpy()))
    _, rp0, col0, sc0 = results[0]
    cand_np = cand_to_numpy(cand)
    for h in range(2):
        assert compare_selection(mode, value, cand_np, csr_rows(rp0, col0, h, nb), sc0, h, nb, cand["nnz"]) == 0
    for bound, rp, col, sc in results[1:]:
        np.testing.assert_array_equal(rp, rp0, err_msg=f"bound {bound}")
        np.testing.assert_array_equal(col[: rp0[-1]], col0[: rp0[-1]], err_msg=f"bound {bound}")
        np.testing.assert_array_equal(sc, sc0, err_msg=f"bound {bound}")
