"""Parity at the five workloads' full sizes, in the launch configuration the
bench times (all heads of the layer in one call per stage), on sampled outputs
the oracle can compute one by one:

* candidates: sampled query blocks bit-exact (token-level oracle);
* scores: sampled (head, query block) rows within the fp32 tolerance;
* selection: every query block of two heads bit-exact against the oracle fed
  the GPU's fp32 scores;
* attention: sampled query blocks of those heads (every token of the block)
  against the oracle over the GPU's kept blocks, element by element.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (
    WORKLOADS, bf16_bits_to_f64, head_amplitudes, head_tensor_bf16, make_qkv_bf16, shared_field)
from gpu_util import (AMBIGUOUS_GAP, LSE_ABS, O_MAX_ABS, O_MEAN_ABS, SCORE_REL, cand_to_numpy,
                      check_device_status, compare_selection, csr_rows, gpu_inputs)
from oracle import attention as OA
from oracle import geometry as OG
from oracle import selection as OS

pytestmark = pytest.mark.gpu

CASES = [(name, i) for name in ("wan13b_480p", "wan14b_480p", "wan14b_720p", "hunyuan_720p")
         for i in range(len(WORKLOADS[name].runs))]

_inputs = {}


def _qkv(name):
    if name not in _inputs:
        _inputs.clear()
        torch.cuda.empty_cache()
        wl = WORKLOADS[name]
        _inputs[name] = gpu_inputs(make_qkv_bf16(wl))
    return _inputs[name]


@pytest.mark.parametrize("name,run", CASES, ids=[f"{n}-run{i}" for n, i in CASES])
def test_full_size_parity_sampled(name, run):
    wl = WORKLOADS[name]
    mode, value, gamma = wl.runs[run]
    g = wl.geom if gamma is None else wl.with_gamma(gamma).geom
    q, k, v = _qkv(name)
    B, H, N, D = q.shape
    nb = g.n_blocks
    rng = np.random.default_rng(1000 + 10 * list(WORKLOADS).index(name) + run)

    cand = abi.dynrad_build_candidates(g)
    rp, col, scores = abi.dynrad_select_blocks(q, k, g, cand, mode, value, scores=True)
    o, lse = abi.dynrad_sparse_attn(q, k, v, g.block, rp, col)
    torch.cuda.synchronize()
    check_device_status()
    cand_np = cand_to_numpy(cand)
    rp_np = rp.cpu().numpy().astype(np.int64)
    col_np = col[: int(rp_np[-1])].cpu().numpy().astype(np.int64)
    sc = scores.cpu().numpy()

    # candidates: sampled rows, bit-exact
    rows = sorted(set([0, nb - 1] + rng.choice(nb, 4, replace=False).tolist()))
    want = OG.candidate_csr(g, rows=rows)
    for i, r in enumerate(rows):
        got_row = cand_np["col"][cand_np["row_ptr"][r]:cand_np["row_ptr"][r + 1]]
        np.testing.assert_array_equal(got_row, want["col"][want["row_ptr"][i]:want["row_ptr"][i + 1]])
        assert cand_np["forced_lo"][r] == want["forced_lo"][i] and cand_np["forced_hi"][r] == want["forced_hi"][i]

    f = shared_field(wl)
    amps = head_amplitudes(wl)
    heads = sorted(set([0, H - 1] if H > 1 else [0]))
    ambiguous = 0
    for h in heads:
        qh, kh, vh = (bf16_bits_to_f64(head_tensor_bf16(wl, t, 0, h, field_=f, amps=amps)) for t in "qkv")
        # scores: sampled rows
        qbar = OS.block_means(qh, g.block)
        kbar = OS.block_means(kh, g.block)
        for r in rng.choice(nb, 8, replace=False):
            a, e = cand_np["row_ptr"][r], cand_np["row_ptr"][r + 1]
            cols = cand_np["col"][a:e]
            ref = OS.block_scores(qbar, kbar, r, cols)
            got = sc[h * cand["nnz"] + a: h * cand["nnz"] + e].astype(np.float64)
            scale = np.linalg.norm(qbar[r]) * np.linalg.norm(kbar[cols], axis=1) / math.sqrt(D)
            assert np.all(np.abs(got - ref) <= SCORE_REL * scale + 1e-7), (name, run, h, r)
        # selection: all rows of this head, from the GPU's scores
        kept = csr_rows(rp_np, col_np, h, nb)
        ambiguous += compare_selection(mode, value, cand_np, kept, sc, h, nb, cand["nnz"])
        # attention: sampled query blocks, every token
        o_h = o[0, h].float().cpu().numpy()
        lse_h = lse[0, h].cpu().numpy()
        lrp = np.concatenate([[0], np.cumsum([len(x) for x in kept])])
        lcol = np.concatenate(kept)
        sample = sorted(set([nb - 1] + rng.choice(nb, 5, replace=False).tolist()))
        res = OA.sparse_attention_rows(qh, kh, vh, g.block, lrp, lcol, rows=sample)
        errs = []
        for r, (toks, ob, lb) in res.items():
            err = np.abs(o_h[toks].astype(np.float64) - ob)
            assert err.max() <= O_MAX_ABS, (name, run, h, r, err.max())
            errs.append(err)
            assert np.abs(lse_h[toks] - lb).max() <= LSE_ABS, (name, run, h, r)
        assert np.concatenate(errs).mean() <= O_MEAN_ABS
    assert ambiguous == 0, f"{ambiguous} rows within {AMBIGUOUS_GAP} of the dynamic threshold"
