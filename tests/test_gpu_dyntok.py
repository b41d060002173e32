"""Paper-exact dynamic-threshold mode on the GPU (Eqs. 9-11 and 19: fused-head
proxy logits on candidate token pairs, per-frame-pair z-scores, tau thresholds
with the top-pair fallback, block aggregation) against the oracle.

The GPU forms the logits in fp32 and the oracle in fp64 from the same bf16
inputs, so a pair whose z-score lies within fp32 rounding of tau may fall on
either side.  The mask is monotone in tau, so every GPU row must lie between
the oracle's rows at tau + delta and tau - delta (delta = 1e-3 in z units, far
above the fp32 error of ~1e-5); rows where those two agree are thereby checked
exactly."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (WORKLOADS, Geometry, bf16_bits_to_f64, make_qkv_bf16,
                                                             random_qkv_bf16)
from gpu_util import cand_to_numpy, check_device_status, compare_attention, csr_rows, gpu_inputs
from oracle import attention as OA
from oracle import dynamic_tokens as DT
from oracle import geometry as OG

pytestmark = pytest.mark.gpu

DELTA = 1e-3
SMALL = [Geometry(4, 8, 8, 32, 0.5, 2.0), Geometry(5, 6, 7, 32, 0.7, 0.3),
         Geometry(4, 4, 16, 64, 0.5, 2.0, theta_c=0.1, theta_m=0.2), Geometry(6, 8, 8, 32, 0.4, 2.0, force_t=0),
         Geometry(7, 6, 16, 128, 0.4, 1.0)]


def _run(geom, bits, tau1, tau2, hf):
    q, k, _ = gpu_inputs(bits)
    cand = abi.dynrad_build_candidates(geom)
    rp, col, st = abi.dynrad_build_token_mask(q, k, geom, cand, tau1, tau2, hf=hf, stats=True)
    torch.cuda.synchronize()
    check_device_status()
    rp = rp.cpu().numpy().astype(np.int64)
    col = col.cpu().numpy().astype(np.int64)[: rp[-1]]
    return rp, col, st.cpu().numpy(), cand


def _check_rows(geom, gpu_rows, qf, kf, tau1, tau2, rows, label):
    lo = DT.dynamic_mask_rows(geom, qf, kf, tau1, tau2, rows, tau_shift=DELTA)
    hi = DT.dynamic_mask_rows(geom, qf, kf, tau1, tau2, rows, tau_shift=-DELTA)
    ambiguous = 0
    for r, g, a, b in zip(rows, gpu_rows, lo, hi):
        gs, as_, bs = set(g.tolist()), set(a.tolist()), set(b.tolist())
        assert as_ <= gs <= bs, (label, r, sorted(as_ - gs), sorted(gs - bs))
        ambiguous += as_ != bs
    return ambiguous


@pytest.mark.parametrize("gi", range(len(SMALL)))
@pytest.mark.parametrize("tau1,tau2,hf", [(0.5, 1.5, 2), (2.5, 0.0, 1), (-0.5, 50.0, 2)])
def test_small_geometries_against_the_oracle(gi, tau1, tau2, hf):
    geom = SMALL[gi]
    B, H, D = 2, 3, 64
    bits = random_qkv_bf16(17 + gi, B, H, geom.n_tokens, D, scale=1.0)
    rp, col, st, _ = _run(geom, bits, tau1, tau2, hf)
    F, nb = geom.frames, geom.n_blocks
    nt = geom.height * geom.width
    for b in range(B):
        qf = np.stack([bf16_bits_to_f64(bits["q"][b, h]) for h in range(hf)])
        kf = np.stack([bf16_bits_to_f64(bits["k"][b, h]) for h in range(hf)])
        for i in range(F):
            for j in range(F):
                t = abs(i - j)
                n, mu, sigma, _, _, _ = DT.frame_pair_stats(geom, qf, kf, i, j)
                if t < 2 or n == 0:
                    assert st[b, i * F + j, 2] == -math.inf
                    continue
                scale = max(1.0, abs(mu), sigma)
                assert abs(st[b, i * F + j, 0] - mu) <= 1e-5 * scale, (b, i, j)
                assert abs(st[b, i * F + j, 1] - sigma) <= 1e-5 * scale, (b, i, j)
        rows_gpu = []
        for h in range(H):       # every head of batch element b carries its mask
            rr = csr_rows(rp, col, b * H + h, nb)
            if h == 0:
                rows_gpu = rr
            else:
                assert all(np.array_equal(x, y) for x, y in zip(rr, rows_gpu))
        _check_rows(geom, rows_gpu, qf, kf, tau1, tau2, list(range(nb)), f"geom {gi} b {b}")


@pytest.mark.parametrize("D,hf", [(64, 3), (64, 4), (128, 1), (128, 3), (128, 4)])
def test_every_fused_width(D, hf):
    # the tensor-core tile kernel serves H_f * D <= 256, the warp-level MMA
    # kernel the wider (128, 3) and (128, 4); every instance against the oracle
    geom = SMALL[1]
    B, H = 1, 4
    tau1, tau2 = 0.5, 1.5
    bits = random_qkv_bf16(41 + D + hf, B, H, geom.n_tokens, D, scale=1.0)
    rp, col, st, _ = _run(geom, bits, tau1, tau2, hf)
    F, nb = geom.frames, geom.n_blocks
    qf = np.stack([bf16_bits_to_f64(bits["q"][0, h]) for h in range(hf)])
    kf = np.stack([bf16_bits_to_f64(bits["k"][0, h]) for h in range(hf)])
    for i in range(F):
        for j in range(F):
            if abs(i - j) < 2:
                continue
            n, mu, sigma, _, _, _ = DT.frame_pair_stats(geom, qf, kf, i, j)
            if n == 0:
                continue
            scale = max(1.0, abs(mu), sigma)
            assert abs(st[0, i * F + j, 0] - mu) <= 1e-5 * scale, (D, hf, i, j)
            assert abs(st[0, i * F + j, 1] - sigma) <= 1e-5 * scale, (D, hf, i, j)
    _check_rows(geom, csr_rows(rp, col, 0, nb), qf, kf, tau1, tau2, list(range(nb)), f"D {D} hf {hf}")


def test_very_low_thresholds_give_the_candidate_set():
    geom = SMALL[0]
    bits = random_qkv_bf16(5, 1, 2, geom.n_tokens, 64)
    rp, col, _, cand = _run(geom, bits, -1e30, -1e30, 2)
    c = cand_to_numpy(cand)
    nb = geom.n_blocks
    for h in range(2):
        rows = csr_rows(rp, col, h, nb)
        for r in range(nb):
            np.testing.assert_array_equal(rows[r], c["col"][c["row_ptr"][r]:c["row_ptr"][r + 1]])


def test_wan13b_geometry_sampled_rows_and_stats():
    wl = WORKLOADS["wan13b_480p"]
    geom = wl.geom
    bits = make_qkv_bf16(wl)
    tau1, tau2, hf = 1.0, 2.0, 2
    rp, col, st, _ = _run(geom, bits, tau1, tau2, hf)
    qf = np.stack([bf16_bits_to_f64(bits["q"][0, h]) for h in range(hf)])
    kf = np.stack([bf16_bits_to_f64(bits["k"][0, h]) for h in range(hf)])
    F, nb = geom.frames, geom.n_blocks
    rng = np.random.default_rng(7)
    for i, j in [(0, 2), (5, 20), (20, 0)] + [tuple(x) for x in rng.integers(0, F, (3, 2))]:
        if abs(i - j) < 2:
            continue
        n, mu, sigma, _, _, _ = DT.frame_pair_stats(geom, qf, kf, i, j)
        scale = max(1.0, abs(mu), sigma)
        assert abs(st[0, i * F + j, 0] - mu) <= 1e-5 * scale and abs(st[0, i * F + j, 1] - sigma) <= 1e-5 * scale
    rows = sorted({0, nb - 1} | set(rng.choice(nb, 2, replace=False).tolist()))
    gpu_rows = csr_rows(rp, col, 0, nb)
    _check_rows(geom, [gpu_rows[r] for r in rows], qf, kf, tau1, tau2, rows, "wan13b")


def test_attention_over_the_token_mask_tiny():
    wl = WORKLOADS["tiny"]
    bits = make_qkv_bf16(wl)
    q, k, v = gpu_inputs(bits)
    B, H, N, D = q.shape
    cand = abi.dynrad_build_candidates(wl.geom)
    rp, col, _ = abi.dynrad_build_token_mask(q, k, wl.geom, cand, 0.5, 1.0, hf=2)
    o, lse = abi.dynrad_sparse_attn(q, k, v, wl.geom.block, rp, col)
    torch.cuda.synchronize()
    check_device_status()
    rp_np = rp.cpu().numpy().astype(np.int64)
    col_np = col.cpu().numpy().astype(np.int64)[: rp_np[-1]]
    nb = wl.geom.n_blocks
    o_ref = np.zeros((B, H, N, D))
    lse_ref = np.zeros((B, H, N))
    for h in range(H):
        qh, kh, vh = (bf16_bits_to_f64(bits[t][0, h]) for t in "qkv")
        rows = csr_rows(rp_np, col_np, h, nb)
        lrp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
        o_ref[0, h], lse_ref[0, h] = OA.sparse_attention(qh, kh, vh, wl.geom.block, lrp, np.concatenate(rows))
    compare_attention(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "token-level dynamic")
