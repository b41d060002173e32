"""Paper-exact static-ratio mode on the GPU (Eq. 8 seeded token-pair sampling,
block aggregation) against the oracle: per-frame-pair thresholds T(i, j) and
block masks bit for bit, on small geometries in full and on the workloads'
geometries by sampled frame pairs and rows; and the attention over the mask."""
import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, Geometry, make_qkv_bf16
from gpu_util import cand_to_numpy, check_device_status, compare_attention, gpu_inputs
from oracle import attention as OA
from oracle import geometry as OG
from oracle import sampling as OSm
from block_sparse_attention_candidate_b200.workloads import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

SMALL = [Geometry(4, 16, 16, 32, 0.5, 2.0), Geometry(5, 3, 5, 32, 0.7, 0.3),
         Geometry(6, 8, 8, 32, 0.4, 0.1), Geometry(4, 4, 16, 64, 0.5, 2.0, theta_c=0.1, theta_m=0.2),
         Geometry(7, 6, 7, 32, 1.0, 2.0, force_t=0), Geometry(7, 6, 16, 128, 0.4, 1.0)]


def _gpu_mask(geom, rho1, rho2, seed, replicas=1):
    cand = abi.dynrad_build_candidates(geom)
    rp, col, thr = abi.dynrad_build_sampled_mask(geom, cand, rho1, rho2, seed, replicas=replicas, thresholds=True)
    torch.cuda.synchronize()
    check_device_status()
    rp = rp.cpu().numpy().astype(np.int64)
    col = col.cpu().numpy().astype(np.int64)[: rp[-1]]
    thr = thr.cpu().numpy().view(np.uint64)
    return rp, col, thr, cand


@pytest.mark.parametrize("gi", range(len(SMALL)))
@pytest.mark.parametrize("rho1,rho2,seed", [(0.3, 0.1, 7), (0.8, 0.5, 12345), (1.0, 1.0, 1)])
def test_small_geometries_bit_exact(gi, rho1, rho2, seed):
    geom = SMALL[gi]
    rp, col, thr, _ = _gpu_mask(geom, rho1, rho2, seed)
    F = geom.frames
    for i in range(F):
        for j in range(F):
            _, _, T = OSm.frame_pair_threshold(geom, i, j, rho1, rho2, seed)
            want = np.uint64(2 ** 64 - 1) if T is None else np.uint64(T)
            assert thr[i * F + j] == want, (i, j)
    ref = OSm.sampled_mask_csr(geom, rho1, rho2, seed)
    np.testing.assert_array_equal(rp, ref["row_ptr"])
    np.testing.assert_array_equal(col, ref["col"])


def test_full_retention_is_the_candidate_set_and_replicas_repeat():
    geom = WORKLOADS["wan13b_480p"].geom
    rp, col, _, cand = _gpu_mask(geom, 1.0, 1.0, 3, replicas=3)
    c = cand_to_numpy(cand)
    nb, nnz = geom.n_blocks, c["row_ptr"][-1]
    assert rp[-1] == 3 * nnz
    for r in range(3):
        np.testing.assert_array_equal(rp[r * nb:(r + 1) * nb + 1] - r * nnz, c["row_ptr"])
        np.testing.assert_array_equal(col[r * nnz:(r + 1) * nnz], c["col"])


@pytest.mark.parametrize("name,rho1,rho2", [("wan13b_480p", 0.3, 0.1), ("wan14b_720p", 0.5, 0.2),
                                            ("hunyuan_720p", 0.3, 0.1)])
def test_workload_geometry_sampled(name, rho1, rho2):
    geom = WORKLOADS[name].geom
    seed = 2026
    rp, col, thr, cand = _gpu_mask(geom, rho1, rho2, seed)
    F = geom.frames
    rng = np.random.default_rng(len(name))
    # thresholds of sampled frame pairs (both near- and far-field distances)
    pairs = {(0, 2), (F - 1, 0), (3, 9)} | {tuple(x) for x in rng.integers(0, F, (6, 2))}
    thr_ref = {}
    for i, j in sorted(pairs):
        _, _, T = OSm.frame_pair_threshold(geom, i, j, rho1, rho2, seed)
        want = np.uint64(2 ** 64 - 1) if T is None else np.uint64(T)
        assert thr[i * F + j] == want, (name, i, j)
    # rows: the oracle restricted to each row's query tokens
    nb = geom.n_blocks
    rows = sorted({0, nb - 1} | set(rng.choice(nb, 3, replace=False).tolist()))
    for r, want in zip(rows, OSm.sampled_mask_rows(geom, rho1, rho2, seed, rows)):
        np.testing.assert_array_equal(col[rp[r]:rp[r + 1]], want, err_msg=f"{name} row {r}")
    # a subset of the candidate set, forced ranges included
    c = cand_to_numpy(cand)
    for r in rows:
        got = set(col[rp[r]:rp[r + 1]].tolist())
        assert got <= set(c["col"][c["row_ptr"][r]:c["row_ptr"][r + 1]].tolist())
        assert set(range(c["forced_lo"][r], c["forced_hi"][r] + 1)) <= got


def test_attention_over_the_sampled_mask_tiny():
    wl = WORKLOADS["tiny"]
    bits = make_qkv_bf16(wl)
    q, k, v = gpu_inputs(bits)
    B, H, N, D = q.shape
    cand = abi.dynrad_build_candidates(wl.geom)
    rp, col, _ = abi.dynrad_build_sampled_mask(wl.geom, cand, 0.3, 0.1, 99, replicas=B * H)
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
        lrp = rp_np[h * nb:(h + 1) * nb + 1] - rp_np[h * nb]
        lcol = col_np[rp_np[h * nb]:rp_np[(h + 1) * nb]]
        o_ref[0, h], lse_ref[0, h] = OA.sparse_attention(qh, kh, vh, wl.geom.block, lrp, lcol)
    compare_attention(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "sampled static")


def _ws_sizes(geom, cand):
    import ctypes
    L = abi.lib()
    g = abi.make_geom(geom)
    least = int(L.dynrad_sampled_mask_workspace_min_bytes(ctypes.byref(g), cand["nnz"]))
    full = int(L.dynrad_sampled_mask_workspace_bytes(ctypes.byref(g), cand["nnz"]))
    assert 0 < least < full
    return least, full


@pytest.mark.parametrize("name", ["small0", "small3", "wan13b_480p"])
def test_pool_size_does_not_change_the_result(name):
    # no pool (every frame pair recomputes its keys in each radix pass), half a
    # pool (some pooled, some not) and the full pool give the same T and mask
    geom = SMALL[int(name[5:])] if name.startswith("small") else WORKLOADS[name].geom
    rho1, rho2, seed = 0.3, 0.1, 77
    cand = abi.dynrad_build_candidates(geom)
    least, full = _ws_sizes(geom, cand)
    outs = []
    for ws in (least, least + (full - least) // 2, full):
        rp, col, thr = abi.dynrad_build_sampled_mask(geom, cand, rho1, rho2, seed, thresholds=True,
                                                     workspace_bytes=ws)
        torch.cuda.synchronize()
        check_device_status()
        rp = rp.cpu().numpy().astype(np.int64)
        outs.append((rp, col.cpu().numpy().astype(np.int64)[: rp[-1]], thr.cpu().numpy().view(np.uint64)))
    for rp, col, thr in outs[:2]:
        np.testing.assert_array_equal(thr, outs[2][2])
        np.testing.assert_array_equal(rp, outs[2][0])
        np.testing.assert_array_equal(col, outs[2][1])
    if name.startswith("small"):
        F = geom.frames
        for i in range(F):
            for j in range(F):
                _, _, T = OSm.frame_pair_threshold(geom, i, j, rho1, rho2, seed)
                want = np.uint64(2 ** 64 - 1) if T is None else np.uint64(T)
                assert outs[0][2][i * F + j] == want, (i, j)
    else:
        F = geom.frames
        for i, j in [(0, 2), (F - 1, 0), (5, 17)]:
            _, _, T = OSm.frame_pair_threshold(geom, i, j, rho1, rho2, seed)
            want = np.uint64(2 ** 64 - 1) if T is None else np.uint64(T)
            assert outs[0][2][i * F + j] == want, (i, j)
