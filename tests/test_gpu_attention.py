"""Stage 3 on the GPU vs the oracle: O and LSE of the block-sparse attention,
element by element, on the same bf16 inputs and the same CSR."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (
    WORKLOADS, Geometry, bf16_bits_to_f64, make_qkv_bf16, random_qkv_bf16)
from gpu_util import check_device_status, compare_attention, csr_rows, full_csr, gpu_inputs
from oracle import attention as OA

pytestmark = pytest.mark.gpu


def _attn_gpu(bits, block, rp, col, scale=0.0):
    q, k, v = gpu_inputs(bits)
    rpt = torch.from_numpy(rp.astype(np.int32)).cuda()
    colt = torch.from_numpy(col.astype(np.int32) if len(col) else np.zeros(1, np.int32)).cuda()
    o, lse = abi.dynrad_sparse_attn(q, k, v, block, rpt, colt, scale)
    torch.cuda.synchronize()
    check_device_status()
    return (o.float().cpu().numpy(), lse.cpu().numpy())


def _oracle_all(bits, block, rp, col, B, H, scale=None):
    n, d = bits["q"].shape[2], bits["q"].shape[3]
    nb = -(-n // block)
    o = np.zeros((B, H, n, d))
    lse = np.zeros((B, H, n))
    for b in range(B):
        for h in range(H):
            bh = b * H + h
            q, k, v = (bf16_bits_to_f64(bits[t][b, h]) for t in "qkv")
            rows = csr_rows(rp, col, bh, nb)
            lrp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
            lcol = np.concatenate(rows) if rows else np.zeros(0, np.int64)
            o[b, h], lse[b, h] = OA.sparse_attention(q, k, v, block, lrp, lcol, scale=scale)
    return o, lse


def _random_csr(rng, B, H, nb, density):
    rows = []
    for _ in range(B * H):
        for r in range(nb):
            m = rng.random(nb) < density
            m[r] = True
            rows.append(np.flatnonzero(m))
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
    return rp, np.concatenate(rows)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("block", [32, 64, 128])
@pytest.mark.parametrize("n", [1000, 777])
def test_random_csr_ragged(D, block, n):
    B, H = 1, 2
    nb = -(-n // block)
    rng = np.random.default_rng(D * 1000 + block + n)
    bits = random_qkv_bf16(D + block + n, B, H, n, D, scale=1.5)
    rp, col = _random_csr(rng, B, H, nb, 0.4)
    o, lse = _attn_gpu(bits, block, rp, col)
    o_ref, lse_ref = _oracle_all(bits, block, rp, col, B, H)
    compare_attention(o, lse, o_ref, lse_ref, f"D={D} B_s={block} N={n}")


@pytest.mark.parametrize("D,block", [(64, 32), (128, 64), (128, 128)])
def test_dense_csr_matches_sdpa(D, block):
    B, H, n = 1, 2, 1536 + 40
    nb = -(-n // block)
    bits = random_qkv_bf16(7 + D + block, B, H, n, D)
    rp, col = full_csr(nb, B * H)
    o, lse = _attn_gpu(bits, block, rp, col)
    q, k, v = (torch.from_numpy(bf16_bits_to_f64(bits[t])) for t in "qkv")
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    lse_ref = torch.logsumexp((q @ k.transpose(-1, -2)) / math.sqrt(D), dim=-1).numpy()
    compare_attention(o, lse, ref, lse_ref, "dense")


def test_empty_rows_give_zero_and_minus_inf():
    B, H, n, D, block = 1, 1, 640, 128, 64
    nb = n // block
    bits = random_qkv_bf16(3, B, H, n, D)
    rows = [np.array([r]) if r % 3 else np.zeros(0, np.int64) for r in range(nb)]
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
    col = np.concatenate(rows)
    o, lse = _attn_gpu(bits, block, rp, col)
    for r in range(nb):
        sl = slice(r * block, (r + 1) * block)
        if r % 3 == 0:
            assert np.all(o[0, 0, sl] == 0) and np.all(np.isneginf(lse[0, 0, sl]))
    o_ref, lse_ref = _oracle_all(bits, block, rp, col, B, H)
    compare_attention(o, lse, o_ref, lse_ref, "empty rows")


def test_explicit_scale():
    B, H, n, D, block = 1, 1, 512, 64, 64
    nb = n // block
    bits = random_qkv_bf16(11, B, H, n, D)
    rp, col = full_csr(nb, 1)
    o, lse = _attn_gpu(bits, block, rp, col, scale=0.05)
    o_ref, lse_ref = _oracle_all(bits, block, rp, col, B, H, scale=0.05)
    compare_attention(o, lse, o_ref, lse_ref, "scale")


def test_large_logits_rescale_path():
    # strongly varying logits force the lazy O rescale (row max grows > 2^8)
    B, H, n, D, block = 1, 2, 1024, 128, 64
    nb = n // block
    rng = np.random.default_rng(5)
    bits = random_qkv_bf16(13, B, H, n, D, scale=1.0)
    from block_sparse_attention_candidate_b200.workloads import round_to_bf16_bits
    ramp = np.linspace(0.2, 6.0, n, dtype=np.float32)[:, None]
    kf = rng.standard_normal((B, H, n, D), dtype=np.float32) * ramp
    bits["k"] = round_to_bf16_bits(kf)
    bits["q"] = round_to_bf16_bits(rng.standard_normal((B, H, n, D), dtype=np.float32) * 3)
    rp, col = full_csr(nb, B * H)
    o, lse = _attn_gpu(bits, block, rp, col)
    o_ref, lse_ref = _oracle_all(bits, block, rp, col, B, H)
    compare_attention(o, lse, o_ref, lse_ref, "rescale")


@pytest.mark.parametrize("mode,value", [("static", 0.25), ("dynamic", 0.8)])
def test_tiny_end_to_end(mode, value):
    wl = WORKLOADS["tiny"]
    bits = make_qkv_bf16(wl)
    q, k, v = gpu_inputs(bits)
    cand = abi.dynrad_build_candidates(wl.geom)
    rp, col, _ = abi.dynrad_select_blocks(q, k, wl.geom, cand, mode, value)
    o, lse = abi.dynrad_sparse_attn(q, k, v, wl.geom.block, rp, col)
    torch.cuda.synchronize()
    check_device_status()
    rp_np = rp.cpu().numpy().astype(np.int64)
    col_np = col.cpu().numpy().astype(np.int64)[: rp_np[-1]]
    o_ref, lse_ref = _oracle_all(bits, wl.geom.block, rp_np, col_np, 1, wl.heads)
    compare_attention(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"tiny {mode}")


def test_fma_pipe_exp2_against_cuda_exp2f():
    # the softmax computes one exponential in four with the FMA-pipe
    # approximation; check it against CUDA's exp2f over the range the kernel
    # feeds it (running-max-shifted logits: x <= 8 with lazy rescale)
    x = torch.cat([torch.linspace(-124.0, 8.0, 2_000_001), torch.tensor([0.0, -0.5, 0.5, 7.999, -1e-7])])
    x = x.float().cuda()
    poly, ref = abi.dynrad_debug_exp2(x)
    torch.cuda.synchronize()
    rel = ((poly.double() - ref.double()) / ref.double()).abs()
    assert float(rel.max()) < 8e-5
    # far below the range the result is tiny and positive (no inf / nan)
    low = torch.tensor([-1000.0, -200.0, -126.0], device="cuda")
    pl, _ = abi.dynrad_debug_exp2(low)
    assert bool(torch.isfinite(pl).all()) and float(pl.max()) < 1e-37


@pytest.mark.parametrize("n", [1, 40, 100])
@pytest.mark.parametrize("D,block", [(64, 32), (128, 64), (64, 128)])
def test_sequences_shorter_than_one_tile(n, D, block):
    # fewer tokens than one 128-row query tile (and than one block for n < block):
    # the tensor maps' boxes run past the sequence and read zeros there
    B, H = 1, 2
    nb = -(-n // block)
    bits = random_qkv_bf16(100 + n + D + block, B, H, n, D)
    rp, col = full_csr(nb, B * H)
    o, lse = _attn_gpu(bits, block, rp, col)
    o_ref, lse_ref = _oracle_all(bits, block, rp, col, B, H)
    compare_attention(o, lse, o_ref, lse_ref, f"N={n}")
