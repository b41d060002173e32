"""Backward of stage 3 on the GPU (dQ, dK, dV under the same kept-block CSR)
against the float64 oracle on the same bf16 inputs.

Tolerances.  The GPU rounds P and dS to bf16 as tensor-core operands (relative
2^-9 each), takes D_r from the bf16 forward output O, and rounds dQ, dK, dV to
bf16; the oracle is exact float64.  The errors are independent per term and
mostly cancel in the sums, so per tensor the Frobenius error stays within 1e-2
of the reference's norm and the largest element error within 2e-2 of its
largest magnitude.  Outputs the oracle makes exactly zero (keys no query block
keeps, rows with no kept block, padded rows) must be exactly zero."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (WORKLOADS, bf16_bits_to_f64, make_qkv_bf16,
                                                             random_qkv_bf16, round_to_bf16_bits)
from gpu_util import bits_to_tensor, check_device_status, csr_rows, full_csr, gpu_inputs
from oracle import backward as OB

pytestmark = pytest.mark.gpu

FROB_REL = 1e-2
MAX_REL = 2e-2


def _dout_bits(seed, B, H, n, D):
    return random_qkv_bf16(seed, B, H, n, D)["q"]


def _gpu(bits, do_bits, block, rp, col, scale=0.0):
    q, k, v = gpu_inputs(bits)
    do = bits_to_tensor(do_bits)
    rpt = torch.from_numpy(rp.astype(np.int32)).cuda()
    colt = torch.from_numpy(col.astype(np.int32) if len(col) else np.zeros(1, np.int32)).cuda()
    o, lse = abi.dynrad_sparse_attn(q, k, v, block, rpt, colt, scale)
    dq, dk, dv = abi.dynrad_attn_backward(q, k, v, o, lse, do, block, rpt, colt, scale)
    torch.cuda.synchronize()
    check_device_status()
    return tuple(t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))


def _oracle(bits, do_bits, block, rp, col, B, H, scale=None):
    n, d = bits["q"].shape[2], bits["q"].shape[3]
    nb = -(-n // block)
    out = [np.zeros((B, H, n, d)) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            q, k, v = (bf16_bits_to_f64(bits[t][b, h]) for t in "qkv")
            do = bf16_bits_to_f64(do_bits[b, h])
            rows = csr_rows(rp, col, b * H + h, nb)
            lrp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
            lcol = np.concatenate(rows) if rows else np.zeros(0, np.int64)
            g = OB.sparse_attention_backward(q, k, v, do, block, lrp, lcol, scale)
            for t in range(3):
                out[t][b, h] = g[t]
    return out


def _compare(got, ref, what, names=("dQ", "dK", "dV")):
    for name, g, r in zip(names, got, ref):
        zero = r == 0
        assert np.all(g[zero] == 0), f"{what} {name}: nonzero where the oracle is exactly zero"
        nr = np.linalg.norm(r)
        if nr == 0:
            continue
        fro = np.linalg.norm(g - r) / nr
        mx = np.abs(g - r).max() / np.abs(r).max()
        assert fro <= FROB_REL, f"{what} {name}: Frobenius rel err {fro:.2e}"
        assert mx <= MAX_REL, f"{what} {name}: max err / max |ref| {mx:.2e}"


def _random_csr(rng, BH, nb, density, empty_rows=(), dead_cols=()):
    rows = []
    for _ in range(BH):
        keep = rng.random((nb, nb)) < density
        keep |= np.eye(nb, dtype=bool)
        for c in dead_cols:
            keep[:, c] = False
        for r in empty_rows:
            keep[r, :] = False
        rows += [np.flatnonzero(keep[r]) for r in range(nb)]
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
    return rp, np.concatenate(rows)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("block", [32, 64, 128])
@pytest.mark.parametrize("n", [777, 1024])
def test_random_csr_ragged(D, block, n):
    B, H = 1, 2
    nb = -(-n // block)
    rng = np.random.default_rng(D * 7 + block + n)
    bits = random_qkv_bf16(D + block + n, B, H, n, D)
    do = _dout_bits(5 + n, B, H, n, D)
    rp, col = _random_csr(rng, B * H, nb, 0.4, empty_rows=(1,), dead_cols=(nb - 2,))
    got = _gpu(bits, do, block, rp, col)
    ref = _oracle(bits, do, block, rp, col, B, H)
    _compare(got, ref, f"D={D} B_s={block} N={n}")


@pytest.mark.parametrize("D,block", [(64, 64), (128, 128)])
def test_dense_csr_matches_torch_autograd(D, block):
    B, H, n = 2, 1, 600
    nb = -(-n // block)
    bits = random_qkv_bf16(31 + D, B, H, n, D)
    do_bits = _dout_bits(32 + D, B, H, n, D)
    rp, col = full_csr(nb, B * H)
    got = _gpu(bits, do_bits, block, rp, col)
    q, k, v = (torch.from_numpy(bf16_bits_to_f64(bits[t])).requires_grad_() for t in "qkv")
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    (o * torch.from_numpy(bf16_bits_to_f64(do_bits))).sum().backward()
    _compare(got, [t.grad.numpy() for t in (q, k, v)], "dense vs autograd")


def test_explicit_scale_and_large_logits():
    B, H, n, D, block = 1, 2, 640, 128, 64
    nb = n // block
    bits = random_qkv_bf16(41, B, H, n, D, scale=3.0)      # logits of a few tens
    do = _dout_bits(42, B, H, n, D)
    rp, col = _random_csr(np.random.default_rng(43), B * H, nb, 0.5)
    got = _gpu(bits, do, block, rp, col, scale=0.2)
    ref = _oracle(bits, do, block, rp, col, B, H, scale=0.2)
    _compare(got, ref, "scale 0.2, large logits")


def test_empty_mask_gives_zero_gradients():
    B, H, n, D, block = 1, 1, 300, 64, 64
    nb = -(-n // block)
    bits = random_qkv_bf16(51, B, H, n, D)
    do = _dout_bits(52, B, H, n, D)
    rp = np.zeros(B * H * nb + 1, np.int64)
    got = _gpu(bits, do, block, rp, np.zeros(0, np.int64))
    for g in got:
        assert np.all(g == 0)


def test_unsupported_block_and_capacity():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 64, device="cuda")
    rp = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    col = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.DynradError) as e:
        abi.dynrad_attn_backward(q, q, q, q, lse, q, 48, rp, col)
    assert e.value.status == abi.DYNRAD_ERR_UNSUPPORTED
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(abi.DynradError) as e:
        abi.dynrad_attn_backward(q, q, q, q, lse, q, 64, rp, col, workspace=ws)
    assert e.value.status == abi.DYNRAD_ERR_CAPACITY


@pytest.mark.parametrize("name", ["wan14b_720p", "hunyuan_720p"])
def test_full_size_sampled(name):
    """All heads of the layer in one call at the workload's N, D and block,
    over a seeded random CSR (15% density plus the diagonal; one key block per
    head kept by only a few query blocks, so that its dK / dV rows are cheap
    for the oracle).  Checked against the oracle: dQ of sampled query blocks
    and dK / dV of that key block, in the first and last head; and in every
    head the identity sum_q q.dQ_q = sum_k k.dK_k (both equal scale sum dS * QK^T)."""
    wl = WORKLOADS[name]
    g = wl.geom
    B, H, N, D, block = 1, wl.heads, g.n_tokens, wl.head_dim, g.block
    nb = g.n_blocks
    rng = np.random.default_rng(61)
    gen = np.random.Generator(np.random.PCG64(62))
    bits = make_qkv_bf16(wl)
    do_bits = round_to_bf16_bits(gen.standard_normal((B, H, N, D), dtype=np.float32))
    rows, j_sparse = [], []
    for _ in range(B * H):
        keep = (rng.random((nb, nb)) < 0.15) | np.eye(nb, dtype=bool)
        j = int(rng.integers(1, nb - 1))
        keep[:, j] = False
        keep[rng.choice(nb, 6, replace=False), j] = True
        keep[j, j] = True
        j_sparse.append(j)
        rows += [np.flatnonzero(keep[r]) for r in range(nb)]
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
    col = np.concatenate(rows)
    q, k, v = gpu_inputs(bits)
    do = bits_to_tensor(do_bits)
    rpt = torch.from_numpy(rp.astype(np.int32)).cuda()
    colt = torch.from_numpy(col.astype(np.int32)).cuda()
    o, lse = abi.dynrad_sparse_attn(q, k, v, block, rpt, colt)
    dq, dk, dv = abi.dynrad_attn_backward(q, k, v, o, lse, do, block, rpt, colt)
    torch.cuda.synchronize()
    check_device_status()
    scale = 1.0 / math.sqrt(D)

    # identity on every head (GPU outputs only, fp64 sums)
    s_q = (q.double() * dq.double()).sum(dim=(2, 3)).flatten().cpu().numpy()
    s_k = (k.double() * dk.double()).sum(dim=(2, 3)).flatten().cpu().numpy()
    mag = (q.double() * dq.double()).abs().sum(dim=(2, 3)).flatten().cpu().numpy()
    assert np.all(np.abs(s_q - s_k) <= 1e-2 * mag), np.abs(s_q - s_k).max()

    for h in sorted({0, H - 1}):
        qh, kh, vh = (bf16_bits_to_f64(bits[t][0, h]) for t in "qkv")
        doh = bf16_bits_to_f64(do_bits[0, h])
        hrows = csr_rows(rp, col, h, nb)
        lrp = np.concatenate([[0], np.cumsum([len(x) for x in hrows])])
        lcol = np.concatenate(hrows)
        dq_h = dq[0, h].float().cpu().numpy()
        for i in sorted({0, nb - 1} | set(rng.choice(nb, 2, replace=False).tolist())):
            r, _, _, _, dq_ref = OB.query_block_backward(qh, kh, vh, doh, block, hrows[i], i)
            _compare([dq_h[r]], [dq_ref], f"{name} head {h} block {i}", names=("dQ",))
        keys, dk_ref, dv_ref = OB.key_block_backward(qh, kh, vh, doh, block, lrp, lcol, j_sparse[h])
        _compare([dk[0, h].float().cpu().numpy()[keys], dv[0, h].float().cpu().numpy()[keys]], [dk_ref, dv_ref],
                 f"{name} head {h} block {j_sparse[h]}", names=("dK", "dV"))


@pytest.mark.parametrize("n", [40, 100])
@pytest.mark.parametrize("D,block", [(128, 64), (64, 128), (64, 32)])
def test_sequences_shorter_than_one_tile(n, D, block):
    B, H = 1, 2
    nb = -(-n // block)
    bits = random_qkv_bf16(200 + n + D, B, H, n, D)
    do = _dout_bits(201 + n, B, H, n, D)
    rp, col = full_csr(nb, B * H)
    got = _gpu(bits, do, block, rp, col)
    ref = _oracle(bits, do, block, rp, col, B, H)
    _compare(got, ref, f"N={n} D={D} B_s={block}")


@pytest.mark.parametrize("mode,value", [("static", 0.25), ("dynamic", 0.8)])
def test_tiny_workload_selected_mask(mode, value):
    """Candidates, selection, attention and its gradient through the library on
    the tiny workload (block 32); the oracle gets the same bf16 inputs and the
    kept CSR."""
    wl = WORKLOADS["tiny"]
    g = wl.geom
    bits = make_qkv_bf16(wl)
    B, H, N, D = bits["q"].shape
    do_bits = _dout_bits(301, B, H, N, D)
    q, k, _ = gpu_inputs(bits)
    cand = abi.dynrad_build_candidates(g)
    rp, col, _ = abi.dynrad_select_blocks(q, k, g, cand, mode, value, scores=True)
    torch.cuda.synchronize()
    rp_np = rp.cpu().numpy().astype(np.int64)
    col_np = col.cpu().numpy().astype(np.int64)[: rp_np[-1]]
    got = _gpu(bits, do_bits, g.block, rp_np, col_np)
    ref = _oracle(bits, do_bits, g.block, rp_np, col_np, B, H)
    _compare(got, ref, f"tiny {mode} {value}")
