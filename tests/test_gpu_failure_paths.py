"""The attention kernel's own failure paths on the GPU, made to fire without a
fault: (a) a CSR whose rows hold out-of-range, repeated and descending block
indices -- the producer skips them, reads nothing outside the rows' ranges and
records DYNRAD_ERR_DEVICE, and the output is the attention over the entries its
walk keeps; (b) a test-only wait on a barrier nothing completes, under a short limit,
runs out -- the CTA unwinds (copies and tensor-core products in flight finish, tensor memory is
freed), the status reads DYNRAD_ERR_DEVICE, and the next normal call is exact."""
import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import random_qkv_bf16
from gpu_util import check_device_status, compare_attention, full_csr, gpu_inputs
from test_gpu_attention import _oracle_all

pytestmark = pytest.mark.gpu


def walk_kept(row, nb):
    """The entries the kernel's list walk keeps: in [0, nb) and strictly above
    the last kept entry; everything else is skipped (and flagged)."""
    kept, last = [], -1
    for c in row:
        if 0 <= c < nb and c > last:
            kept.append(int(c))
            last = int(c)
    return np.array(kept, dtype=np.int64)


def _run(bits, block, rp, col):
    q, k, v = gpu_inputs(bits)
    rpt = torch.from_numpy(rp.astype(np.int32)).cuda()
    colt = torch.from_numpy(col.astype(np.int32)).cuda()
    o, lse = abi.dynrad_sparse_attn(q, k, v, block, rpt, colt)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("block", [32, 64, 128])
def test_malformed_column_indices_are_skipped_and_flagged(block):
    B, H, n, D = 1, 2, 1500, 128
    nb = -(-n // block)
    rng = np.random.default_rng(block)
    bits = random_qkv_bf16(50 + block, B, H, n, D)
    rows = []
    for r in range(B * H * nb):
        good = np.flatnonzero((rng.random(nb) < 0.4) | (np.arange(nb) == r % nb))
        bad = list(good)
        # one malformed pattern per row, cycling: below range, above range,
        # a repeat, a descending pair, all together
        kind = r % 5
        if kind in (0, 4):
            bad.insert(rng.integers(0, len(bad) + 1), -1 - int(rng.integers(0, 5)))
        if kind in (1, 4):
            bad.insert(rng.integers(0, len(bad) + 1), nb + int(rng.integers(0, 3)))
        if kind in (2, 4):
            i = int(rng.integers(0, len(bad)))
            bad.insert(i, bad[i])
        if kind in (3, 4) and len(good) > 1:
            i = int(rng.integers(1, len(bad)))
            bad.insert(i, int(rng.integers(0, max(1, bad[i - 1]))) if bad[i - 1] > 0 else 0)
        rows.append(np.array(bad, dtype=np.int64))
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])])
    col = np.concatenate(rows)
    abi.dynrad_device_status(clear=True)
    o, lse = _run(bits, block, rp, col)
    assert abi.dynrad_device_status(clear=True) == abi.DYNRAD_ERR_DEVICE
    kept = [walk_kept(x, nb) for x in rows]
    krp = np.concatenate([[0], np.cumsum([len(x) for x in kept])])
    kcol = np.concatenate(kept)
    o_ref, lse_ref = _oracle_all(bits, block, krp, kcol, B, H)
    compare_attention(o, lse, o_ref, lse_ref, f"malformed CSR, block {block}")


def test_wait_that_runs_out_unwinds_and_the_next_call_is_exact():
    # every CTA's MMA warp waits, at its second step, for a barrier nothing
    # completes, under a 20 us limit: with K / V copies and tensor-core
    # products of the first steps in flight, the wait runs out and the CTA
    # unwinds
    B, H, n, D, block = 1, 4, 16384, 128, 64
    nb = n // block
    big = random_qkv_bf16(77, B, H, n, D)
    rp, col = full_csr(nb, B * H)
    check_device_status()
    try:
        abi.dynrad_debug_attn_stall(20_000, 1)
        _run(big, block, rp, col)
        status = abi.dynrad_device_status(clear=True)
    finally:
        abi.dynrad_debug_attn_stall(0, -1)
    assert status == abi.DYNRAD_ERR_DEVICE
    # the context is usable and the kernel exact again
    o_big, _ = _run(big, block, rp, col)
    check_device_status()
    assert np.isfinite(o_big).all()
    small = random_qkv_bf16(78, 1, 2, 1000, D)
    snb = -(-1000 // block)
    srp, scol = full_csr(snb, 2)
    o, lse = _run(small, block, srp, scol)
    check_device_status()
    o_ref, lse_ref = _oracle_all(small, block, srp, scol, 1, 2)
    compare_attention(o, lse, o_ref, lse_ref, "after an unwound launch")


def test_stall_hook_rejects_bad_step():
    with pytest.raises(abi.DynradError):
        abi.dynrad_debug_attn_stall(0, -2)
