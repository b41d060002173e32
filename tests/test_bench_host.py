"""Host-side arithmetic of bench.py that the reported numbers rest on (no GPU)."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _random_csr(rng, bh, nb, density):
    rows = [np.flatnonzero((rng.random(nb) < density) | (np.arange(nb) == r % nb)) for r in range(bh * nb)]
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int64)
    return rp, np.concatenate(rows).astype(np.int64), rows


@pytest.mark.parametrize("block", [32, 64, 128])
def test_backward_tile_fill_by_enumeration(block):
    rng = np.random.default_rng(block)
    bh, nb = 3, 11
    rp, col, rows = _random_csr(rng, bh, nb, 0.3)
    r = 128 // block
    steps_per_member = max(1, block // 64)
    useful = len(col) * block * block
    want = {}
    # dQ side: tiles of r query blocks stream the union of their kept lists
    steps = 0
    for h in range(bh):
        for t0 in range(0, nb, r):
            union = set()
            for i in range(t0, min(t0 + r, nb)):
                union |= set(rows[h * nb + i].tolist())
            steps += len(union) * steps_per_member
    want["dq"] = useful / (steps * 128 * 64)
    # dK / dV side: tiles of r key blocks stream the query blocks that keep any of them
    steps = 0
    for h in range(bh):
        for t0 in range(0, nb, r):
            members = {i for i in range(nb) if any(j in set(rows[h * nb + i].tolist()) for j in range(t0, t0 + r))}
            steps += len(members) * steps_per_member
    want["dkv"] = useful / (steps * 128 * 64)
    got = bench.backward_tile_fill(rp, col, bh, nb, block)
    for side in ("dq", "dkv"):
        assert got[side] == pytest.approx(want[side], abs=1e-4), side


def test_kept_flops_counts_valid_tokens():
    # 2 blocks of 64 over n = 100 tokens: block 1 holds 36 tokens
    rp = np.array([0, 2, 3])
    col = np.array([0, 1, 1])
    d = 128
    want = 4 * d * (64 * 64 + 64 * 36 + 36 * 36)
    assert bench.kept_flops(rp, col, 100, 64, 1, d) == pytest.approx(want)
