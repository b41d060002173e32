"""Pins of the attention backward oracle: torch autograd on the dense case (a
library routine for the special case), central finite differences on a sparse
mask, and the identity rowsum(dP * P) = rowsum(dO * O)."""
import math

import numpy as np
import torch

from oracle import attention as OA
from oracle import backward as OB


def _csr(keep):
    nb = keep.shape[0]
    rp = np.concatenate([[0], np.cumsum(keep.sum(axis=1))])
    col = np.concatenate([np.flatnonzero(keep[r]) for r in range(nb)])
    return rp, col


def test_dense_case_matches_torch_autograd():
    rng = np.random.default_rng(0)
    n, d, block = 40, 8, 8
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    nb = n // block
    rp, col = _csr(np.ones((nb, nb), dtype=bool))
    dq, dk, dv, o = OB.sparse_attention_backward(q, k, v, do, block, rp, col)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.softmax(tq @ tk.T / math.sqrt(d), dim=-1) @ tv
    (to * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_sparse_mask_finite_differences_and_forward_agreement():
    rng = np.random.default_rng(1)
    n, d, block = 30, 4, 8                       # ragged last block
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    nb = -(-n // block)
    keep = rng.random((nb, nb)) < 0.5
    keep[:, 0] = True
    keep[1, :] = False                            # a row with no kept block
    rp, col = _csr(keep)
    dq, dk, dv, o = OB.sparse_attention_backward(q, k, v, do, block, rp, col)
    o_fwd, _ = OA.sparse_attention(q, k, v, block, rp, col)
    np.testing.assert_allclose(o, o_fwd, atol=1e-12)
    assert np.all(o[8:16] == 0) and np.all(dq[8:16] == 0)

    def loss(qq, kk, vv):
        oo, _ = OA.sparse_attention(qq, kk, vv, block, rp, col)
        return float((oo * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for (i, j) in [(0, 0), (3, 2), (17, 1), (29, 3), (12, 0)]:
            xp, xm = x.copy(), x.copy()
            xp[i, j] += h
            xm[i, j] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - g[i, j]) < 1e-6, (name, i, j, fd, g[i, j])


def test_softmax_gradient_identity():
    rng = np.random.default_rng(2)
    n, d, block = 24, 6, 8
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    nb = n // block
    rp, col = _csr((rng.random((nb, nb)) < 0.6) | np.eye(nb, dtype=bool))
    mask = OA.token_mask(block, n, rp, col)
    p = OB.masked_softmax((q @ k.T) / math.sqrt(d), mask)
    o = p @ v
    dp = do @ v.T
    np.testing.assert_allclose((dp * p).sum(axis=1), (do * o).sum(axis=1), atol=1e-12)


def test_block_restricted_forms_match_the_full_backward():
    rng = np.random.default_rng(3)
    n, d, block = 45, 5, 8                        # ragged last block
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    nb = -(-n // block)
    keep = rng.random((nb, nb)) < 0.45
    keep[2, :] = False                            # a row with no kept block
    keep[:, 4] = False                            # a key block nobody keeps
    keep[0, 4] = True                             # ... except query block 0
    keep[:, 3] = False                            # a key block nobody keeps at all
    rp, col = _csr(keep)
    dq, dk, dv, _ = OB.sparse_attention_backward(q, k, v, do, block, rp, col, scale=0.7)
    for i in range(nb):
        rows, _, _, _, dq_i = OB.query_block_backward(q, k, v, do, block, col[rp[i]:rp[i + 1]], i, scale=0.7)
        np.testing.assert_allclose(dq_i, dq[rows], atol=1e-12)
    for j in range(nb):
        keys, dk_j, dv_j = OB.key_block_backward(q, k, v, do, block, rp, col, j, scale=0.7)
        np.testing.assert_allclose(dk_j, dk[keys], atol=1e-12)
        np.testing.assert_allclose(dv_j, dv[keys], atol=1e-12)
    assert np.all(dk[24:32] == 0) and np.all(dv[24:32] == 0)
