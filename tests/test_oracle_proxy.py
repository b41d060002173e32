"""Pins of the proxy task (DynamicRad Appendix C.2 Eq. 20 features, C.4 Eq. 22
objective), of the log-sum-exp identity the GPU objective uses, and of the
host TPE optimizer."""
import math

import numpy as np

from block_sparse_attention_candidate_b200 import proxy as P
from block_sparse_attention_candidate_b200.workloads import ar_features
from oracle import proxy as OP


def test_ar_features_are_stationary_with_the_eq20_correlation():
    frames, nt, d = 6, 400, 32
    for delta in (0.02, 0.15, 0.40):
        h = ar_features(3, frames, nt, d, delta).reshape(frames, nt, d).astype(np.float64)
        for t in range(frames):
            assert abs(h[t].var() - 1.0) < 0.03                      # every h_t ~ N(0, I)
        for k in (1, 3):
            corr = (h[:-k] * h[k:]).mean()
            want = (1.0 - delta * delta) ** (k / 2.0)                # E[h_t . h_{t+k}] / D
            assert abs(corr - want) < 0.02, (delta, k, corr, want)


def test_full_mask_has_zero_error_and_the_full_penalty():
    h = np.random.default_rng(0).standard_normal((64, 8))
    nb = 4
    rp = np.arange(nb + 1) * nb
    col = np.tile(np.arange(nb), nb)
    loss, nmse, s = OP.objective(h, 16, rp, col)
    assert nmse < 1e-28 and s == 0.0 and abs(loss - 10.0 * 0.8) < 1e-12


def test_diagonal_mask_error_brute_force():
    rng = np.random.default_rng(1)
    h = rng.standard_normal((48, 6))
    block, nb = 16, 3
    rp, col = np.arange(nb + 1), np.arange(nb)
    _, nmse, s = OP.objective(h, block, rp, col)
    # by hand: each row's softmax over its own block only
    num = den = 0.0
    for i in range(48):
        logits = [float(h[i] @ h[j]) / math.sqrt(6) for j in range(48)]
        z = sum(math.exp(x) for x in logits)
        a = [math.exp(x) / z for x in logits]
        blk = range((i // 16) * 16, (i // 16) * 16 + 16)
        zb = sum(math.exp(logits[j]) for j in blk)
        b = [math.exp(logits[j]) / zb if j in blk else 0.0 for j in range(48)]
        num += sum((x - y) ** 2 for x, y in zip(a, b))
        den += sum(x * x for x in a)
    assert abs(nmse - num / den) < 1e-12
    assert abs(s - (1 - 3 / 9)) < 1e-15


def test_lse_identity_of_the_gpu_objective():
    # the GPU evaluates the Frobenius norms from log-sum-exps at scale c and 2c;
    # check that algebra against the matrices (float64)
    rng = np.random.default_rng(2)
    n, d, block = 96, 8, 16
    h = rng.standard_normal((n, d))
    nb = n // block
    keep = rng.random((nb, nb)) < 0.5
    np.fill_diagonal(keep, True)
    rp = np.concatenate([[0], np.cumsum(keep.sum(axis=1))])
    col = np.concatenate([np.flatnonzero(keep[r]) for r in range(nb)])
    _, nmse, _ = OP.objective(h, block, rp, col)
    s = (h @ h.T) / math.sqrt(d)
    tok = np.repeat(np.repeat(keep, block, 0), block, 1)

    def lse(x, m):
        x = np.where(m, x, -np.inf)
        mx = x.max(axis=1)
        return mx + np.log(np.exp(x - mx[:, None]).sum(axis=1))

    full = np.ones_like(tok)
    ld, lk, l2d, l2k = lse(s, full), lse(s, tok), lse(2 * s, full), lse(2 * s, tok)
    all2, kept2, inv_m = np.exp(l2d - 2 * ld), np.exp(l2k - 2 * ld), np.exp(ld - lk)
    err = (1 - inv_m) ** 2 * kept2 + (all2 - kept2)
    assert abs(err.sum() / all2.sum() - nmse) < 1e-12


def test_tpe_beats_its_own_random_start_on_a_quadratic():
    space = {"a": (0.0, 1.0), "b": (0.0, 1.0), "c": (0.0, 1.0)}
    target = np.array([0.73, 0.21, 0.55])

    def f(x):
        v = np.array([x["a"], x["b"], x["c"]])
        return float(((v - target) ** 2).sum())

    hist = P.tpe_minimize(f, space, trials=60, seed=4)
    ys = [y for _, y in hist]
    assert len(hist) == 60
    assert min(ys) < 0.2 * min(ys[:8])            # the model-based phase improves on the start
    assert min(ys) < 0.01
    # deterministic for a seed
    assert [y for _, y in P.tpe_minimize(f, space, trials=20, seed=4)] == ys[:20]
