"""The offline-profiling objective evaluated through the library (candidate
mask, four attention calls, dynrad_proxy_error) against the oracle's dense
matrices on the same bf16 proxy features (Appendix C.2-C.4, Eqs. 20, 22)."""
import numpy as np
import pytest

from block_sparse_attention_candidate_b200 import proxy as P
from block_sparse_attention_candidate_b200.workloads import DRIFT_REGIMES, bf16_bits_to_f64
from gpu_util import check_device_status
from oracle import geometry as OG
from oracle import proxy as OP

pytestmark = pytest.mark.gpu

SHAPE = P.ProxyShape(frames=8, height=8, width=16, dim=64, block=32)   # N = 1024


@pytest.mark.parametrize("regime", ["low", "mid", "high"])
def test_gpu_objective_matches_the_oracle(regime):
    prob = P.ProxyProblem(DRIFT_REGIMES[regime], SHAPE, seed=5)
    h = bf16_bits_to_f64(prob.bits)
    for x in ({"gamma": 1.0, "lam": 0.1, "theta_m": 0.5, "theta_c": 0.5},
              {"gamma": 2.5, "lam": 0.9, "theta_m": 0.1, "theta_c": 0.2},
              {"gamma": 1.3, "lam": 0.4, "theta_m": 0.9, "theta_c": 0.9}):
        loss, nmse, sp = prob.evaluate(x)
        check_device_status()
        cand = OG.candidate_csr(prob.geometry(x))
        want_loss, want_nmse, want_sp = OP.objective(h, SHAPE.block, cand["row_ptr"], cand["col"])
        assert sp == pytest.approx(want_sp, abs=1e-12)
        assert abs(nmse - want_nmse) <= 5e-3 + 2e-2 * want_nmse, (regime, x, nmse, want_nmse)
        assert abs(loss - want_loss) <= 5e-3 + 2e-2 * abs(want_loss)


def test_profile_loop_runs_and_keeps_the_best():
    table = P.profile_regimes(trials=6, seed=1, regimes=("mid",), shape=SHAPE)
    row = table["mid"]
    assert row["trials"] == 6 and np.isfinite(row["loss"]) and 0.0 <= row["sparsity"] <= 1.0
    for k, (lo, hi) in P.SEARCH_SPACE.items():
        assert lo <= row["x"][k] <= hi
