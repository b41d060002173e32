"""Stage 1 on the GPU vs the oracle: candidate CSR and forced ranges, bit-exact."""
import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, Geometry
from gpu_util import cand_to_numpy, check_device_status
from oracle import geometry as OG

pytestmark = pytest.mark.gpu

GRIDS = [
    Geometry(4, 4, 4, 8, 0.5, 2.0),
    Geometry(5, 3, 5, 8, 0.3, 2.0),
    Geometry(6, 4, 4, 4, 0.2, 0.5),
    Geometry(6, 8, 8, 16, 0.05, 0.5),
    Geometry(3, 5, 7, 32, 0.5, 1.0),
    Geometry(6, 4, 4, 4, 0.2, 0.1),
    Geometry(5, 4, 6, 8, 0.4, 2.0, theta_c=0.25, theta_m=0.3),
    Geometry(4, 4, 4, 8, 0.3, 2.0, theta_c=0.5, theta_m=0.5, force_t=0),
    Geometry(7, 6, 10, 32, 0.3, 0.2),
    Geometry(9, 12, 12, 64, 0.4, 0.05, theta_c=0.1, theta_m=0.2),
    Geometry(12, 10, 13, 128, 0.6, 3.0),
    WORKLOADS["tiny"].geom,
]


@pytest.mark.parametrize("geom", GRIDS, ids=lambda g: f"{g.frames}x{g.height}x{g.width}b{g.block}")
def test_candidates_bit_exact_full(geom):
    cand = abi.dynrad_build_candidates(geom)
    check_device_status()
    got = cand_to_numpy(cand)
    want = OG.candidate_csr(geom)
    assert cand["nnz"] == len(want["col"])
    assert cand["max_row"] == int(np.diff(want["row_ptr"]).max())
    for key in ("row_ptr", "col", "forced_lo", "forced_hi"):
        np.testing.assert_array_equal(got[key], want[key], err_msg=key)


@pytest.mark.parametrize("name,gamma", [("wan13b_480p", None), ("wan14b_720p", 0.3), ("wan14b_720p", 0.7),
                                        ("hunyuan_720p", None)])
def test_candidates_bit_exact_sampled_rows_full_size(name, gamma):
    wl = WORKLOADS[name]
    geom = wl.with_gamma(gamma).geom if gamma is not None else wl.geom
    cand = abi.dynrad_build_candidates(geom)
    check_device_status()
    got = cand_to_numpy(cand)
    nb = geom.n_blocks
    rng = np.random.default_rng(17)
    rows = sorted(set([0, 1, nb // 2, nb - 2, nb - 1] + rng.choice(nb, 11, replace=False).tolist()))
    want = OG.candidate_csr(geom, rows=rows)
    for i, r in enumerate(rows):
        g_row = got["col"][got["row_ptr"][r]:got["row_ptr"][r + 1]]
        w_row = want["col"][want["row_ptr"][i]:want["row_ptr"][i + 1]]
        np.testing.assert_array_equal(g_row, w_row, err_msg=f"row {r}")
        assert got["forced_lo"][r] == want["forced_lo"][i] and got["forced_hi"][r] == want["forced_hi"][i]
    # structure over all rows: ascending, diagonal inside the forced range
    rp, col = got["row_ptr"], got["col"]
    for r in range(nb):
        row = col[rp[r]:rp[r + 1]]
        assert np.all(np.diff(row) > 0)
        assert got["forced_lo"][r] <= r <= got["forced_hi"][r]
        assert row[0] <= got["forced_lo"][r] and row[-1] >= got["forced_hi"][r]


def test_capacity_error_is_reported():
    geom = WORKLOADS["tiny"].geom
    nb = geom.n_blocks
    rp = torch.empty(nb + 1, dtype=torch.int32, device="cuda")
    flo = torch.empty(nb, dtype=torch.int32, device="cuda")
    fhi = torch.empty(nb, dtype=torch.int32, device="cuda")
    col = torch.full((10,), -7, dtype=torch.int32, device="cuda")
    import ctypes
    L = abi.lib()
    nnz = ctypes.c_int64(0)
    rc = L.dynrad_build_candidates(ctypes.byref(abi.make_geom(geom)), ctypes.c_void_p(rp.data_ptr()),
                                   ctypes.c_void_p(col.data_ptr()), 4, ctypes.c_void_p(flo.data_ptr()),
                                   ctypes.c_void_p(fhi.data_ptr()), ctypes.byref(nnz), None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == abi.DYNRAD_ERR_CAPACITY
    assert (col[4:] == -7).all()           # nothing written past the capacity
    assert abi.dynrad_device_status(clear=True) == abi.DYNRAD_ERR_CAPACITY
    assert abi.dynrad_device_status(clear=True) == 0
