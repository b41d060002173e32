"""The selection entry point that allocates nothing.

dynrad_select_blocks_static_scratch serves callers that cannot allocate device
memory (an embedding application's caching allocator owns the GPU, or the
device-wide synchronisation of cudaMalloc is unacceptable): it runs the same
selection with the library's built-in device scratch.  Its results must equal
those of dynrad_select_blocks with a caller workspace, call after call.

Kept last in collection order (file name) so that a first-failure run has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, make_qkv_bf16
from gpu_util import SCORE_REL, check_device_status, gpu_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,value", [("static", 0.2), ("dynamic", 0.8)])
def test_static_scratch_matches_workspace_entry_point(mode, value):
    wl = WORKLOADS["wan13b_480p"]          # 12 heads x 32,760 tokens: fits the 32 MiB scratch
    g = wl.geom
    q, k, _ = gpu_inputs(make_qkv_bf16(wl))
    cand = abi.dynrad_build_candidates(g)
    need = abi.dynrad_select_workspace_bytes(wl.batch, wl.heads, g.n_tokens, wl.head_dim, g, cand["nnz"])
    assert 0 < need <= abi.lib().dynrad_static_scratch_bytes()
    rp_ref, col_ref, sc_ref = abi.dynrad_select_blocks(q, k, g, cand, mode, value, scores=True)
    torch.cuda.synchronize()
    check_device_status()
    n_ref = int(rp_ref[-1])
    rp_ref, col_ref, sc_ref = rp_ref.clone(), col_ref[:n_ref].clone(), sc_ref.clone()
    for i in range(2):                      # two checked calls share the scratch
        if i == 1:
            # in between, a call on other inputs (Q and K swapped, another
            # ratio / threshold) leaves other pooled means, plan and partial
            # sums in the scratch: a stage that read the scratch before writing
            # it would now see stale, wrong values
            rp2 = torch.full_like(rp_ref, -1)
            col2 = torch.full((wl.batch * wl.heads * cand["nnz"],), -1, dtype=torch.int32, device="cuda")
            abi.dynrad_select_blocks_static_scratch(k, q, g, cand, mode, value * 0.5, rp2, col2)
            torch.cuda.synchronize()
            check_device_status()
            assert not torch.equal(rp2, rp_ref)
        rp = torch.full_like(rp_ref, -1)
        col = torch.full((wl.batch * wl.heads * cand["nnz"],), -1, dtype=torch.int32, device="cuda")
        sc = torch.full_like(sc_ref, float("nan"))
        abi.dynrad_select_blocks_static_scratch(q, k, g, cand, mode, value, rp, col, sc)
        torch.cuda.synchronize()
        check_device_status()
        assert torch.equal(rp, rp_ref)
        assert torch.equal(col[:n_ref], col_ref)
        # same kernels on the same inputs: scores agree to the tolerance the
        # parity tests use (in practice bit for bit)
        d = (sc - sc_ref).abs()
        assert torch.isfinite(sc).all()
        assert float(d.max()) <= SCORE_REL * float(sc_ref.abs().max())


def test_static_scratch_rejects_oversized_problems():
    wl = WORKLOADS["wan14b_720p"]          # needs ~60 MB of scratch
    g = wl.geom
    L = abi.lib()
    need = abi.dynrad_select_workspace_bytes(wl.batch, wl.heads, g.n_tokens, wl.head_dim, g, 331078)
    assert need > L.dynrad_static_scratch_bytes()
    p = ctypes.c_void_p(0x10000)
    rc = L.dynrad_select_blocks_static_scratch(p, p, wl.batch, wl.heads, g.n_tokens, wl.head_dim,
                                               ctypes.byref(abi.make_geom(g)), p, p, 331078, 0, p, p, 0, 0.15,
                                               p, p, 100, None, None)
    assert rc == abi.DYNRAD_ERR_CAPACITY
