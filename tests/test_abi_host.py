"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every symbol include/dynrad.h declares, and rejects bad arguments before any
device work."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, Geometry

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dynrad.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(dynrad_[a-z_0-9]+)\s*\(", src, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert set(names) == set(abi.EXPORTED), names
    L = abi.lib()
    for n in names:
        assert hasattr(L, n), n


def test_geom_struct_layout_matches_c():
    # four int32, five doubles, one int32 -> 64 bytes with natural alignment
    assert ctypes.sizeof(abi.DynradGeom) == 64
    assert abi.DynradGeom.gamma.offset == 16 and abi.DynradGeom.force_t.offset == 56


def test_num_blocks_and_status_strings():
    for wl in WORKLOADS.values():
        assert abi.dynrad_num_blocks(wl.geom) == wl.geom.n_blocks
    assert abi.status_string(0) == "ok"
    assert "capacity" in abi.status_string(abi.DYNRAD_ERR_CAPACITY)
    assert abi.status_string(99) == "unknown status"


@pytest.mark.parametrize("bad", [
    Geometry(0, 4, 4, 8, 0.5, 2.0), Geometry(4, 4, 4, 0, 0.5, 2.0), Geometry(4, 4, 4, 8, 0.0, 2.0),
    Geometry(4, 4, 4, 8, 0.5, -1.0), Geometry(4, 4, 4, 8, 0.5, 2.0, theta_c=1.5),
    Geometry(4, 4, 4, 8, 0.5, 2.0, force_t=2), Geometry(4, 4, 4, 8, 0.5, 2.0, eps=-1.0),
    Geometry(4, 4, 4, 8, float("nan"), 2.0)])
def test_bad_geometry_rejected(bad):
    L = abi.lib()
    g = abi.make_geom(bad)
    assert L.dynrad_num_blocks(ctypes.byref(g)) == 0
    nnz = ctypes.c_int64(0)
    fake = ctypes.c_void_p(0x1000)
    rc = L.dynrad_build_candidates(ctypes.byref(g), fake, None, 0, fake, fake, ctypes.byref(nnz), None, None)
    assert rc == abi.DYNRAD_ERR_INVALID_ARG
    assert L.dynrad_select_workspace_bytes(1, 1, 64, 64, ctypes.byref(g), 10) == 0


def test_select_argument_errors_before_launch():
    L = abi.lib()
    geom = WORKLOADS["tiny"].geom
    g = abi.make_geom(geom)
    p = ctypes.c_void_p(0x10000)
    n = geom.n_tokens

    def call(**kw):
        a = dict(q=p, k=p, B=1, H=2, N=n, D=64, cand_row_ptr=p, cand_col=p, cand_nnz=100, cand_max_row=0,
                 flo=p, fhi=p, mode=0, value=0.25, row_ptr=p, col_idx=p, col_cap=100, scores=None,
                 ws=p, ws_bytes=0, stream=None)
        a.update(kw)
        return L.dynrad_select_blocks(a["q"], a["k"], a["B"], a["H"], a["N"], a["D"], ctypes.byref(g),
                                      a["cand_row_ptr"], a["cand_col"], a["cand_nnz"], a["cand_max_row"],
                                      a["flo"], a["fhi"], a["mode"], a["value"], a["row_ptr"], a["col_idx"],
                                      a["col_cap"], a["scores"], a["ws"], a["ws_bytes"], a["stream"])

    assert call(q=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(N=n + 1) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(D=96) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(mode=7) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(value=0.0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(value=1.5) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(q=ctypes.c_void_p(0x10008)) == abi.DYNRAD_ERR_INVALID_ARG      # not 16-byte aligned
    assert call(ws=ctypes.c_void_p(0x10010)) == abi.DYNRAD_ERR_INVALID_ARG     # not 256-byte aligned
    # workspace too small: rejected before any launch
    assert call(ws_bytes=16) == abi.DYNRAD_ERR_CAPACITY


def test_attention_argument_errors_before_launch():
    L = abi.lib()
    p = ctypes.c_void_p(0x10000)

    def call(**kw):
        a = dict(q=p, k=p, v=p, B=1, H=1, N=128, D=128, block=64, rp=p, col=p, scale=0.0, o=p, lse=p)
        a.update(kw)
        return L.dynrad_sparse_attn(a["q"], a["k"], a["v"], a["B"], a["H"], a["N"], a["D"], a["block"],
                                    a["rp"], a["col"], a["scale"], a["o"], a["lse"], None)

    assert call(v=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(D=80) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(block=48) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(N=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(scale=-1.0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(o=ctypes.c_void_p(0x10004)) == abi.DYNRAD_ERR_INVALID_ARG


def test_workspace_size_formula():
    wl = WORKLOADS["wan14b_720p"]
    g = wl.geom
    nnz = 331078
    ws = abi.dynrad_select_workspace_bytes(1, 40, g.n_tokens, 128, g, nnz)
    rows = 40 * g.n_blocks
    nbp = (g.n_blocks + 31) // 32 * 32
    # qbar [BH, Nb, D] + kbar transposed [BH, D, Nb padded to 32] (fp32) + the
    # kept lists + scan partials, each 256-byte aligned
    need = rows * 128 * 4 + 40 * 128 * nbp * 4 + 40 * nnz * 4
    assert need <= ws < need + 4096
