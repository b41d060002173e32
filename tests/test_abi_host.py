"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every symbol include/dynrad.h declares, and rejects bad arguments before any
device work."""
import ctypes
import math
import os
import re

import pytest

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, Geometry
from oracle import geometry

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
    # qbar and kbar [BH, Nb, D] (fp32) + the scoring plan (per group of 8
    # rows: offset, size and static kept count; union members and 8 scatter
    # positions, at most cand_nnz entries) + dynamic mode's kept lists at the
    # candidate offsets and scan partials + the launch's counters (ticket, plan
    # counters, one per head), each region 256-byte aligned
    groups = (g.n_blocks + 7) // 8
    tiles = (rows + 1 + 4095) // 4096
    need = 2 * rows * 128 * 4 + 3 * groups * 4 + nnz * 4 * 9 + 40 * nnz * 4 + tiles * 8 + 16 + 40 * 4
    assert need <= ws < need + 4096


def _c_layout(struct, fields):
    """sizeof / offsetof of a struct of include/dynrad.h, from gcc."""
    import shutil
    import subprocess
    import tempfile
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    body = "\n".join(f'  printf("%zu\\n", offsetof({struct}, {f}));' for f in fields)
    src = (f'#include <stddef.h>\n#include <stdio.h>\n#include "dynrad.h"\n'
           f'int main(void) {{\n  printf("%zu\\n", sizeof({struct}));\n{body}\n  return 0;\n}}\n')
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), "-o", exe, c], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    return [int(x) for x in out]


def test_host_run_struct_layout_matches_c():
    names = [f[0] for f in abi.DynradHostRun._fields_]
    got = _c_layout("dynrad_host_run", names)
    assert got[0] == ctypes.sizeof(abi.DynradHostRun)
    for n, off in zip(names, got[1:]):
        assert getattr(abi.DynradHostRun, n).offset == off, n


def _fake_runs(n, geom, o=0x20000, nnz=100):
    arr = (abi.DynradHostRun * max(1, n))()
    for i in range(n):
        arr[i] = abi.DynradHostRun(abi.make_geom(geom), 0x10000, 0x10000, nnz, 0, 0x10000, 0x10000, 0, 0.25,
                                   o, 0x30000)
    return arr


def test_host_path_argument_errors_before_any_device_work():
    L = abi.lib()
    geom = WORKLOADS["tiny"].geom
    n = geom.n_tokens
    p = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)   # 256-byte aligned, never dereferenced on these paths

    def call(runs=None, n_runs=2, chunk=1, ws_ptr=ws, ws_bytes=1 << 40, q=p, N=n, D=64, scale=0.0):
        runs = _fake_runs(2, geom) if runs is None else runs
        return L.dynrad_host_path(q, p, p, 1, 2, N, D, runs, n_runs, chunk, scale, ws_ptr, ws_bytes, None)

    assert call(q=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(n_runs=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(runs=_fake_runs(17, geom), n_runs=17) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(chunk=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(N=n + 1) == abi.DYNRAD_ERR_INVALID_ARG            # geometry does not match N
    assert call(D=96) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(ws_ptr=ctypes.c_void_p(0x100010)) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(ws_bytes=4096) == abi.DYNRAD_ERR_CAPACITY
    assert call(runs=_fake_runs(2, geom, o=0)) == abi.DYNRAD_ERR_INVALID_ARG   # null o_host
    assert call(scale=-1.0) == abi.DYNRAD_ERR_INVALID_ARG
    assert L.dynrad_host_path_workspace_bytes(1, 2, n, 64, _fake_runs(2, geom), 0, 1) == 0


def test_host_path_workspace_size_formula():
    L = abi.lib()
    wl = WORKLOADS["wan14b_720p"]
    g = wl.geom
    B, H, N, D, chunk, nnz = 1, 40, g.n_tokens, 128, 4, 331078
    runs = _fake_runs(4, g, nnz=nnz)
    got = L.dynrad_host_path_workspace_bytes(B, H, N, D, runs, 4, chunk)
    qkv = B * H * N * D * 2
    sel = abi.dynrad_select_workspace_bytes(1, chunk, N, D, g, nnz)
    # Q, K, V; O and LSE per run; per compute stream one chunk's kept CSR and
    # selection workspace
    need = 3 * qkv + 4 * (qkv + B * H * N * 4) + 2 * ((chunk * g.n_blocks + 1) * 4 + chunk * nnz * 4 + sel)
    assert need <= got < need + 256 * 16


def test_sampled_mask_argument_errors_before_launch():
    L = abi.lib()
    geom = WORKLOADS["tiny"].geom
    g = abi.make_geom(geom)
    p = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)

    def call(rho1=0.3, rho2=0.1, reps=1, ws_ptr=ws, ws_bytes=1 << 40, rp=p, geom_=g, nnz=100):
        return L.dynrad_build_sampled_mask(ctypes.byref(geom_), rho1, rho2, 7, p, p, nnz, p, p, reps, rp, p, 1000,
                                           None, ws_ptr, ws_bytes, None)

    assert call(rp=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(rho1=0.0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(rho2=1.5) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(reps=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(nnz=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(ws_ptr=ctypes.c_void_p(0x100010)) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(ws_bytes=64) == abi.DYNRAD_ERR_CAPACITY
    g16 = abi.make_geom(Geometry(4, 4, 4, 16, 0.5, 2.0))
    assert call(geom_=g16) == abi.DYNRAD_ERR_UNSUPPORTED
    F = geom.frames
    assert L.dynrad_sampled_mask_workspace_min_bytes(ctypes.byref(g), 0) == 0
    assert L.dynrad_sampled_mask_workspace_bytes(ctypes.byref(g), 0) == 0
    least = L.dynrad_sampled_mask_workspace_min_bytes(ctypes.byref(g), 100)
    # frame-pair records (56 B), two counters each plus two, thresholds, kept
    # lists, keep flags, scan partials
    fixed = F * F * (56 + 16 + 8) + 16 + 400 + 100 + 8
    assert fixed <= least < fixed + 256 * 6
    assert call(ws_bytes=least - 1) == abi.DYNRAD_ERR_CAPACITY
    # the pool: per sampled frame pair, slots for its widest key window
    w, r = geometry.frame_tables(geom)
    nt = geom.tokens_per_frame
    keys = 0
    for t in range(2, F):
        if not r[t]:
            continue
        wc = min(int(w[t]), nt - 1)
        n = nt * (2 * wc + 1) - wc * (wc + 1)
        e = 7.0 * math.sqrt(n) + 128.0
        slots = min(n, math.ceil(e + 8.0 * math.sqrt(e) + 64.0), 2 ** 31 - 1)
        keys += 2 * (F - t) * (slots + 2)
    need = L.dynrad_sampled_mask_workspace_bytes(ctypes.byref(g), 100)
    assert least + 8 * keys <= need < least + 8 * keys + 256


def test_token_mask_argument_errors_before_launch():
    L = abi.lib()
    geom = WORKLOADS["tiny"].geom
    g = abi.make_geom(geom)
    p = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    n = geom.n_tokens

    def call(q=p, B=1, H=2, N=n, D=64, hf=2, tau1=0.5, tau2=1.0, ws_ptr=ws, ws_bytes=1 << 40, geom_=g):
        return L.dynrad_build_token_mask(q, p, B, H, N, D, hf, ctypes.byref(geom_), tau1, tau2, p, p, 100, p, p,
                                         p, p, 1000, None, ws_ptr, ws_bytes, None)

    assert call(q=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(N=n + 1) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(hf=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(hf=3) == abi.DYNRAD_ERR_INVALID_ARG            # more fused heads than heads
    assert call(H=8, hf=5) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(tau1=float("inf")) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(D=96) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(ws_ptr=ctypes.c_void_p(0x100008)) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(ws_bytes=1024) == abi.DYNRAD_ERR_CAPACITY
    assert call(geom_=abi.make_geom(Geometry(4, 4, 4, 16, 0.5, 2.0)), N=64) == abi.DYNRAD_ERR_UNSUPPORTED
    need = L.dynrad_token_mask_workspace_bytes(2, n, ctypes.byref(g), 100)
    F, nb = geom.frames, geom.n_blocks
    # per (batch, frame pair) sums, maxima and thresholds; per (batch, row, key
    # token) link counters; kept lists, per-batch CSR, scan partials
    base = 2 * F * F * 32 + 2 * nb * n * 4 + 2 * 100 * 4 * 2 + (2 * nb + 1) * 4 + 8
    assert base <= need < base + 256 * 9


def test_proxy_error_argument_errors():
    L = abi.lib()
    p = ctypes.c_void_p(0x10000)
    assert L.dynrad_proxy_error(None, p, p, p, 10, p, None) == abi.DYNRAD_ERR_INVALID_ARG
    assert L.dynrad_proxy_error(p, p, p, p, 0, p, None) == abi.DYNRAD_ERR_INVALID_ARG
    assert L.dynrad_proxy_error(p, p, p, p, 10, None, None) == abi.DYNRAD_ERR_INVALID_ARG


def test_backward_argument_errors_before_launch():
    L = abi.lib()
    p = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)

    def call(**kw):
        a = dict(q=p, B=1, H=2, N=300, D=128, block=64, cap=100, scale=0.0, dq=p, ws=ws, ws_bytes=1 << 40)
        a.update(kw)
        return L.dynrad_attn_backward(a["q"], p, p, p, p, p, a["B"], a["H"], a["N"], a["D"], a["block"], p, p,
                                      a["cap"], a["scale"], a["dq"], p, p, a["ws"], a["ws_bytes"], None)

    assert call(q=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(dq=None) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(N=0) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(cap=-1) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(scale=-0.5) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(scale=float("nan")) == abi.DYNRAD_ERR_INVALID_ARG
    assert call(D=96) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(block=48) == abi.DYNRAD_ERR_UNSUPPORTED
    assert call(dq=ctypes.c_void_p(0x10008)) == abi.DYNRAD_ERR_INVALID_ARG    # not 16-byte aligned
    assert call(ws=ctypes.c_void_p(0x100010)) == abi.DYNRAD_ERR_INVALID_ARG   # not 256-byte aligned
    assert call(B=300, H=300) == abi.DYNRAD_ERR_UNSUPPORTED                   # B*H > 65535
    assert call(ws_bytes=1024) == abi.DYNRAD_ERR_CAPACITY


def test_backward_workspace_size_formula():
    L = abi.lib()
    B, H, N, block, cap = 1, 40, 75600, 64, 11_000_000
    nb = -(-N // block)
    rows = B * H * nb
    tiles = -(-(rows + 1) // 2048)
    got = L.dynrad_attn_backward_workspace_bytes(B, H, N, block, cap)
    # (lse log2 e, D_r) per query row padded to 64 rows (2 x fp32), transposed CSR
    # offsets and entries (int32), scan partials
    need = B * H * (-(-N // 64) * 64) * 8 + (rows + 1) * 4 + cap * 4 + tiles * 8
    assert need <= got < need + 4 * 256
    assert L.dynrad_attn_backward_workspace_bytes(0, H, N, block, cap) == 0


def test_attention_binding_checks_shapes_dtypes_and_csr_length():
    import torch
    chk = abi._check_attn_args
    bf = torch.bfloat16

    def t(*shape, dtype=bf):
        return torch.zeros(shape, dtype=dtype)

    q = t(1, 2, 1000, 64)
    nb = -(-1000 // 64)
    rp = t(2 * nb + 1, dtype=torch.int32)
    col = t(5, dtype=torch.int32)
    lse = t(1, 2, 1000, dtype=torch.float32)
    chk(q, (q, q, None), 64, rp, col, None)                       # forward, outputs allocated
    chk(q, (q, q, q), 64, rp, col, lse)                           # forward into caller buffers
    chk(q, (q, q, q, q, q, q, q), 64, rp, col, lse)               # backward with caller gradients
    chk(t(1, 1, 4096, 64), (), 32, t(129, dtype=torch.int32), col, lse.new_zeros(4096))  # one head, flat lse
    chk(t(1, 1, 64, 64), (), 48, t(2, dtype=torch.int32), col, t(1, 1, 64, dtype=torch.float32))  # size left to the library
    bad = [
        lambda: chk(t(1, 2, 1000, 64, dtype=torch.float16), (), 64, rp, col),
        lambda: chk(q, (t(1, 2, 1000, 128),), 64, rp, col),
        lambda: chk(q, (q.float(),), 64, rp, col),
        lambda: chk(t(2, 1000, 64), (), 64, rp, col),
        lambda: chk(q, (), 64, rp, col, t(1, 2, 999, dtype=torch.float32)),
        lambda: chk(q, (), 64, rp, col, t(1, 2, 1000)),
        lambda: chk(q, (), 64, rp.long(), col),
        lambda: chk(q, (), 64, rp, col.long()),
        lambda: chk(q, (), 64, rp[:-1], col),                      # one offset short
        lambda: chk(q, (), 32, rp, col),                           # block 32 reads 2 * 32 + 1 offsets
    ]
    for i, f in enumerate(bad):
        with pytest.raises(ValueError):
            f()
