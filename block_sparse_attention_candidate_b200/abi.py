"""ctypes binding of libdynrad.so (declared in include/dynrad.h).

Argument marshalling only: tensors become device pointers, the stream is
torch's current stream, every step of the path runs in the library's kernels.
There is no fallback: if the library is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdynrad.so")

DYNRAD_OK = 0
DYNRAD_ERR_INVALID_ARG = 1
DYNRAD_ERR_UNSUPPORTED = 2
DYNRAD_ERR_CAPACITY = 3
DYNRAD_ERR_CUDA = 4
DYNRAD_ERR_DEVICE = 5

DYNRAD_STATIC_RATIO = 0
DYNRAD_DYNAMIC_THRESHOLD = 1
MODES = {"static": DYNRAD_STATIC_RATIO, "dynamic": DYNRAD_DYNAMIC_THRESHOLD}

# every extern "C" symbol include/dynrad.h declares
EXPORTED = (
    "dynrad_num_blocks",
    "dynrad_build_candidates",
    "dynrad_select_workspace_bytes",
    "dynrad_select_blocks",
    "dynrad_sparse_attn",
    "dynrad_device_status",
    "dynrad_status_string",
    "dynrad_debug_exp2",
    "dynrad_static_scratch_bytes",
    "dynrad_select_blocks_static_scratch",
    "dynrad_host_path_workspace_bytes",
    "dynrad_host_path",
    "dynrad_sampled_mask_workspace_bytes",
    "dynrad_sampled_mask_workspace_min_bytes",
    "dynrad_build_sampled_mask",
    "dynrad_token_mask_workspace_bytes",
    "dynrad_build_token_mask",
    "dynrad_proxy_error",
    "dynrad_attn_backward_workspace_bytes",
    "dynrad_attn_backward",
    "dynrad_debug_attn_stall",
)


class DynradGeom(ctypes.Structure):
    _fields_ = [
        ("frames", ctypes.c_int32),
        ("height", ctypes.c_int32),
        ("width", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("gamma", ctypes.c_double),
        ("lambda_", ctypes.c_double),
        ("theta_c", ctypes.c_double),
        ("theta_m", ctypes.c_double),
        ("eps", ctypes.c_double),
        ("force_t", ctypes.c_int32),
    ]


class DynradHostRun(ctypes.Structure):
    _fields_ = [
        ("geom", DynradGeom),
        ("cand_row_ptr", ctypes.c_void_p),
        ("cand_col", ctypes.c_void_p),
        ("cand_nnz", ctypes.c_int64),
        ("cand_max_row", ctypes.c_int64),
        ("forced_lo", ctypes.c_void_p),
        ("forced_hi", ctypes.c_void_p),
        ("mode", ctypes.c_int32),
        ("rho_or_tau", ctypes.c_double),
        ("o_host", ctypes.c_void_p),
        ("lse_host", ctypes.c_void_p),
    ]


class DynradError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None

_VP = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_I64P = ctypes.POINTER(ctypes.c_int64)
_I32P = ctypes.POINTER(ctypes.c_int32)
_GP = ctypes.POINTER(DynradGeom)


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if libdynrad.so is absent (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_attention_candidate_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.dynrad_num_blocks.restype = _I64
        L.dynrad_num_blocks.argtypes = [_GP]
        L.dynrad_build_candidates.restype = ctypes.c_int
        L.dynrad_build_candidates.argtypes = [_GP, _VP, _VP, _I64, _VP, _VP, _I64P, _I64P, _VP]
        L.dynrad_select_workspace_bytes.restype = _SZ
        L.dynrad_select_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _GP, _I64]
        L.dynrad_select_blocks.restype = ctypes.c_int
        L.dynrad_select_blocks.argtypes = [_VP, _VP, _I32, _I32, _I32, _I32, _GP, _VP, _VP, _I64, _I64,
                                           _VP, _VP, _I32, ctypes.c_double, _VP, _VP, _I64, _VP, _VP, _SZ,
                                           _VP]
        L.dynrad_sparse_attn.restype = ctypes.c_int
        L.dynrad_sparse_attn.argtypes = [_VP, _VP, _VP, _I32, _I32, _I32, _I32, _I32, _VP, _VP,
                                         ctypes.c_float, _VP, _VP, _VP]
        L.dynrad_device_status.restype = ctypes.c_int
        L.dynrad_device_status.argtypes = [_I32P, _I32, _VP]
        L.dynrad_status_string.restype = ctypes.c_char_p
        L.dynrad_status_string.argtypes = [_I32]
        L.dynrad_debug_exp2.restype = ctypes.c_int
        L.dynrad_debug_exp2.argtypes = [_VP, _VP, _VP, _I64, _VP]
        L.dynrad_static_scratch_bytes.restype = _SZ
        L.dynrad_static_scratch_bytes.argtypes = []
        L.dynrad_select_blocks_static_scratch.restype = ctypes.c_int
        L.dynrad_select_blocks_static_scratch.argtypes = [_VP, _VP, _I32, _I32, _I32, _I32, _GP, _VP, _VP, _I64,
                                                          _I64, _VP, _VP, _I32, ctypes.c_double, _VP, _VP, _I64,
                                                          _VP, _VP]
        L.dynrad_host_path_workspace_bytes.restype = _SZ
        L.dynrad_host_path_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, ctypes.POINTER(DynradHostRun), _I32,
                                                       _I32]
        L.dynrad_host_path.restype = ctypes.c_int
        L.dynrad_host_path.argtypes = [_VP, _VP, _VP, _I32, _I32, _I32, _I32, ctypes.POINTER(DynradHostRun), _I32,
                                       _I32, ctypes.c_float, _VP, _SZ, _VP]
        L.dynrad_sampled_mask_workspace_bytes.restype = _SZ
        L.dynrad_sampled_mask_workspace_bytes.argtypes = [_GP, _I64]
        L.dynrad_sampled_mask_workspace_min_bytes.restype = _SZ
        L.dynrad_sampled_mask_workspace_min_bytes.argtypes = [_GP, _I64]
        L.dynrad_build_sampled_mask.restype = ctypes.c_int
        L.dynrad_build_sampled_mask.argtypes = [_GP, ctypes.c_double, ctypes.c_double, ctypes.c_uint64, _VP, _VP, _I64,
                                                _VP, _VP, _I32, _VP, _VP, _I64, _VP, _VP, _SZ, _VP]
        L.dynrad_token_mask_workspace_bytes.restype = _SZ
        L.dynrad_token_mask_workspace_bytes.argtypes = [_I32, _I32, _GP, _I64]
        L.dynrad_build_token_mask.restype = ctypes.c_int
        L.dynrad_build_token_mask.argtypes = [_VP, _VP, _I32, _I32, _I32, _I32, _I32, _GP, ctypes.c_double,
                                              ctypes.c_double, _VP, _VP, _I64, _VP, _VP, _VP, _VP, _I64, _VP, _VP,
                                              _SZ, _VP]
        L.dynrad_proxy_error.restype = ctypes.c_int
        L.dynrad_proxy_error.argtypes = [_VP, _VP, _VP, _VP, _I64, _VP, _VP]
        L.dynrad_attn_backward_workspace_bytes.restype = _SZ
        L.dynrad_attn_backward_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _I64]
        L.dynrad_attn_backward.restype = ctypes.c_int
        L.dynrad_attn_backward.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _I32, _I32, _I32, _I32, _I32, _VP, _VP,
                                           _I64, ctypes.c_float, _VP, _VP, _VP, _VP, _SZ, _VP]
        L.dynrad_debug_attn_stall.restype = ctypes.c_int
        L.dynrad_debug_attn_stall.argtypes = [ctypes.c_uint64, _I32]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().dynrad_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != DYNRAD_OK:
        raise DynradError(rc, where)


def make_geom(g) -> DynradGeom:
    """C geometry struct from an object with frames, height, width, block,
    gamma, lam, theta_c, theta_m, eps, force_t (workloads.Geometry)."""
    return DynradGeom(int(g.frames), int(g.height), int(g.width), int(g.block), float(g.gamma),
                      float(g.lam), float(g.theta_c), float(g.theta_m), float(g.eps), int(g.force_t))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


_ATTN_BLOCKS = (32, 64, 128)


def _check_attn_args(q, others, block, row_ptr, col_idx, lse=None) -> None:
    """Host checks that keep the attention kernels inside the caller's buffers:
    q and every tensor of `others` bf16 [B, H, N, D] of one shape, lse fp32
    with B*H*N elements, the CSR int32 with at least B*H*Nb + 1 offsets (for
    the block sizes the library implements; others are left to its status
    code).  Raises ValueError."""
    if q.dim() != 4 or q.dtype != torch.bfloat16:
        raise ValueError("q must be a bf16 [B, H, N, D] tensor")
    for t in others:
        if t is not None and (t.dtype != torch.bfloat16 or t.shape != q.shape):
            raise ValueError("q, k, v, o, dout and the gradients must be bf16 tensors of one shape")
    B, H, N, _ = q.shape
    if lse is not None and (lse.dtype != torch.float32 or lse.numel() != B * H * N):
        raise ValueError("lse must be an fp32 tensor of B*H*N elements")
    if row_ptr.dtype != torch.int32 or col_idx.dtype != torch.int32:
        raise ValueError("row_ptr and col_idx must be int32 tensors")
    if int(block) in _ATTN_BLOCKS:
        need = B * H * (-(-N // int(block))) + 1
        if row_ptr.numel() < need:
            raise ValueError(f"row_ptr holds {row_ptr.numel()} offsets; B*H*Nb + 1 = {need} are read")


def dynrad_num_blocks(geom) -> int:
    return int(lib().dynrad_num_blocks(ctypes.byref(make_geom(geom))))


def dynrad_build_candidates(geom, device=None, stream=None) -> dict:
    """Stage 1.  Returns dict(row_ptr, col, forced_lo, forced_hi: int32 CUDA
    tensors; nnz, max_row: ints).  Synchronizes once (size query)."""
    L = lib()
    cg = make_geom(geom)
    nb = int(L.dynrad_num_blocks(ctypes.byref(cg)))
    if nb <= 0:
        raise DynradError(DYNRAD_ERR_INVALID_ARG, "dynrad_build_candidates")
    device = device or torch.device("cuda", torch.cuda.current_device())
    row_ptr = torch.empty(nb + 1, dtype=torch.int32, device=device)
    flo = torch.empty(nb, dtype=torch.int32, device=device)
    fhi = torch.empty(nb, dtype=torch.int32, device=device)
    nnz = ctypes.c_int64(0)
    mx = ctypes.c_int64(0)
    st = _stream(stream)
    _check(L.dynrad_build_candidates(ctypes.byref(cg), _ptr(row_ptr), None, 0, _ptr(flo), _ptr(fhi),
                                     ctypes.byref(nnz), ctypes.byref(mx), st), "dynrad_build_candidates")
    col = torch.empty(max(1, nnz.value), dtype=torch.int32, device=device)
    _check(L.dynrad_build_candidates(ctypes.byref(cg), _ptr(row_ptr), _ptr(col), col.numel(), _ptr(flo),
                                     _ptr(fhi), ctypes.byref(nnz), ctypes.byref(mx), st),
           "dynrad_build_candidates")
    return {"row_ptr": row_ptr, "col": col[: nnz.value], "forced_lo": flo, "forced_hi": fhi,
            "nnz": nnz.value, "max_row": mx.value, "nb": nb}


def dynrad_build_candidates_into(geom, cand: dict, stream=None) -> None:
    """Stage 1 into existing buffers (from dynrad_build_candidates): the fill
    call only, asynchronous, no host synchronization."""
    L = lib()
    cg = make_geom(geom)
    _check(L.dynrad_build_candidates(ctypes.byref(cg), _ptr(cand["row_ptr"]), _ptr(cand["col"]),
                                     cand["col"].numel(), _ptr(cand["forced_lo"]), _ptr(cand["forced_hi"]),
                                     None, None, _stream(stream)), "dynrad_build_candidates")


def dynrad_select_workspace_bytes(B, H, N, D, geom, cand_nnz) -> int:
    return int(lib().dynrad_select_workspace_bytes(B, H, N, D, ctypes.byref(make_geom(geom)), cand_nnz))


class SelectBuffers:
    """Caller-owned outputs and workspace of dynrad_select_blocks (reusable)."""

    def __init__(self, B, H, N, D, geom, cand, device=None, scores=False):
        device = device or torch.device("cuda", torch.cuda.current_device())
        nb = cand["nb"]
        ws = dynrad_select_workspace_bytes(B, H, N, D, geom, cand["nnz"])
        if ws == 0:
            raise DynradError(DYNRAD_ERR_INVALID_ARG, "dynrad_select_workspace_bytes")
        self.workspace = torch.empty(ws + 256, dtype=torch.uint8, device=device)
        off = (-self.workspace.data_ptr()) % 256
        self.ws_view = self.workspace[off:off + ws]
        self.row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(B * H * cand["nnz"], dtype=torch.int32, device=device)
        self.scores = torch.empty(B * H * cand["nnz"], dtype=torch.float32, device=device) if scores else None


def dynrad_select_blocks(q, k, geom, cand, mode, value, scores=False, buffers=None, stream=None):
    """Stage 2.  q, k: bf16 [B, H, N, D] CUDA.  Returns (row_ptr, col_idx,
    scores or None); col_idx has capacity B*H*cand_nnz (use row_ptr[-1])."""
    _require_cuda(q, k)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise ValueError("q, k must be bf16")
    B, H, N, D = q.shape
    buf = buffers or SelectBuffers(B, H, N, D, geom, cand, q.device, scores)
    if scores and buf.scores is None:
        raise ValueError("buffers were made without a score array")
    L = lib()
    cg = make_geom(geom)
    _check(L.dynrad_select_blocks(_ptr(q), _ptr(k), B, H, N, D, ctypes.byref(cg), _ptr(cand["row_ptr"]),
                                  _ptr(cand["col"]), cand["nnz"], cand["max_row"], _ptr(cand["forced_lo"]),
                                  _ptr(cand["forced_hi"]), MODES[mode] if isinstance(mode, str) else mode,
                                  float(value), _ptr(buf.row_ptr), _ptr(buf.col_idx), buf.col_idx.numel(),
                                  _ptr(buf.scores) if scores else None, _ptr(buf.ws_view),
                                  buf.ws_view.numel(), _stream(stream)),
           "dynrad_select_blocks")
    return buf.row_ptr, buf.col_idx, (buf.scores if scores else None)


def dynrad_sparse_attn(q, k, v, block, row_ptr, col_idx, scale=0.0, out=None, lse=None, stream=None):
    """Stage 3.  q, k, v: bf16 [B, H, N, D] CUDA; CSR over B*H*Nb rows.
    Returns (o bf16 [B, H, N, D], lse fp32 [B, H, N])."""
    _require_cuda(q, k, v, row_ptr, col_idx, out, lse)
    _check_attn_args(q, (k, v, out), block, row_ptr, col_idx, lse)
    B, H, N, D = q.shape
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(lib().dynrad_sparse_attn(_ptr(q), _ptr(k), _ptr(v), B, H, N, D, int(block), _ptr(row_ptr),
                                    _ptr(col_idx), float(scale), _ptr(o), _ptr(lse_t), _stream(stream)),
           "dynrad_sparse_attn")
    return o, lse_t


def dynrad_attn_backward(q, k, v, o, lse, dout, block, row_ptr, col_idx, scale=0.0, grads=None, workspace=None,
                         stream=None):
    """Gradient of stage 3 under the same CSR.  q, k, v, o, dout: bf16
    [B, H, N, D] CUDA; lse fp32 [B, H, N] from dynrad_sparse_attn.
    Returns (dq, dk, dv), bf16 [B, H, N, D]."""
    _require_cuda(q, k, v, o, lse, dout, row_ptr, col_idx, *(grads or ()))
    _check_attn_args(q, (k, v, o, dout) + tuple(grads or ()), block, row_ptr, col_idx, lse)
    B, H, N, D = q.shape
    dq, dk, dv = grads if grads is not None else tuple(torch.empty_like(q) for _ in range(3))
    cap = col_idx.numel()
    L = lib()
    need = L.dynrad_attn_backward_workspace_bytes(B, H, N, int(block), cap)
    if need == 0:
        raise DynradError(1, "dynrad_attn_backward_workspace_bytes")
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    _check(L.dynrad_attn_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), B, H, N, D, int(block),
                                  _ptr(row_ptr), _ptr(col_idx), cap, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                                  _ptr(ws), ws.numel(), _stream(stream)), "dynrad_attn_backward")
    return dq, dk, dv


def dynrad_select_blocks_static_scratch(q, k, geom, cand, mode, value, row_ptr, col_idx, scores=None,
                                        stream=None) -> None:
    """Stage 2 into caller-provided outputs, with the library's built-in device
    scratch instead of a workspace: the call allocates nothing (for callers
    that cannot allocate device memory).  Calls that overlap on the GPU race."""
    _require_cuda(q, k, row_ptr, col_idx, scores)
    B, H, N, D = q.shape
    L = lib()
    _check(L.dynrad_select_blocks_static_scratch(
        _ptr(q), _ptr(k), B, H, N, D, ctypes.byref(make_geom(geom)), _ptr(cand["row_ptr"]), _ptr(cand["col"]),
        cand["nnz"], cand["max_row"], _ptr(cand["forced_lo"]), _ptr(cand["forced_hi"]),
        MODES[mode] if isinstance(mode, str) else mode, float(value), _ptr(row_ptr), _ptr(col_idx),
        col_idx.numel(), _ptr(scores), _stream(stream)), "dynrad_select_blocks_static_scratch")


def dynrad_debug_exp2(x: torch.Tensor):
    """(approximation, CUDA exp2f) of 2^x for a float32 CUDA tensor."""
    _require_cuda(x)
    poly = torch.empty_like(x)
    ref = torch.empty_like(x)
    _check(lib().dynrad_debug_exp2(_ptr(x), _ptr(poly), _ptr(ref), x.numel(), _stream()), "dynrad_debug_exp2")
    return poly, ref


def dynrad_device_status(clear: bool = True, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().dynrad_device_status(ctypes.byref(v), 1 if clear else 0, _stream(stream)),
           "dynrad_device_status")
    return int(v.value)


def make_host_runs(runs) -> ctypes.Array:
    """C array of dynrad_host_run from dicts with geom, cand (from
    dynrad_build_candidates), mode, value, o_host, lse_host (pinned CPU
    tensors bf16 [B, H, N, D] / fp32 [B, H, N])."""
    arr = (DynradHostRun * len(runs))()
    for i, r in enumerate(runs):
        c = r["cand"]
        for t in (r["o_host"], r["lse_host"]):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("o_host / lse_host must be contiguous host tensors")
        arr[i] = DynradHostRun(make_geom(r["geom"]), c["row_ptr"].data_ptr(), c["col"].data_ptr(), c["nnz"],
                               c["max_row"], c["forced_lo"].data_ptr(), c["forced_hi"].data_ptr(),
                               MODES[r["mode"]] if isinstance(r["mode"], str) else int(r["mode"]), float(r["value"]),
                               r["o_host"].data_ptr(), r["lse_host"].data_ptr())
    return arr


def dynrad_host_path_workspace_bytes(B, H, N, D, runs, chunk_bh) -> int:
    arr = make_host_runs(runs)
    return int(lib().dynrad_host_path_workspace_bytes(B, H, N, D, arr, len(runs), int(chunk_bh)))


class HostPathWorkspace:
    """Device workspace of dynrad_host_path (reusable across calls)."""

    def __init__(self, B, H, N, D, runs, chunk_bh, device=None):
        device = device or torch.device("cuda", torch.cuda.current_device())
        n = dynrad_host_path_workspace_bytes(B, H, N, D, runs, chunk_bh)
        if n == 0:
            raise DynradError(DYNRAD_ERR_INVALID_ARG, "dynrad_host_path_workspace_bytes")
        self.buffer = torch.empty(n + 256, dtype=torch.uint8, device=device)
        off = (-self.buffer.data_ptr()) % 256
        self.view = self.buffer[off:off + n]


def dynrad_host_path(q_host, k_host, v_host, runs, chunk_bh=4, scale=0.0, workspace=None, stream=None):
    """Stages 2 and 3 from pinned host Q, K, V (bf16 [B, H, N, D]) to each
    run's pinned host o_host / lse_host, copies overlapped with the kernels.
    Asynchronous on `stream` (torch's current stream by default)."""
    for t in (q_host, k_host, v_host):
        if t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("q_host, k_host, v_host must be contiguous bf16 host tensors")
    B, H, N, D = q_host.shape
    arr = make_host_runs(runs)
    ws = workspace or HostPathWorkspace(B, H, N, D, runs, chunk_bh)
    _check(lib().dynrad_host_path(ctypes.c_void_p(q_host.data_ptr()), ctypes.c_void_p(k_host.data_ptr()),
                                  ctypes.c_void_p(v_host.data_ptr()), B, H, N, D, arr, len(runs), int(chunk_bh),
                                  float(scale), _ptr(ws.view), ws.view.numel(), _stream(stream)),
           "dynrad_host_path")
    return ws


def dynrad_build_sampled_mask(geom, cand, rho1, rho2, seed, replicas=1, thresholds=False, stream=None,
                              workspace_bytes=None):
    """Paper-exact static-ratio mask (Eq. 8, seeded token-pair sampling), the
    same for every head, written ``replicas`` times.  Returns (row_ptr int32
    [replicas*Nb+1], col_idx int32 with capacity replicas*cand_nnz, thresholds
    int64 [F*F] holding the uint64 T(i, j) bits, or None).  ``workspace_bytes``
    (default: the full size) may be anything from
    dynrad_sampled_mask_workspace_min_bytes up; a smaller pool only slows the
    build."""
    L = lib()
    cg = make_geom(geom)
    device = cand["row_ptr"].device
    ws_bytes = int(L.dynrad_sampled_mask_workspace_bytes(ctypes.byref(cg), cand["nnz"]))
    if ws_bytes == 0:
        raise DynradError(DYNRAD_ERR_INVALID_ARG, "dynrad_sampled_mask_workspace_bytes")
    if workspace_bytes is not None:
        ws_bytes = int(workspace_bytes)
    ws = torch.empty(ws_bytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    nb = cand["nb"]
    row_ptr = torch.empty(replicas * nb + 1, dtype=torch.int32, device=device)
    col = torch.empty(max(1, replicas * cand["nnz"]), dtype=torch.int32, device=device)
    thr = torch.empty(geom.frames * geom.frames, dtype=torch.int64, device=device) if thresholds else None
    _check(L.dynrad_build_sampled_mask(ctypes.byref(cg), float(rho1), float(rho2), int(seed) & ((1 << 64) - 1),
                                       _ptr(cand["row_ptr"]), _ptr(cand["col"]), cand["nnz"], _ptr(cand["forced_lo"]),
                                       _ptr(cand["forced_hi"]), int(replicas), _ptr(row_ptr), _ptr(col), col.numel(),
                                       _ptr(thr), ctypes.c_void_p(ws.data_ptr() + off), ws_bytes, _stream(stream)),
           "dynrad_build_sampled_mask")
    return row_ptr, col, thr


def dynrad_build_token_mask(q, k, geom, cand, tau1, tau2, hf=2, stats=False, stream=None):
    """Paper-exact dynamic-threshold mask (Eqs. 9-11, 19) from bf16 [B, H, N, D]
    CUDA q, k: one mask per batch element from its first ``hf`` heads, written
    for every head.  Returns (row_ptr int32 [B*H*Nb+1], col_idx int32 with
    capacity B*H*cand_nnz, stats float64 [B, F*F, 3] (mu, sigma, threshold) or None)."""
    _require_cuda(q, k)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise ValueError("q, k must be bf16")
    B, H, N, D = q.shape
    L = lib()
    cg = make_geom(geom)
    ws_bytes = int(L.dynrad_token_mask_workspace_bytes(B, N, ctypes.byref(cg), cand["nnz"]))
    if ws_bytes == 0:
        raise DynradError(DYNRAD_ERR_INVALID_ARG, "dynrad_token_mask_workspace_bytes")
    ws = torch.empty(ws_bytes + 256, dtype=torch.uint8, device=q.device)
    off = (-ws.data_ptr()) % 256
    nb = cand["nb"]
    row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=q.device)
    col = torch.empty(max(1, B * H * cand["nnz"]), dtype=torch.int32, device=q.device)
    st = torch.empty((B, geom.frames * geom.frames, 3), dtype=torch.float64, device=q.device) if stats else None
    _check(L.dynrad_build_token_mask(_ptr(q), _ptr(k), B, H, N, D, int(hf), ctypes.byref(cg), float(tau1), float(tau2),
                                     _ptr(cand["row_ptr"]), _ptr(cand["col"]), cand["nnz"], _ptr(cand["forced_lo"]),
                                     _ptr(cand["forced_hi"]), _ptr(row_ptr), _ptr(col), col.numel(), _ptr(st),
                                     ctypes.c_void_p(ws.data_ptr() + off), ws_bytes, _stream(stream)),
           "dynrad_build_token_mask")
    return row_ptr, col, st


def dynrad_proxy_error(lse_dense, lse_kept, lse2_dense, lse2_kept, stream=None):
    """(||A_dense - A_masked||_F^2, ||A_dense||_F^2) from four fp32 CUDA LSE vectors."""
    _require_cuda(lse_dense, lse_kept, lse2_dense, lse2_kept)
    out = torch.empty(2, dtype=torch.float64, device=lse_dense.device)
    _check(lib().dynrad_proxy_error(_ptr(lse_dense), _ptr(lse_kept), _ptr(lse2_dense), _ptr(lse2_kept),
                                    lse_dense.numel(), _ptr(out), _stream(stream)), "dynrad_proxy_error")
    return out


def dynrad_debug_attn_stall(wait_ns: int = 0, stall_step: int = -1) -> None:
    """Test hook of the attention forward's failure path: limit (ns) of its
    pipeline waits and the step at which its MMA warp waits for a barrier
    nothing completes; (0, -1) restores normal operation.  Process-wide."""
    _check(lib().dynrad_debug_attn_stall(int(wait_ns), int(stall_step)), "dynrad_debug_attn_stall")
