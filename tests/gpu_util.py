"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle on
the same seeded inputs, compare."""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import (
    bf16_bits_to_f64, make_qkv_bf16, round_to_bf16_bits)
from oracle import attention as OA
from oracle import geometry as OG
from oracle import selection as OS

# Tolerances (GPU vs float64 oracle on identical bf16 inputs)
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
# fp32 block scores: a 128-term fp32 dot product of fp32 means; relative to
# the scale |qbar| |kbar| / sqrt(d) of the products summed
SCORE_REL = 2e-5
# dynamic-mode decisions closer than this (relative to Z) to tau * Z may go
# either way (GPU: exact 36-bit fixed-point sums; oracle: exactly rounded fp64)
AMBIGUOUS_GAP = 1e-8


def bits_to_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)


def gpu_inputs(qkv_bits: dict, device="cuda"):
    return tuple(bits_to_tensor(qkv_bits[t], device) for t in "qkv")


def check_device_status():
    st = abi.dynrad_device_status(clear=True)
    assert st == 0, f"device status {st}: {abi.status_string(st)}"


def cand_to_numpy(cand):
    return {k: cand[k].cpu().numpy().astype(np.int64) for k in ("row_ptr", "col", "forced_lo", "forced_hi")}


def csr_rows(row_ptr: np.ndarray, col: np.ndarray, bh: int, nb: int):
    """Per-row kept lists of one (b, h) slice of the flat CSR."""
    base = bh * nb
    return [col[row_ptr[base + r]:row_ptr[base + r + 1]] for r in range(nb)]


def compare_selection(mode, value, cand_np, kept_rows, scores_flat, bh, nb, cand_nnz, rows=None):
    """Oracle selection fed the GPU's fp32 scores; indices must match exactly
    except rows whose dynamic decision is within AMBIGUOUS_GAP of tau.
    Returns the number of ambiguous rows."""
    ambiguous = 0
    rows = range(nb) if rows is None else rows
    for r in rows:
        a, b = int(cand_np["row_ptr"][r]), int(cand_np["row_ptr"][r + 1])
        cols = cand_np["col"][a:b]
        s = scores_flat[bh * cand_nnz + a: bh * cand_nnz + b].astype(np.float64)
        lo, hi = int(cand_np["forced_lo"][r]), int(cand_np["forced_hi"][r])
        if mode == "static":
            want = OS.select_static(cols, s, lo, hi, value)
        else:
            want, info = OS.dynamic_cut(cols, s, lo, hi, value)
            if info["ambiguous_gap"] < AMBIGUOUS_GAP and not np.array_equal(want, kept_rows[r]):
                ambiguous += 1
                continue
        assert np.array_equal(want, kept_rows[r]), (mode, value, bh, r, want, kept_rows[r])
    return ambiguous


def compare_attention(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray,
                      what=""):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    assert err.max() <= O_MAX_ABS, f"{what}: max |O err| {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: mean |O err| {err.mean():.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse_gpu)), f"{what}: LSE finiteness differs"
    if fin.any():
        le = np.abs(lse_gpu[fin].astype(np.float64) - lse_ref[fin])
        assert le.max() <= LSE_ABS, f"{what}: max |LSE err| {le.max():.3e}"
    return float(err.max()), float(err.mean())


def full_csr(nb: int, bh_count: int):
    rp = (np.arange(bh_count * nb + 1, dtype=np.int64) * nb)
    col = np.tile(np.arange(nb, dtype=np.int64), bh_count * nb)
    return rp, col
