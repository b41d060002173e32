"""The seeded input generator shared by both sides (no GPU): bf16 rounding,
regenerability of single heads, determinism and the field's statistics."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import workloads as W


def test_bf16_rounding_matches_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10,
                        # exact ties between two bf16 neighbours (the low 16 bits are 0x8000)
                        (rng.integers(0x3F800000 >> 16, 0x47000000 >> 16, 2000).astype(np.uint32) << 16
                         | np.uint32(0x8000)).view(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40], dtype=np.float32)])
    got = W.round_to_bf16_bits(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_bf16_bits_decode_exactly():
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]            # finite values only
    got = W.bf16_bits_to_f64(bits)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(W.round_to_bf16_bits(got.astype(np.float32)), bits)


def test_single_heads_regenerate_and_thread_count_does_not_matter():
    wl = W.WORKLOADS["wan14b_480p"]                      # per-head amplitudes
    full = W.make_qkv_bf16(wl, heads=[0, 1, 2, 3], threads=1)
    for h in (3, 1):
        one = W.make_qkv_bf16(wl, heads=[h], threads=4)
        for t in "qkv":
            np.testing.assert_array_equal(one[t][:, 0], full[t][:, h])
            np.testing.assert_array_equal(one[t][0, 0], W.head_tensor_bf16(wl, t, 0, h))


def test_generation_is_deterministic_and_tensors_differ():
    wl = W.WORKLOADS["tiny"]
    a, b = W.make_qkv_bf16(wl), W.make_qkv_bf16(wl, threads=1)
    for t in "qkv":
        np.testing.assert_array_equal(a[t], b[t])
    assert not np.array_equal(a["q"], a["k"]) and not np.array_equal(a["k"], a["v"])
    assert not np.array_equal(a["q"][0, 0], a["q"][0, 1])


def test_field_statistics_and_amplitudes():
    wl = W.WORKLOADS["wan13b_480p"]
    f = W.shared_field(wl).astype(np.float64)
    assert f.shape == (wl.n_tokens, wl.head_dim)
    rms = np.sqrt((f ** 2).mean(axis=0))                 # unit RMS per channel in expectation
    assert 0.5 < rms.mean() < 1.5
    amps = W.head_amplitudes(W.WORKLOADS["wan14b_480p"])
    lo, hi = W.WORKLOADS["wan14b_480p"].amp_range
    assert amps.shape == (1, 40) and np.all(amps >= lo) and np.all(amps <= hi) and amps.std() > 0.05
    np.testing.assert_array_equal(W.head_amplitudes(wl), np.full((1, wl.heads), wl.amp))
    # a head's tensor is amp * field + unit noise: its correlation with the field
    q = W.head_tensor_f32(wl, "q", 0, 0).astype(np.float64)
    c = (q * f).sum() / math.sqrt((q * q).sum() * (f * f).sum())
    want = wl.amp * rms.mean() / math.sqrt(wl.amp ** 2 * (rms ** 2).mean() + 1.0)
    assert abs(c - want) < 0.05
