"""Seeded synthetic workloads: the five attention-layer shapes and their Q/K/V.

This module only draws numbers.  It holds none of the method's arithmetic (no
window, no pooling, no selection, no softmax), so that both the CPU oracle
(via the tests) and the CUDA path can be fed the same bytes.

Recipe (one reading of "spatiotemporally correlated Q/K/V shaped like the
Wan2.1 and HunyuanVideo attention layers"):

* A shared low-frequency field F(t, h, w) in R^D, sum of 8 random Fourier modes
  a_m * cos(2*pi*(ft*t/F + fh*h/Hh + fw*w/W) + phi_m) with integer wave numbers
  ft in {0,1,2}, fh, fw in {-2..2}, a_m ~ N(0, (2/8) I_D) (unit RMS per channel)
  and phi_m ~ U[0, 2*pi)^D.
* Q, K and V of every (batch, head) are amp * F + N(0, 1) with independent noise.
  amp = 0.7, or per head U[0.3, 1.0] where a workload asks for it.
* The HunyuanVideo-like workload adds a second 8-mode field G that translates
  along w at 2 latent px per frame: (F(t,h,w) + G(h, w - 2t)) / sqrt(2).
* Values are drawn in fp32 and rounded to bf16 (round to nearest even); the
  bf16 bits are what both sides consume.
* Every stream comes from numpy PCG64 seeded through SeedSequence(seed).spawn,
  one child per purpose and one grandchild per (tensor, batch, head), so a
  single head can be regenerated on its own at any size.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np


@dataclass(frozen=True)
class Geometry:
    """Latent token grid and the radial-window parameters (DynamicRad, Sec. 3.1)."""
    frames: int
    height: int
    width: int
    block: int
    gamma: float
    lam: float
    theta_c: float = 0.0
    theta_m: float = 0.0
    eps: float = 1e-6
    force_t: int = 1

    @property
    def tokens_per_frame(self) -> int:
        return self.height * self.width

    @property
    def n_tokens(self) -> int:
        return self.frames * self.height * self.width

    @property
    def n_blocks(self) -> int:
        return -(-self.n_tokens // self.block)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    geom: Geometry
    seed: int
    # (mode, value, geometry override of gamma or None)
    runs: tuple = ()
    amp: float = 0.7
    amp_range: Optional[tuple] = None   # per-head U[lo, hi] amplitude
    translate_px: int = 0               # translating component, latent px/frame
    fp32_inputs: bool = False           # the workload is specified in fp32

    @property
    def n_tokens(self) -> int:
        return self.geom.n_tokens

    def with_gamma(self, gamma: float) -> "Workload":
        return replace(self, geom=replace(self.geom, gamma=gamma))


STATIC = "static"
DYNAMIC = "dynamic"

WORKLOADS = {
    "tiny": Workload(
        "tiny", 1, 2, 64, Geometry(4, 16, 16, 32, 0.5, 2.0), seed=0,
        runs=((STATIC, 0.25, None), (DYNAMIC, 0.8, None)), fp32_inputs=True),
    "wan13b_480p": Workload(
        "wan13b_480p", 1, 12, 128, Geometry(21, 30, 52, 64, 0.5, 4.0), seed=1,
        runs=((STATIC, 0.2, None),)),
    "wan14b_480p": Workload(
        "wan14b_480p", 1, 40, 128, Geometry(21, 30, 52, 64, 0.5, 4.0), seed=2,
        runs=((DYNAMIC, 0.8, None),), amp_range=(0.3, 1.0)),
    "wan14b_720p": Workload(
        "wan14b_720p", 1, 40, 128, Geometry(21, 45, 80, 64, 0.3, 4.0), seed=3,
        runs=((STATIC, 0.15, 0.3), (STATIC, 0.15, 0.7),
              (DYNAMIC, 0.9, 0.3), (DYNAMIC, 0.9, 0.7))),
    "hunyuan_720p": Workload(
        "hunyuan_720p", 1, 24, 128, Geometry(33, 45, 80, 128, 0.4, 8.0), seed=4,
        runs=((DYNAMIC, 0.8, None),), translate_px=2),
}


# ----------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------
_FIELD, _AMP, _NOISE, _TRANSLATE = range(4)
_TENSORS = ("q", "k", "v")


def _children(seed: int):
    return np.random.SeedSequence(seed).spawn(4)


def _fourier_field(rng: np.random.Generator, frames: int, height: int, width: int,
                   dim: int, n_modes: int = 8, shift_px: int = 0,
                   use_time: bool = True) -> np.ndarray:
    """Sum of n_modes random cosines over the (t, h, w) grid -> float32 [N, dim].

    With shift_px != 0 the field is sampled at w - shift_px * t, periodic in w,
    and has no own time dependence (a pattern translating along w)."""
    ft = rng.integers(0, 3, size=n_modes) if use_time else np.zeros(n_modes, np.int64)
    fh = rng.integers(-2, 3, size=n_modes)
    fw = rng.integers(-2, 3, size=n_modes)
    amp = rng.normal(0.0, math.sqrt(2.0 / n_modes), size=(n_modes, dim))
    phase = rng.uniform(0.0, 2.0 * math.pi, size=(n_modes, dim))
    t = np.arange(frames, dtype=np.float64)[:, None, None]
    h = np.arange(height, dtype=np.float64)[None, :, None]
    w = np.arange(width, dtype=np.float64)[None, None, :]
    w_eff = w - shift_px * t
    out = np.zeros((frames * height * width, dim), dtype=np.float32)
    for m in range(n_modes):
        arg = 2.0 * math.pi * (ft[m] * t / frames + fh[m] * h / height + fw[m] * w_eff / width)
        arg = np.broadcast_to(arg, (frames, height, width)).reshape(-1, 1)
        out += (amp[m][None, :] * np.cos(arg + phase[m][None, :])).astype(np.float32)
    return out


def shared_field(wl: Workload) -> np.ndarray:
    """The field shared by Q, K, V and all heads (float32 [N, D])."""
    g = wl.geom
    ss = _children(wl.seed)
    f = _fourier_field(np.random.Generator(np.random.PCG64(ss[_FIELD])),
                       g.frames, g.height, g.width, wl.head_dim)
    if wl.translate_px:
        gfield = _fourier_field(np.random.Generator(np.random.PCG64(ss[_TRANSLATE])),
                                g.frames, g.height, g.width, wl.head_dim,
                                shift_px=wl.translate_px, use_time=False)
        f = ((f + gfield) / np.float32(math.sqrt(2.0))).astype(np.float32)
    return f


def head_amplitudes(wl: Workload) -> np.ndarray:
    """Field amplitude per (batch, head), float64 [B, H]."""
    if wl.amp_range is None:
        return np.full((wl.batch, wl.heads), wl.amp, dtype=np.float64)
    ss = _children(wl.seed)
    rng = np.random.Generator(np.random.PCG64(ss[_AMP]))
    lo, hi = wl.amp_range
    return rng.uniform(lo, hi, size=(wl.batch, wl.heads))


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.  Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _noise_seed(wl: Workload, tensor: int, b: int, h: int) -> np.random.SeedSequence:
    ss_noise = _children(wl.seed)[_NOISE]
    # grandchild index (tensor, b, h) -> a fixed spawn key, independent of sizes
    return np.random.SeedSequence(ss_noise.entropy,
                                  spawn_key=tuple(ss_noise.spawn_key) + (tensor, b, h))


def head_tensor_f32(wl: Workload, tensor: str, b: int, h: int,
                    field_: Optional[np.ndarray] = None,
                    amps: Optional[np.ndarray] = None) -> np.ndarray:
    """fp32 values of one (tensor, batch, head) slice, [N, D]."""
    ti = _TENSORS.index(tensor)
    if field_ is None:
        field_ = shared_field(wl)
    if amps is None:
        amps = head_amplitudes(wl)
    rng = np.random.Generator(np.random.PCG64(_noise_seed(wl, ti, b, h)))
    noise = rng.standard_normal(field_.shape, dtype=np.float32)
    noise += np.float32(amps[b, h]) * field_
    return noise


def head_tensor_bf16(wl: Workload, tensor: str, b: int, h: int, **kw) -> np.ndarray:
    """bf16 bits (uint16 [N, D]) of one (tensor, batch, head) slice."""
    return round_to_bf16_bits(head_tensor_f32(wl, tensor, b, h, **kw))


def make_qkv_bf16(wl: Workload, heads: Optional[Sequence[int]] = None,
                  threads: int = 0) -> dict:
    """Q, K, V as bf16 bits, uint16 [B, H', N, D] for the selected heads.

    Heads are generated independently (one noise stream each), in parallel
    threads; the result does not depend on the thread count."""
    heads = list(range(wl.heads)) if heads is None else list(heads)
    f = shared_field(wl)
    amps = head_amplitudes(wl)
    n, d = wl.n_tokens, wl.head_dim
    out = {t: np.empty((wl.batch, len(heads), n, d), dtype=np.uint16) for t in _TENSORS}
    jobs = [(t, b, hi, h) for t in _TENSORS for b in range(wl.batch) for hi, h in enumerate(heads)]

    def run(job):
        t, b, hi, h = job
        out[t][b, hi] = head_tensor_bf16(wl, t, b, h, field_=f, amps=amps)

    nthreads = threads or min(16, len(jobs), max(1, (__import__("os").cpu_count() or 1)))
    if nthreads <= 1:
        for j in jobs:
            run(j)
    else:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(run, jobs))
    return out


def make_qkv_f32(wl: Workload) -> dict:
    """Q, K, V in fp32 ([B, H, N, D]); used only for the fp32 information run."""
    f = shared_field(wl)
    amps = head_amplitudes(wl)
    return {t: np.stack([np.stack([head_tensor_f32(wl, t, b, h, field_=f, amps=amps)
                                   for h in range(wl.heads)]) for b in range(wl.batch)])
            for t in _TENSORS}


def random_qkv_bf16(seed: int, batch: int, heads: int, n: int, dim: int,
                    scale: float = 1.0) -> dict:
    """Unstructured N(0, scale^2) Q/K/V as bf16 bits, for edge-case tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return {t: round_to_bf16_bits(rng.standard_normal((batch, heads, n, dim), dtype=np.float32)
                                  * np.float32(scale))
            for t in _TENSORS}


# ---------------------------------------------------------------------------
# Feature-drift proxy (DynamicRad, Appendix C.2, Eq. 20): the synthetic task the
# offline parameter search is run on.  This draws the features only; the
# proxy attention matrix and the objective are computed elsewhere.
# ---------------------------------------------------------------------------
DRIFT_REGIMES = {"low": 0.02, "mid": 0.15, "high": 0.40}


def ar_features(seed: int, frames: int, tokens_per_frame: int, dim: int, delta: float) -> np.ndarray:
    """Hidden states h of every token, float32 [frames * tokens_per_frame, dim]:
    each spatial token position carries its own auto-regressive chain over the
    frames, h_0 ~ N(0, I), h_t = sqrt(1 - delta^2) h_{t-1} + delta eps_t with
    eps_t ~ N(0, I) (so every h_t is N(0, I))."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    h = np.empty((frames, tokens_per_frame, dim), dtype=np.float64)
    h[0] = rng.standard_normal((tokens_per_frame, dim))
    a = math.sqrt(1.0 - delta * delta)
    for t in range(1, frames):
        h[t] = a * h[t - 1] + delta * rng.standard_normal((tokens_per_frame, dim))
    return h.reshape(frames * tokens_per_frame, dim).astype(np.float32)
