#!/usr/bin/env python
"""Benchmark of the DynamicRad block-sparse attention hot path on one B200.

One step = one pass of the whole path -- candidates (stage 1), pooling +
scoring + selection into CSR (stage 2), block-sparse attention (stage 3) -- for
every run of the workload.  The default workload is the Wan2.1-14B-like 720p
layer (B=1, H=40, D=128, 21x45x80 = 75,600 tokens, B_s = 64) with its four
runs: static rho = 0.15 and dynamic tau = 0.9, each at gamma 0.3 and 0.7.

Prints ONE JSON line (rank 0).  ``value`` = effective TFLOP/s on kept blocks
(4 * D * sum over kept (I, J) of n_I * n_J, summed over the step's runs)
divided by the device time of the whole step, inputs resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle, bounded sample

With torchrun (N > 1) every rank runs the same step on its own GPU with its own
copy of the layer: weak scaling, no collective on the data path; the timed
region is bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time
from dataclasses import replace

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_candidate_b200.workloads import (  # noqa: E402
    WORKLOADS, bf16_bits_to_f64, head_tensor_bf16, make_qkv_bf16, shared_field, head_amplitudes)

METRIC = ("sparse-attn effective TFLOPS (kept blocks) at Wan-14B 720p, whole path "
          "(candidates + selection + attention) per step")
UNIT = "TFLOP/s"
KERNELS_PER_RUN = 5   # 3 candidate kernels, 1 selection kernel, 1 attention kernel


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def runs_of(wl):
    """[(label, mode, value, geometry)] of a workload."""
    out = []
    for mode, value, gamma in wl.runs:
        g = wl.geom if gamma is None else replace(wl.geom, gamma=gamma)
        out.append((f"{mode}_{value}_g{g.gamma}", mode, value, g))
    return out


def kept_flops(row_ptr: np.ndarray, col: np.ndarray, n: int, block: int, bh: int, d: int) -> float:
    """4 * d * sum over kept (I, J) of n_I * n_J (valid tokens only)."""
    nb = -(-n // block)
    nvalid = np.full(nb, block, dtype=np.int64)
    nvalid[-1] = n - (nb - 1) * block
    counts = np.diff(row_ptr)
    kept_tok = np.add.reduceat(nvalid[col], row_ptr[:-1]) if len(col) else np.zeros(len(counts))
    kept_tok = np.where(counts > 0, kept_tok, 0)
    rows_n = np.tile(nvalid, bh)
    return float(4.0 * d * np.sum(rows_n.astype(np.float64) * kept_tok))


def backward_tile_fill(row_ptr: np.ndarray, col: np.ndarray, bh: int, nb: int, block: int):
    """Share of the backward's tensor-core tile area that kept pairs fill, per
    side: a 128-row tile (128 / block blocks) streams the union of its blocks'
    lists in 64-row steps, and a step's rows whose block lacks the member are
    masked.  (dQ side: tiles of query blocks over their kept lists; dK/dV side:
    tiles of key blocks over the query blocks that keep them.)"""
    r = 128 // block
    rows = np.repeat(np.arange(bh * nb, dtype=np.int64), np.diff(row_ptr[: bh * nb + 1]))
    head, qb = rows // nb, rows % nb
    useful = float(len(col))
    out = {}
    for side, tile_blk, member in (("dq", qb, col), ("dkv", col, qb)):
        key = (head * nb + tile_blk // r) * nb + member
        steps = len(np.unique(key)) * max(1, block // 64)   # a 32-row block fills half a step
        out[side] = round(useful * block * block / (steps * 128.0 * 64.0), 4)
    return out


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank timing over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def attention_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("attention.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_candidate_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it was
    taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "sparse_attn_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("source_sha") != attention_source_sha():
        return None
    return j.get("per_launch_bytes", {}).get(workload)


class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)}


# ----------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and --impl reference)
# ----------------------------------------------------------------------------
def oracle_sample(wl, n_rows: int, seed: int = 0, head: int = 0):
    """The float64 oracle on a bounded sample of the workload: for every run,
    candidates, scores and selection of ``n_rows`` sampled query blocks of one
    head, and their attention.  Returns (kept FLOPs processed, seconds)."""
    from threadpoolctl import threadpool_limits
    from oracle import attention as OA
    from oracle import geometry as OG
    from oracle import selection as OS

    with threadpool_limits(limits=1):
        f = shared_field(wl)
        amps = head_amplitudes(wl)
        q, k, v = (bf16_bits_to_f64(head_tensor_bf16(wl, t, 0, head, field_=f, amps=amps)) for t in "qkv")
        rng = np.random.default_rng(seed)
        flops = 0.0
        t0 = time.perf_counter()
        for _, mode, value, g in runs_of(wl):
            nb = g.n_blocks
            rows = sorted(rng.choice(nb, size=n_rows, replace=False).tolist())
            cand = OG.candidate_csr(g, rows=rows)
            qbar = OS.block_means(q, g.block)
            kbar = OS.block_means(k, g.block)
            for i, r in enumerate(rows):
                cols = cand["col"][cand["row_ptr"][i]:cand["row_ptr"][i + 1]]
                s = OS.block_scores(qbar, kbar, r, cols)
                kept = OS.select_row(mode, cols, s, int(cand["forced_lo"][i]), int(cand["forced_hi"][i]), value)
                keys = OA.block_key_tokens(g.block, g.n_tokens, kept)
                toks = np.arange(r * g.block, min((r + 1) * g.block, g.n_tokens))
                OA.attend_block(q[toks], k, v, keys, 1.0 / math.sqrt(q.shape[1]))
                flops += 4.0 * q.shape[1] * len(toks) * len(keys)
        return flops, time.perf_counter() - t0


def _oracle_worker(job):
    """One process of the parallel CPU leg: generate its head's inputs, wait
    for every worker, then run oracle_sample on that head (1 BLAS thread).
    Returns (kept FLOPs, seconds, start time, end time)."""
    wl, n_rows, seed, head, barrier = job
    oracle_sample(wl, 1, seed=seed + 7919, head=head)     # warm imports and caches
    barrier.wait(timeout=600)
    t0 = time.time()
    f, s = oracle_sample(wl, n_rows, seed=seed, head=head)
    return f, s, t0, time.time()


def _barrier_worker(args):
    return _oracle_worker(args[:4] + (_BARRIER,))


_BARRIER = None


def _init_worker(barrier):
    global _BARRIER
    _BARRIER = barrier


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample_parallel(wl, n_rows: int, seed: int = 0, workers: int = 0):
    """The float64 oracle on all usable host cores: one spawned process per core
    (1 BLAS thread each), worker i on head i mod H with its own row sample; the
    workers start together.  Returns (kept FLOPs, wall seconds of the parallel
    section, workers)."""
    import multiprocessing as mp
    workers = workers or usable_cores()
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(workers)
    jobs = [(wl, n_rows, seed + 101 * i, i % wl.heads) for i in range(workers)]
    with ctx.Pool(workers, initializer=_init_worker, initargs=(barrier,)) as pool:
        # bounded: a worker that cannot start (or dies) ends the leg with an error
        res = pool.map_async(_barrier_worker, jobs, chunksize=1).get(timeout=900)
    flops = sum(r[0] for r in res)
    wall = max(r[3] for r in res) - min(r[2] for r in res)
    return flops, wall, workers


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    n_rows = args.ref_rows
    for _ in range(args.warmup if args.warmup < 1 else 1):
        oracle_sample(wl, 1, seed=999)
    tot_f, tot_s = 0.0, 0.0
    cores = usable_cores()
    for i in range(args.steps):
        f, s, cores = oracle_sample_parallel(wl, n_rows, seed=i)
        tot_f += f
        tot_s += s
    value = tot_f / tot_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": f"per step: {cores} processes (one per usable host core, 1 BLAS thread each), "
                                   f"process i on head i mod {wl.heads}, {n_rows} random query blocks per run x "
                                   f"{len(wl.runs)} runs, full path (candidates, scores, selection, attention)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(wl, args):
    g = wl.geom
    return {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
            "grid": [g.frames, g.height, g.width], "tokens": g.n_tokens, "block": g.block,
            "runs": [lbl for lbl, *_ in runs_of(wl)],
            "l2": "inputs larger than L2 (Q/K/V %.2f GB per step)" % (3 * wl.batch * wl.heads * g.n_tokens *
                                                                      wl.head_dim * 2 / 1e9),
            "parallelism": (("heads x%d (strong scaling, one layer split by heads, no collective)" % args.gpus)
                            if getattr(args, "shard", "replicas") == "heads" and args.gpus > 1 else
                            ("replicas x%d (weak scaling, one layer per GPU, no collective)" % args.gpus))}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dynrad", choices=["dynrad", "reference"])
    ap.add_argument("--workload", default="wan14b_720p", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sampled", action="store_true",
                    help="skip the paper-exact static-ratio (seeded sampling) measurement")
    ap.add_argument("--sampled-rho", default="0.3,0.1", help="rho_1,rho_2 of the sampled static mode")
    ap.add_argument("--sampled-theta", default="0.2,0.5",
                    help="theta_c,theta_m (block aggregation) of the sampled static mode")
    ap.add_argument("--no-token", action="store_true",
                    help="skip the paper-exact dynamic-threshold (token-level) measurement")
    ap.add_argument("--token-tau", default="0.0,1.0", help="tau_1,tau_2 of the token-level dynamic mode")
    ap.add_argument("--token-theta", default="0.2,0.5",
                    help="theta_c,theta_m (block aggregation) of the token-level dynamic mode")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the attention backward (dQ, dK, dV under the selected mask) measurement")
    ap.add_argument("--e2e-chunk", type=int, default=4,
                    help="(batch, head) rows per chunk of the end-to-end host path")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=12, help="query blocks per run in the CPU sample")
    ap.add_argument("--ref-rows", type=int, default=3, help="query blocks per run per reference step")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling a smaller case)")
    ap.add_argument("--run", type=int, default=-1, help="time only this run of the workload")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="with several ranks: every rank runs a whole layer (replicas, weak scaling) or its "
                         "range of the layer's heads (heads, strong scaling; no exchange is needed)")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.heads > 0:
        wl = replace(wl, heads=args.heads)
    if args.run >= 0:
        wl = replace(wl, runs=(wl.runs[args.run],))
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    import torch.distributed as dist
    from block_sparse_attention_candidate_b200 import abi

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    heads_sel = None
    if world > 1 and args.shard == "heads":
        from block_sparse_attention_candidate_b200.sharding import head_range
        h0, h1 = head_range(wl.heads, world, rank)
        heads_sel = range(h0, h1)
    B, H, D, N = wl.batch, (len(heads_sel) if heads_sel is not None else wl.heads), wl.head_dim, wl.n_tokens

    # inputs: seeded synthetic layer (host, pinned) -> HBM; with head sharding
    # only this rank's heads (each head's stream is independent of the others)
    bits = make_qkv_bf16(wl, heads=heads_sel)
    host = {t: torch.from_numpy(bits[t].view(np.int16)).view(torch.bfloat16).pin_memory() for t in "qkv"}
    del bits
    q, k, v = (host[t].to(dev, non_blocking=False) for t in "qkv")
    torch.cuda.synchronize()

    runs = []
    for label, mode, value, g in runs_of(wl):
        cand = abi.dynrad_build_candidates(g)
        sel = abi.SelectBuffers(B, H, N, D, g, cand, dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        runs.append({"label": label, "mode": mode, "value": value, "geom": g, "cand": cand, "sel": sel,
                     "o": o, "lse": lse})

    stream = torch.cuda.current_stream()

    def run_path(r, qq, kk, vv, ev=None):
        if ev is not None:
            ev[0].record(stream)
        abi.dynrad_build_candidates_into(r["geom"], r["cand"])
        if ev is not None:
            ev[1].record(stream)
        abi.dynrad_select_blocks(qq, kk, r["geom"], r["cand"], r["mode"], r["value"], buffers=r["sel"])
        if ev is not None:
            ev[2].record(stream)
        abi.dynrad_sparse_attn(qq, kk, vv, r["geom"].block, r["sel"].row_ptr, r["sel"].col_idx,
                               out=r["o"], lse=r["lse"])
        if ev is not None:
            ev[3].record(stream)

    def step(ev_list=None):
        for i, r in enumerate(runs):
            run_path(r, q, k, v, None if ev_list is None else ev_list[i])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = abi.dynrad_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {abi.status_string(st)}")

    # kept work (selection is deterministic: the CSR is the same every step)
    flops_run = []
    for r in runs:
        rp = r["sel"].row_ptr.cpu().numpy().astype(np.int64)
        col = r["sel"].col_idx[: int(rp[-1])].cpu().numpy().astype(np.int64)
        flops_run.append(kept_flops(rp, col, N, r["geom"].block, B * H, D))
        nb = r["geom"].n_blocks
        r["kept_blocks"] = int(rp[-1])
        r["density"] = int(rp[-1]) / (B * H * nb * nb)
    flops_step = sum(flops_run)

    # ---- timed region: K steps, device time
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler("GPU-" + uuid if not uuid.startswith("GPU-") else uuid)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in runs] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for s in range(args.steps):
        step(ev[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    ms_step = total_ms / args.steps
    st = abi.dynrad_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status after timing: {abi.status_string(st)}")

    stage_ms = np.zeros((len(runs), 3))
    for s in range(args.steps):
        for i in range(len(runs)):
            e = ev[s][i]
            stage_ms[i] += [e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
    stage_ms /= args.steps
    attn_ms_total = float(stage_ms[:, 2].sum())

    peaks = load_peaks()
    # whole-job work: every rank's kept FLOPs (replicas: world copies of one
    # layer; head shards: the parts of one layer)
    flops_job = flops_step
    if world > 1:
        t = torch.tensor([flops_step], dtype=torch.float64, device=dev)
        dist.all_reduce(t)
        flops_job = float(t.item())
    value = flops_job / (ms_step * 1e-3) / 1e12
    achieved = flops_step / (attn_ms_total * 1e-3) / 1e12
    traffic = recorded_traffic(wl.name)

    # ---- per-run details, dense run of the same kernel
    qk_bytes = 2.0 * B * H * N * D * 2
    run_info = {}
    for i, r in enumerate(runs):
        g = r["geom"]
        run_info[r["label"]] = {
            "stage1_ms": round(stage_ms[i, 0], 4), "stage2_ms": round(stage_ms[i, 1], 4),
            "attn_ms": round(stage_ms[i, 2], 4),
            "attn_tflops": round(flops_run[i] / (stage_ms[i, 2] * 1e-3) / 1e12, 1),
            "stage2_gbs_qk": round(qk_bytes / (stage_ms[i, 1] * 1e-3) / 1e9, 1),
            "kept_blocks": r["kept_blocks"], "block_density": round(r["density"], 4),
            "kept_tflop": round(flops_run[i] / 1e12, 3),
            "cand_nnz_per_head": r["cand"]["nnz"],
        }
    dense = None
    if not args.no_dense:
        g0 = runs[0]["geom"]
        nb = g0.n_blocks
        rp = (torch.arange(B * H * nb + 1, device=dev, dtype=torch.int64) * nb).to(torch.int32)
        col = torch.arange(nb, device=dev, dtype=torch.int32).repeat(B * H * nb)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for _ in range(2):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp, col, out=o, lse=lse)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp, col, out=o, lse=lse)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / reps
        dense_flops = 4.0 * D * B * H * float(N) * float(N)
        dense = {"ms": round(dense_ms, 3), "tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 1),
                 "speedup_vs_dense": {lbl: round(dense_ms / ri["attn_ms"], 2) for lbl, ri in run_info.items()}}
        del rp, col, o, lse

    # ---- paper-exact static-ratio mode (Eq. 8 seeded token-pair sampling): mask
    # build (content-free, cacheable) and the attention over it
    sampled = None
    if not args.no_sampled:
        rho1, rho2 = (float(x) for x in args.sampled_rho.split(","))
        th_c, th_m = (float(x) for x in args.sampled_theta.split(","))
        g0 = replace(runs[0]["geom"], theta_c=th_c, theta_m=th_m)
        cand0 = abi.dynrad_build_candidates(g0)
        rp_s, col_s, _ = abi.dynrad_build_sampled_mask(g0, cand0, rho1, rho2, 2026, replicas=B * H)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_build_sampled_mask(g0, cand0, rho1, rho2, 2026, replicas=B * H)
        e1.record(stream)
        torch.cuda.synchronize()
        build_ms = e0.elapsed_time(e1) / reps
        o_s = torch.empty_like(q)
        lse_s = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for _ in range(2):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp_s, col_s, out=o_s, lse=lse_s)
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp_s, col_s, out=o_s, lse=lse_s)
        e1.record(stream)
        torch.cuda.synchronize()
        st = abi.dynrad_device_status(clear=True)
        if st != 0:
            raise RuntimeError(f"device status after the sampled-mask run: {abi.status_string(st)}")
        attn_s = e0.elapsed_time(e1) / reps
        rpn = rp_s.cpu().numpy().astype(np.int64)
        coln = col_s[: int(rpn[-1])].cpu().numpy().astype(np.int64)
        fl = kept_flops(rpn, coln, N, g0.block, B * H, D)
        nb0 = g0.n_blocks
        sampled = {"rho1": rho1, "rho2": rho2, "theta_c": th_c, "theta_m": th_m, "seed": 2026, "gamma": g0.gamma,
                   "mask_build_ms": round(build_ms, 3), "attn_ms": round(attn_s, 3),
                   "attn_tflops": round(fl / (attn_s * 1e-3) / 1e12, 1),
                   "block_density": round(int(rpn[-1]) / (B * H * nb0 * nb0), 4),
                   "candidate_density": round(cand0["nnz"] / (nb0 * nb0), 4),
                   "speedup_vs_dense": round(dense["ms"] / attn_s, 2) if dense else None}
        del rp_s, col_s, o_s, lse_s

    # ---- paper-exact dynamic-threshold mode (Eqs. 9-11, 19: token-level proxy
    # logits of the first two heads): mask build and the attention over it
    token = None
    if not args.no_token:
        t1, t2 = (float(x) for x in args.token_tau.split(","))
        th_c, th_m = (float(x) for x in args.token_theta.split(","))
        g0 = replace(runs[0]["geom"], theta_c=th_c, theta_m=th_m)
        cand0 = abi.dynrad_build_candidates(g0)
        rp_t, col_t, _ = abi.dynrad_build_token_mask(q, k, g0, cand0, t1, t2, hf=2)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_build_token_mask(q, k, g0, cand0, t1, t2, hf=2)
        e1.record(stream)
        torch.cuda.synchronize()
        build_ms = e0.elapsed_time(e1) / reps
        o_t = torch.empty_like(q)
        lse_t = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for _ in range(2):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp_t, col_t, out=o_t, lse=lse_t)
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_sparse_attn(q, k, v, g0.block, rp_t, col_t, out=o_t, lse=lse_t)
        e1.record(stream)
        torch.cuda.synchronize()
        st = abi.dynrad_device_status(clear=True)
        if st != 0:
            raise RuntimeError(f"device status after the token-mask run: {abi.status_string(st)}")
        attn_t = e0.elapsed_time(e1) / reps
        rpn = rp_t.cpu().numpy().astype(np.int64)
        coln = col_t[: int(rpn[-1])].cpu().numpy().astype(np.int64)
        fl = kept_flops(rpn, coln, N, g0.block, B * H, D)
        nb0 = g0.n_blocks
        token = {"tau1": t1, "tau2": t2, "theta_c": th_c, "theta_m": th_m, "fused_heads": 2, "gamma": g0.gamma,
                 "mask_build_ms": round(build_ms, 3), "attn_ms": round(attn_t, 3),
                 "attn_tflops": round(fl / (attn_t * 1e-3) / 1e12, 1),
                 "block_density": round(int(rpn[-1]) / (B * H * nb0 * nb0), 4),
                 "candidate_density": round(cand0["nnz"] / (nb0 * nb0), 4),
                 "speedup_vs_dense": round(dense["ms"] / attn_t, 2) if dense else None}
        del rp_t, col_t, o_t, lse_t

    # ---- backward of the attention under the first run's selected mask (the
    # gradient the mask-aware fine-tuning trains through), dO seeded N(0, 1)
    backward = None
    if not args.no_backward:
        r0 = runs[0]
        gen = torch.Generator(device=dev)
        gen.manual_seed(2027)
        dout = torch.randn(q.shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        grads = tuple(torch.empty_like(q) for _ in range(3))
        rp0, col0 = r0["sel"].row_ptr, r0["sel"].col_idx
        bws = torch.empty(abi.lib().dynrad_attn_backward_workspace_bytes(B, H, N, r0["geom"].block, col0.numel()),
                          dtype=torch.uint8, device=dev)
        run_path(r0, q, k, v)
        for _ in range(2):
            abi.dynrad_attn_backward(q, k, v, r0["o"], r0["lse"], dout, r0["geom"].block, rp0, col0,
                                     grads=grads, workspace=bws)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            abi.dynrad_attn_backward(q, k, v, r0["o"], r0["lse"], dout, r0["geom"].block, rp0, col0,
                                     grads=grads, workspace=bws)
        e1.record(stream)
        torch.cuda.synchronize()
        st = abi.dynrad_device_status(clear=True)
        if st != 0:
            raise RuntimeError(f"device status after the backward run: {abi.status_string(st)}")
        bwd_ms = e0.elapsed_time(e1) / reps
        # algorithmic backward FLOPs: S, dP, dV, dQ, dK products, 2.5x the forward's
        bflops = 2.5 * flops_run[0]
        rpn = rp0.cpu().numpy().astype(np.int64)
        coln = col0[: int(rpn[-1])].cpu().numpy().astype(np.int64)
        backward = {"run": r0["label"], "ms": round(bwd_ms, 3), "tflops": round(bflops / (bwd_ms * 1e-3) / 1e12, 1),
                    "fwd_attn_ms": run_info[r0["label"]]["attn_ms"], "flop_model": "10 * D per kept (query, key)",
                    "tile_fill": backward_tile_fill(rpn, coln, B * H, r0["geom"].n_blocks, r0["geom"].block)}
        del dout, grads, bws

    # ---- end to end through the host-memory entry point: pinned host Q, K, V
    # in, every run's O and LSE back to pinned host memory, the copies
    # overlapped with the kernels by dynrad_host_path (chunks of heads)
    e2e = None
    if not args.no_e2e:
        del q, k, v
        for r in runs:
            del r["o"], r["lse"]
        torch.cuda.empty_cache()
        hruns = [{"geom": r["geom"], "cand": r["cand"], "mode": r["mode"], "value": r["value"],
                  "o_host": torch.empty((B, H, N, D), dtype=torch.bfloat16, pin_memory=True),
                  "lse_host": torch.empty((B, H, N), dtype=torch.float32, pin_memory=True)} for r in runs]
        hws = abi.HostPathWorkspace(B, H, N, D, hruns, args.e2e_chunk, dev)
        h2d = 3 * B * H * N * D * 2
        d2h = len(runs) * (B * H * N * D * 2 + B * H * N * 4)

        def e2e_step():
            for r in runs:
                abi.dynrad_build_candidates_into(r["geom"], r["cand"])
            abi.dynrad_host_path(host["q"], host["k"], host["v"], hruns, chunk_bh=args.e2e_chunk, workspace=hws)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        st = abi.dynrad_device_status(clear=True)
        if st != 0:
            raise RuntimeError(f"device status after the end-to-end run: {abi.status_string(st)}")
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), dev)
        e2e = {"value": flops_job * args.steps / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.steps,
               "path": f"dynrad_host_path, pinned host buffers, chunks of {args.e2e_chunk} heads"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f1, s1 = oracle_sample(wl, args.cpu_rows, seed=12345)
        fa, sa, nw = oracle_sample_parallel(wl, args.cpu_rows, seed=12345)
        cpu = {"value": fa / sa / 1e12, "unit": UNIT, "cores": nw, "cpu_model": cpu_model(), "kind": "oracle",
               "seconds": round(sa, 2),
               "sample": f"{nw} processes (one per usable host core, 1 BLAS thread each), process i on head "
                         f"i mod {wl.heads}, {args.cpu_rows} random query blocks per run x {len(runs)} runs each; "
                         f"full path (candidates, scores, selection, attention) in float64 numpy; value = all "
                         f"processes' kept FLOPs / wall time of the parallel section",
               "single_core": {"value": f1 / s1 / 1e12, "cores": 1, "seconds": round(s1, 2),
                               "sample": f"head 0, {args.cpu_rows} random query blocks per run x {len(runs)} runs"}}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if heads_sel is not None else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded correlated Fourier field + noise)",
        "config": workload_config(wl, args),
        "roofline": {"kernel": "sparse_attn_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_source": peaks["source"] + " bf16 burst",
                     "frac_of_sustained": (round(achieved / peaks["bf16_tflops_sustained"], 4)
                                           if peaks.get("bf16_tflops_sustained") else None),
                     "traffic": traffic},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": KERNELS_PER_RUN * len(runs) * args.steps,
        "clocks": clocks,
        "runs": run_info,
        "dense_same_kernel": dense,
        "sampled_static": sampled,
        "token_dynamic": token,
        "backward": backward,
        "stage_ms_per_step": {"candidates": round(float(stage_ms[:, 0].sum()), 4),
                              "selection": round(float(stage_ms[:, 1].sum()), 4),
                              "attention": round(attn_ms_total, 4)},
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
