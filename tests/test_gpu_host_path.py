"""dynrad_host_path (stages 2 and 3 from and to pinned host memory, copies
overlapped with the kernels in chunks of (batch, head) rows) against the
device-resident calls: every stage is independent per row, so each run's O and
LSE must be the same bits."""
import numpy as np
import pytest
import torch

from block_sparse_attention_candidate_b200 import abi
from block_sparse_attention_candidate_b200.workloads import WORKLOADS, make_qkv_bf16
from gpu_util import check_device_status

pytestmark = pytest.mark.gpu


def _host_inputs(wl):
    bits = make_qkv_bf16(wl)
    return {t: torch.from_numpy(bits[t].view(np.int16)).view(torch.bfloat16).pin_memory() for t in "qkv"}


def _device_reference(host, runs):
    q, k, v = (host[t].cuda() for t in "qkv")
    out = []
    for r in runs:
        rp, col, _ = abi.dynrad_select_blocks(q, k, r["geom"], r["cand"], r["mode"], r["value"])
        o, lse = abi.dynrad_sparse_attn(q, k, v, r["geom"].block, rp, col)
        out.append((o.cpu(), lse.cpu()))
    torch.cuda.synchronize()
    check_device_status()
    return out


def _runs(wl, settings, B, H, N, D):
    runs = []
    for mode, value, gamma in settings:
        g = wl.geom if gamma is None else wl.with_gamma(gamma).geom
        runs.append({"geom": g, "cand": abi.dynrad_build_candidates(g), "mode": mode, "value": value,
                     "o_host": torch.full((B, H, N, D), float("nan"), dtype=torch.bfloat16).pin_memory(),
                     "lse_host": torch.full((B, H, N), float("nan"), dtype=torch.float32).pin_memory()})
    return runs


@pytest.mark.parametrize("chunk", [5, 12, 64])
def test_host_path_matches_device_calls(chunk):
    wl = WORKLOADS["wan13b_480p"]                 # 12 heads x 32,760 tokens; chunk 5 leaves a ragged 2
    host = _host_inputs(wl)
    B, H, N, D = host["q"].shape
    runs = _runs(wl, [("static", 0.2, None), ("dynamic", 0.8, 0.7)], B, H, N, D)
    ref = _device_reference(host, runs)
    ws = abi.HostPathWorkspace(B, H, N, D, runs, chunk)
    for _ in range(2):                            # two calls in a row share the workspace
        for r in runs:
            r["o_host"].fill_(float("nan"))
            r["lse_host"].fill_(float("nan"))
        abi.dynrad_host_path(host["q"], host["k"], host["v"], runs, chunk_bh=chunk, workspace=ws)
        torch.cuda.current_stream().synchronize()
        check_device_status()
        for r, (o, lse) in zip(runs, ref):
            assert torch.equal(r["o_host"].view(torch.int16), o.view(torch.int16))
            assert torch.equal(r["lse_host"], lse)


def test_host_path_three_runs_alternate_queues():
    # (chunk, run) items alternate between two compute queues, each with its own
    # CSR and selection buffers: with three runs a queue serves different runs
    # (different geometries and kept counts) from one chunk to the next
    wl = WORKLOADS["wan13b_480p"]
    host = _host_inputs(wl)
    B, H, N, D = host["q"].shape
    runs = _runs(wl, [("static", 0.2, None), ("dynamic", 0.8, 0.7), ("static", 0.35, 0.3)], B, H, N, D)
    ref = _device_reference(host, runs)
    abi.dynrad_host_path(host["q"], host["k"], host["v"], runs, chunk_bh=5)
    torch.cuda.current_stream().synchronize()
    check_device_status()
    for r, (o, lse) in zip(runs, ref):
        assert torch.equal(r["o_host"].view(torch.int16), o.view(torch.int16))
        assert torch.equal(r["lse_host"], lse)


def test_host_path_tiny_single_chunk():
    wl = WORKLOADS["tiny"]
    host = _host_inputs(wl)
    B, H, N, D = host["q"].shape
    runs = _runs(wl, [(m, v, None) for m, v, _ in wl.runs], B, H, N, D)
    ref = _device_reference(host, runs)
    abi.dynrad_host_path(host["q"], host["k"], host["v"], runs, chunk_bh=B * H + 3)
    torch.cuda.current_stream().synchronize()
    check_device_status()
    for r, (o, lse) in zip(runs, ref):
        assert torch.equal(r["o_host"].view(torch.int16), o.view(torch.int16))
        assert torch.equal(r["lse_host"], lse)


def test_error_after_queued_copies_leaves_the_stream_joined():
    # the second run's rho is out of range, which dynrad_select_blocks reports at
    # chunk 0 after the first run's copy-in and copy-out of that chunk were
    # queued on the call's side streams; the call must still make the caller's
    # stream wait for them, so once the stream passes the call chunk 0 of the
    # first run is in host memory
    wl = WORKLOADS["wan13b_480p"]
    host = _host_inputs(wl)
    B, H, N, D = host["q"].shape
    runs = _runs(wl, [("static", 0.2, None), ("static", 2.0, None)], B, H, N, D)
    ref = _device_reference(host, runs[:1])
    chunk = 2                                     # chunk 0 = rows 0 and 1
    ws = abi.HostPathWorkspace(B, H, N, D, runs, chunk)
    torch.cuda.current_stream().synchronize()
    with pytest.raises(abi.DynradError) as err:
        abi.dynrad_host_path(host["q"], host["k"], host["v"], runs, chunk_bh=chunk, workspace=ws)
    assert err.value.status == abi.DYNRAD_ERR_INVALID_ARG
    passed = torch.cuda.Event()
    passed.record()
    passed.synchronize()
    got_o = runs[0]["o_host"].view(B * H, N, D)[:chunk]
    got_lse = runs[0]["lse_host"].view(B * H, N)[:chunk]
    assert torch.equal(got_o.view(torch.int16), ref[0][0].view(B * H, N, D)[:chunk].view(torch.int16))
    assert torch.equal(got_lse, ref[0][1].view(B * H, N)[:chunk])
    check_device_status()
