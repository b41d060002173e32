"""Information run of the 2-head, 1,024-token workload, whose inputs are
defined in fp32: the oracle on the fp32 values against the oracle on the
bf16-rounded values the GPU path takes (selection and attention each from its
own inputs).  The difference is reported, not a parity bound: it is the cost
of the bf16 inputs, outside the kernels.  The printed figures are the ones the
design notes quote; the assertions only keep them from drifting silently."""
import numpy as np

from block_sparse_attention_candidate_b200.workloads import WORKLOADS, bf16_bits_to_f64, make_qkv_bf16, make_qkv_f32
from oracle import attention as OA
from oracle import geometry as OG
from oracle import selection as OS


def tiny_fp32_vs_bf16():
    wl = WORKLOADS["tiny"]
    g = wl.geom
    f32 = make_qkv_f32(wl)
    b16 = make_qkv_bf16(wl)
    cand = OG.candidate_csr(g)
    out = {}
    for mode, value, _ in wl.runs:
        d_o, d_lse, rows_diff, rows = [], [], 0, 0
        for h in range(wl.heads):
            res = {}
            for name, src in (("f32", {t: f32[t][0, h].astype(np.float64) for t in "qkv"}),
                              ("bf16", {t: bf16_bits_to_f64(b16[t][0, h]) for t in "qkv"})):
                sel, _ = OS.select_head(src["q"], src["k"], g.block, cand, mode, value)
                o, lse = OA.sparse_attention(src["q"], src["k"], src["v"], g.block, sel["row_ptr"], sel["col"])
                res[name] = (sel, o, lse)
            (s1, o1, l1), (s2, o2, l2) = res["f32"], res["bf16"]
            for r in range(g.n_blocks):
                a = s1["col"][s1["row_ptr"][r]:s1["row_ptr"][r + 1]]
                b = s2["col"][s2["row_ptr"][r]:s2["row_ptr"][r + 1]]
                rows += 1
                rows_diff += int(not np.array_equal(a, b))
            d_o.append(np.abs(o1 - o2))
            d_lse.append(np.abs(l1 - l2))
        d_o = np.concatenate([x.ravel() for x in d_o])
        d_lse = np.concatenate(d_lse)
        out[f"{mode}_{value}"] = {"max_abs_dO": float(d_o.max()), "mean_abs_dO": float(d_o.mean()),
                                  "max_abs_dLSE": float(d_lse.max()), "rows_with_other_kept_set": rows_diff,
                                  "rows": rows}
    return out


def test_tiny_fp32_information_run():
    info = tiny_fp32_vs_bf16()
    for run, d in info.items():
        print(f"tiny {run}: fp32 vs bf16 inputs: max|dO| {d['max_abs_dO']:.3e}, mean|dO| {d['mean_abs_dO']:.3e}, "
              f"max|dLSE| {d['max_abs_dLSE']:.3e}, rows with another kept set {d['rows_with_other_kept_set']}"
              f"/{d['rows']}")
        # bf16 rounding of unit-scale inputs: relative 2^-9 per element
        assert d["mean_abs_dO"] < 5e-3 and d["max_abs_dLSE"] < 5e-2
