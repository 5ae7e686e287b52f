"""Results table of the five workloads: parity against the oracle and kernel time.

Run on a GPU machine: ``python -m tests.report_workloads [--json out.json]``. For every
workload (the 128k one in both layouts) it runs ``cp_attn_fwd`` on the seeded
inputs, compares the seeded sampled rows (all rows for the two small workloads)
with the fp64 oracle, and times the call with CUDA events (median of 10 after 3
warm-up calls) while nvidia-smi samples the clocks. Test infrastructure: it uses
the oracle; nothing on the product path imports it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import context_long_sequence_cp_b200 as cp  # noqa: E402
from bench import ClockSampler, NOMINAL_BF16_TFLOPS, load_peaks  # noqa: E402
from tests import gpu_util as G  # noqa: E402
from workloads import WORKLOADS, make_qkv, sample_rows  # noqa: E402


def all_rows(B, H, S):
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
    return np.stack([bb.ravel(), hh.ravel(), ii.ravel()], 1).astype(np.int64)


def one(name, w, layout, peak):
    q, k, v = make_qkv(w)
    plan = cp.Plan(w.B, w.H, w.S, w.D, w.N, w.causal, layout)
    qd, kd, vd = (G.to_layout(x, w.N, layout).cuda() for x in (q, k, v))
    o, lse = cp.attn_fwd(plan, qd, kd, vd)
    for _ in range(3):
        cp.attn_fwd(plan, qd, kd, vd, o=o, lse=lse)
    torch.cuda.synchronize()
    ts = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            cp.attn_fwd(plan, qd, kd, vd, o=o, lse=lse)
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
    st = cp.check(plan)
    ms = statistics.median(ts)
    rows = all_rows(w.B, w.H, w.S) if w.S * w.H * w.B <= 65536 else sample_rows(w)
    o_gpu = G.gather_rows(o, w.B, w.S, w.H, w.N, layout, rows)
    lse_gpu = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    t0 = time.perf_counter()
    o_ref, lse_ref = G.oracle_rows(q, k, v, rows, w.causal)
    t_oracle = time.perf_counter() - t0
    err = G.errors(o_gpu, o_ref, lse_gpu, lse_ref)
    tflops = w.flops / (ms * 1e-3) / 1e12
    clocks = clk.summary()
    plan.close()
    return {
        "workload": name, "layout": layout, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "N": w.N,
        "causal": w.causal, "status": st, "rows_checked": int(len(rows)), **err,
        "within_tolerance": bool(err["o_max"] <= G.TOL_O_MAX and err["o_mean"] <= G.TOL_O_MEAN
                                 and err["lse_max"] <= G.TOL_LSE),
        "ms": ms, "tflops": tflops, "frac_measured": tflops / peak, "frac_nominal": tflops / NOMINAL_BF16_TFLOPS,
        "sm_mhz": clocks.get("sm_mhz"), "reasons": clocks.get("reasons"),
        "oracle_s": t_oracle, "oracle_cores": len(os.sched_getaffinity(0)),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--json", default=None)
    args = ap.parse_args()
    peak = float(load_peaks()[0]["bf16_tflops"])
    out = []
    for name, layouts in (("tiny", None), ("zigzag_4k", None), ("zigzag_32k", None),
                          ("long_128k", ("contiguous", "zigzag")), ("ulysses_16k", None)):
        w = WORKLOADS[name]
        for layout in layouts or (w.layout,):
            r = one(name, w, layout, peak)
            out.append(r)
            print(json.dumps(r), flush=True)
    if args.json:
        with open(args.json, "w") as f:
            json.dump(out, f, indent=1)
    return 0 if all(r["within_tolerance"] and r["status"] == 0 for r in out) else 1


if __name__ == "__main__":
    sys.exit(main())
