"""Benchmark of context-parallel attention on B200: one JSON line on rank 0.

A step is one pass of the hot path over one batch of the 32k zigzag workload
(B=1, H=32, S=32768, D=128, 8 virtual ranks, causal), starting from Q/K/V in
natural [B, S, H, D] layout resident in HBM:
  1. layout map: Q, K, V natural -> zigzag rank-major (index-mapped copy kernel);
  2. fused context-parallel attention (ring-order key walk, online-softmax
     merge, causal tile skipping) writing O and lse;
  3. layout map: O rank-major -> natural.
``value`` counts the metric's FLOPs (4*B*H*S^2*D / 2 for causal) per step.
The attention kernel alone is timed on its own stream for the roofline; the
unfused path (per-step partials + merge kernel) is timed as a component.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
Under torchrun every rank runs its own replica of the workload (independent
problems, no data-path collective: weak scaling) and rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal CP-attention fwd TFLOP/s and % of B200 BF16 dense peak, 1 GPU"
WORKLOAD = "zigzag_32k"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def job_throughput(local_ms: float, flops_per_rank: float, world_size: int, device=None) -> tuple:
    """Whole-job throughput of independent per-rank replicas (weak scaling).

    Every rank ran the same work; the job time is the maximum of the ranks'
    device-timed milliseconds (one all-reduce MAX when world_size > 1, on
    whatever process group is initialised). Returns (job_ms, TFLOP/s over all
    ranks).
    """
    job_ms = float(local_ms)
    if world_size > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([job_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        job_ms = float(t.item())
    return job_ms, world_size * flops_per_rank / (job_ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for ln in open(self.path):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [x for x in sm if x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


def oracle_sample_rate(w, max_rows: int, budget_s: float):
    """Time the CPU oracle on sampled rows of the workload: (TFLOP/s, rows, seconds, cores)."""
    import numpy as np
    from oracle import attention as A
    from workloads import make_qkv, sample_rows
    q, k, v = make_qkv(w)
    rows = sample_rows(w)
    rng = np.random.default_rng(0)
    rows = rows[rng.permutation(len(rows))[:max_rows]]
    f = lambda t: t.float().numpy()
    qn, kn, vn = f(q), f(k), f(v)
    cores = len(os.sched_getaffinity(0))
    done, flops, t0 = 0, 0.0, time.perf_counter()
    chunk = 128
    while done < len(rows) and time.perf_counter() - t0 < budget_s:
        sel = rows[done:done + chunk]
        A.attention_rows(qn, kn, vn, sel, causal=w.causal)
        keys = (sel[:, 2] + 1) if w.causal else np.full(len(sel), w.S)
        flops += float((4.0 * w.D * keys).sum())
        done += len(sel)
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, done, dt, cores


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on bounded samples."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from workloads import WORKLOADS
    w = WORKLOADS[WORKLOAD]
    per_step = 5.0
    rates, secs = [], []
    for i in range(args.warmup + args.steps):
        tf, rows, dt, cores = oracle_sample_rate(w, max_rows=4096, budget_s=per_step)
        if i >= args.warmup:
            rates.append(tf)
            secs.append(dt)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.median(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "N": w.N,
                                        "causal": w.causal, "layout": w.layout},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"up to 4096 seeded sampled query rows per step, {per_step:.0f} s budget; "
                                   f"throughput counted as 4*D*(allowed keys) per row"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["attn", "merge", "permute", "bwd", "ring"], default=None,
                    help="only launch one kernel warmup+steps times (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import context_long_sequence_cp_b200 as cp
    from workloads import WORKLOADS, make_qkv

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = WORKLOADS[WORKLOAD]
    B, H, S, D, N = w.B, w.H, w.S, w.D, w.N
    plan = cp.Plan(B, H, S, D, N, w.causal, w.layout)
    q_h, k_h, v_h = make_qkv(w)                       # natural, bf16, host
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    qz, kz, vz, oz = (torch.empty_like(q).view(N, B, S // N, H, D) for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cp.layout_permute(plan, q, 0, out=qz)
        cp.layout_permute(plan, k, 0, out=kz)
        cp.layout_permute(plan, v, 0, out=vz)
        cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
        cp.layout_permute(plan, oz, 1, out=o)

    launches_per_step = 5

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)


    if args.profile:
        for x, y in ((q, qz), (k, kz), (v, vz)):
            cp.layout_permute(plan, x, 0, out=y)
        if args.profile == "merge":
            op = torch.empty(N, plan.rows, D, dtype=torch.float32, device=dev)
            lp = torch.empty(N, plan.rows, dtype=torch.float32, device=dev)
            cp.attn_fwd_partials(plan, qz, kz, vz, o_parts=op, lse_parts=lp)
            om = torch.empty(plan.rows, D, dtype=torch.bfloat16, device=dev)
            lm = torch.empty(plan.rows, dtype=torch.float32, device=dev)
        if args.profile == "bwd":
            from workloads import make_dout
            dod = torch.empty_like(qz)
            cp.layout_permute(plan, make_dout(q_h.shape, w.seed).to(dev), 0, out=dod)
            cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
            gq, gk, gv = (torch.empty_like(qz) for _ in range(3))
            bws = torch.empty(plan.bwd_workspace_bytes(), dtype=torch.uint8, device=dev)
        if args.profile == "ring":
            # rank 0's one-launch ring forward, fetching the other ranks' blocks
            # (layout tensors standing in for their memory) into its own slots
            rslots_k, rslots_v = torch.empty_like(kz), torch.empty_like(vz)
            rslots_k[0].copy_(kz[0])
            rslots_v[0].copy_(vz[0])
            r_arr = torch.zeros(N, dtype=torch.int32, device=dev)
            r_src = ([kz[j].data_ptr() for j in range(N)], [vz[j].data_ptr() for j in range(N)])
        for _ in range(args.warmup + args.steps):
            if args.profile == "ring":
                cp.attn_fwd_ring(plan, 0, qz[0], rslots_k, rslots_v, r_src[0], r_src[1], r_arr)
            elif args.profile == "bwd":
                cp.attn_bwd(plan, qz, kz, vz, oz, lse, dod, gq, gk, gv, bws)
            elif args.profile == "attn":
                cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
            elif args.profile == "merge":
                cp.merge_partials(op, lp, o_out=om, lse_out=lm)
            else:
                cp.layout_permute(plan, q, 0, out=qz)
        st = cp.check(plan)
        print(json.dumps({"profile": args.profile, "launches": args.warmup + args.steps, "status": st}))
        return 0 if st == 0 else 1

    for _ in range(args.warmup):
        step()
    st = cp.check(plan)
    if st != 0:
        raise RuntimeError(f"warm-up failed: {cp.status_string(st)}")

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
    st = cp.check(plan)
    if st != 0:
        raise RuntimeError(f"timed run failed: {cp.status_string(st)}")
    ms, value = job_throughput(ev0.elapsed_time(ev1) / args.steps, w.flops, ws, dev)

    # --- attention kernel alone (dominant kernel), CUDA events on its stream
    att_ms = []
    for _ in range(max(5, args.steps)):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        att_ms.append(a0.elapsed_time(a1))
    att = statistics.median(att_ms)
    att_tflops = w.flops / (att * 1e-3) / 1e12

    # --- permute kernel alone (HBM-bound): 2 bytes read + 2 written per element
    perm_ms = []
    for _ in range(5):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        cp.layout_permute(plan, q, 0, out=qz)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        perm_ms.append(a0.elapsed_time(a1))
    perm = statistics.median(perm_ms)
    perm_gbs = 2 * q.numel() * 2 / (perm * 1e-3) / 1e9

    # --- RoPE fused into the same layout map (HBM-bound, same algorithmic bytes)
    rope_ms = []
    for _ in range(5):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        cp.rope_permute(plan, q, out=qz)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        rope_ms.append(a0.elapsed_time(a1))
    rope = statistics.median(rope_ms)
    rope_gbs = 2 * q.numel() * 2 / (rope * 1e-3) / 1e9

    # --- backward pass (dQ, dK, dV) on the same inputs; dO seeded like the inputs
    from workloads import make_dout
    dod = torch.empty_like(qz)
    cp.layout_permute(plan, make_dout(q_h.shape, w.seed).to(dev), 0, out=dod)
    cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
    gq, gk, gv = (torch.empty_like(qz) for _ in range(3))
    bws = torch.empty(plan.bwd_workspace_bytes(), dtype=torch.uint8, device=dev)
    for _ in range(2):
        cp.attn_bwd(plan, qz, kz, vz, oz, lse, dod, gq, gk, gv, bws)
    bwd_ms = []
    for _ in range(5):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        cp.attn_bwd(plan, qz, kz, vz, oz, lse, dod, gq, gk, gv, bws)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        bwd_ms.append(a0.elapsed_time(a1))
    bwd = statistics.median(bwd_ms)
    st = cp.check(plan)
    if st != 0:
        raise RuntimeError(f"backward failed: {cp.status_string(st)}")
    del gq, gk, gv, dod, bws

    # --- sequence-parallel step after a tensor-parallel region (HBM-bound):
    # z = dropout(sum of 8 partials) + residual, y = LayerNorm(z); 32768 tokens, H 4096
    from workloads import make_keep_bits
    sp_rows, sp_h, sp_n, sp_p = S, 4096, 8, 0.1
    gsp = torch.Generator().manual_seed(5)
    sp_parts = torch.randn(sp_n, sp_rows, sp_h, generator=gsp).to(torch.bfloat16).to(dev)
    sp_res = torch.randn(sp_rows, sp_h, generator=gsp).to(torch.bfloat16).to(dev)
    sp_gamma = torch.ones(sp_h, device=dev)
    sp_beta = torch.zeros(sp_h, device=dev)
    sp_bits = make_keep_bits(sp_rows, sp_h, sp_p, seed=5)[1].to(dev)
    sp_z = torch.empty(sp_rows, sp_h, dtype=torch.bfloat16, device=dev)
    sp_y = torch.empty_like(sp_z)
    sp_ms = []
    for i in range(7):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        cp.sp_rs_dropout_add_ln(sp_parts, sp_bits, sp_p, sp_res, sp_gamma, sp_beta, z=sp_z, y=sp_y)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 2:
            sp_ms.append(a0.elapsed_time(a1))
    sp_t = statistics.median(sp_ms)
    sp_bytes = (sp_n + 1 + 2) * sp_rows * sp_h * 2 + sp_rows * sp_h // 8 + 2 * sp_h * 4
    sp_gbs = sp_bytes / (sp_t * 1e-3) / 1e9
    del sp_parts, sp_res, sp_bits, sp_z, sp_y

    # --- unfused path: per-step partials + merge kernel
    op = torch.empty(N, plan.rows, D, dtype=torch.float32, device=dev)
    lp = torch.empty(N, plan.rows, dtype=torch.float32, device=dev)
    om = torch.empty(plan.rows, D, dtype=torch.bfloat16, device=dev)
    lm = torch.empty(plan.rows, dtype=torch.float32, device=dev)
    cp.attn_fwd_partials(plan, qz, kz, vz, o_parts=op, lse_parts=lp)
    cp.merge_partials(op, lp, o_out=om, lse_out=lm)
    torch.cuda.synchronize(dev)
    m0, m1, m2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    m0.record(stream)
    cp.attn_fwd_partials(plan, qz, kz, vz, o_parts=op, lse_parts=lp)
    m1.record(stream)
    cp.merge_partials(op, lp, o_out=om, lse_out=lm)
    m2.record(stream)
    torch.cuda.synchronize(dev)
    part_ms, merge_ms = m0.elapsed_time(m1), m1.elapsed_time(m2)
    nonempty = int(torch.isfinite(lp).sum().item())
    merge_bytes = nonempty * (4 * D + 4) + (N * plan.rows - nonempty) * 4 + plan.rows * (2 * D + 4)
    merge_gbs = merge_bytes / (merge_ms * 1e-3) / 1e9
    if cp.check(plan) != 0:
        raise RuntimeError("component runs failed")

    # --- one rank of the multi-GPU ring on its own GPU: rank 0 of N, the other
    # ranks' own K/V blocks read from the layout tensors, standing in for their
    # slot buffers (on N GPUs: their memory over NVLink). The ring driver runs as
    # on N GPUs: fill of the own slot, one host barrier, ONE cooperative launch
    # whose copy warps fetch the other blocks in ring order while its units
    # compute step-major, then the merge. Compared with the same launch on
    # resident blocks (no fetch), with one launch per ring step, and with 1/N of
    # the fused launch (the rank's share of the one-GPU forward). L2 is flushed
    # before every timed call.
    from context_long_sequence_cp_b200 import ring as R

    class _OneRank(R.RingRank):
        def pull_sources(self, c):
            return [kz[j].data_ptr() for j in range(N)], [vz[j].data_ptr() for j in range(N)]

    blk = kz[0].numel() * 2
    q0 = qz[0]
    ro = torch.empty(plan.rows // N, D, dtype=torch.bfloat16, device=dev)
    rl = torch.empty(plan.rows // N, dtype=torch.float32, device=dev)
    l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def time_flushed(fn, reps=5):
        out = []
        for i in range(reps + 1):
            l2_flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            fn()
            a1.record(stream)
            torch.cuda.synchronize(dev)
            if i > 0:
                out.append(a0.elapsed_time(a1))
        return statistics.median(out)

    rr = _OneRank(plan, 0, barrier=lambda: None)
    rr.connect([0] * N)
    for _ in range(2):                    # both slot sets
        r_o, _ = rr.forward(q0, kz[0], vz[0], stream)
        torch.cuda.synchronize(dev)
        ring_err = (r_o.float() - oz[0].float()).abs().max().item()
        if cp.check(plan) != 0 or not ring_err <= 2e-2:
            raise RuntimeError(f"ring rank 0 disagrees with the fused forward: {ring_err}")
    ring_ms = time_flushed(lambda: rr.forward(q0, kz[0], vz[0], stream))
    op_r, lp_r = rr.o_parts, rr.lse_parts

    def launch_only():
        cp.attn_fwd_ring(plan, 0, q0, kz, vz, o_parts=op_r, lse_parts=lp_r, stream=stream)
        cp.merge_partials(op_r, lp_r, o_out=ro, lse_out=rl)

    op_s = torch.empty(N, plan.rows // N, D, dtype=torch.float32, device=dev)
    lp_s = torch.empty(N, plan.rows // N, dtype=torch.float32, device=dev)

    def step_launches():
        for t in range(N):
            cp.attn_fwd_ring_step(plan, 0, t, q0, kz[t], vz[t], op_s[t], lp_s[t], stream)
        cp.merge_partials(op_s, lp_s, o_out=ro, lse_out=rl)

    ring_launch_ms = time_flushed(launch_only)
    ring_steps_ms = time_flushed(step_launches)
    if cp.check(plan) != 0:
        raise RuntimeError("ring runs failed")
    rr.close()
    del l2_flush, op_s, lp_s

    # --- end to end through the public API from pinned host buffers. Every step
    # uploads its own Q/K/V from pinned memory and reads back its own O and lse;
    # as a user of the API would, the steps are pipelined: uploads run on one copy
    # stream, read-backs on another (PCIe is full duplex), the step on the compute
    # stream, with device inputs and outputs double-buffered and events ordering
    # every reuse. The timed region spans the first upload to the last read-back.
    q_p, k_p, v_p = (x.pin_memory() for x in (q_h, k_h, v_h))
    o_p = torch.empty_like(q_h).pin_memory()
    lse_p = torch.empty(B, H, S, dtype=torch.float32).pin_memory()
    ins = [(q, k, v), tuple(torch.empty_like(x) for x in (q, k, v))]
    outs = [(o, lse), (torch.empty_like(o), torch.empty_like(lse))]
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]

    def run_pipelined(nsteps, ev_begin=None, ev_end=None):
        if ev_begin is not None:
            ev_begin.record(up_s)
        for i in range(nsteps):
            b = i % 2
            (qi, ki, vi), (oi, li) = ins[b], outs[b]
            if i >= 2:
                up_s.wait_event(ev_out[b])          # step i-2 is done with these inputs
            with torch.cuda.stream(up_s):
                qi.copy_(q_p, non_blocking=True)
                ki.copy_(k_p, non_blocking=True)
                vi.copy_(v_p, non_blocking=True)
            ev_in[b].record(up_s)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_read[b])       # step i-2's result has been read back
            cp.layout_permute(plan, qi, 0, out=qz)
            cp.layout_permute(plan, ki, 0, out=kz)
            cp.layout_permute(plan, vi, 0, out=vz)
            cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=li)
            cp.layout_permute(plan, oz, 1, out=oi)
            ev_out[b].record(stream)
            down_s.wait_event(ev_out[b])
            with torch.cuda.stream(down_s):
                o_p.copy_(oi, non_blocking=True)
                lse_p.copy_(li, non_blocking=True)
            ev_read[b].record(down_s)
        if ev_end is not None:
            ev_end.record(down_s)

    run_pipelined(2)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(4, min(args.steps, 10))
    run_pipelined(e_steps, e0, e1)
    torch.cuda.synchronize(dev)
    barrier()
    e_ms, e2e_value = job_throughput(e0.elapsed_time(e1) / e_steps, w.flops, ws, dev)
    st = cp.check(plan)
    if st != 0:
        raise RuntimeError(f"end-to-end run failed: {cp.status_string(st)}")
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    traffic = None
    prof = os.path.join(ROOT, "profiles", "attn_fwd_zigzag_32k_traffic.json")
    if os.path.exists(prof):
        # DRAM bytes of one launch from an ncu capture, valid only for the kernel
        # and schedule source it was taken on (null once either changed: the
        # plan's item order decides how much of K/V the L2 serves).
        import hashlib
        csrc = os.path.join(ROOT, "context_long_sequence_cp_b200", "csrc")
        h = hashlib.sha256()
        for name in ("attn_fwd.cu", "sm100.cuh", "geometry.h", "api.cu"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
        with open(prof) as f:
            rec = json.load(f)
        if rec.get("source_sha256_16") == h.hexdigest()[:16]:
            traffic = rec.get("dram_bytes_per_launch")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "S": S, "D": D, "N": N, "causal": w.causal,
                   "layout": w.layout, "flops_per_step": w.flops,
                   "l2": "inputs larger than L2 (3 x 256 MiB of Q/K/V read per step)",
                   "step": "permute Q,K,V natural->zigzag; fused CP attention; permute O back"},
        "roofline": {"kernel": "attn_fwd_kernel<128,false>", "bound": "tensor", "achieved": att_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                     "frac_of_nominal_2250": att_tflops / NOMINAL_BF16_TFLOPS, "ms": att},
        "components": {
            "attention_ms": att, "attention_tflops": att_tflops,
            "permute_ms": perm, "permute_gbs": perm_gbs, "permute_frac_hbm": perm_gbs / float(peaks["hbm_gbs"]),
            "rope_permute_ms": rope, "rope_permute_gbs": rope_gbs,
            "rope_permute_frac_hbm": rope_gbs / float(peaks["hbm_gbs"]),
            "bwd_ms": bwd, "bwd_tflops_useful": 2.5 * w.flops / (bwd * 1e-3) / 1e12,
            "bwd_tflops_executed": 3.5 * w.flops / (bwd * 1e-3) / 1e12,
            "bwd_flops_note": "useful = 2.5x the forward's FLOPs (5 tile products); executed = 3.5x "
                              "(S and dP recomputed by the dQ kernel, no atomics)",
            "sp_step_ms": sp_t, "sp_step_gbs": sp_gbs, "sp_step_frac_hbm": sp_gbs / float(peaks["hbm_gbs"]),
            "sp_step_shape": "8 partials x 32768 tokens x H 4096 bf16, dropout 0.1, residual, LayerNorm",
            "partials_ms": part_ms, "merge_ms": merge_ms, "merge_gbs": merge_gbs,
            "merge_frac_hbm": merge_gbs / float(peaks["hbm_gbs"]),
            "unfused_tflops": w.flops / ((part_ms + merge_ms) * 1e-3) / 1e12,
            "ring_rank_ms": ring_ms, "ring_rank_tflops": w.flops / N / (ring_ms * 1e-3) / 1e12,
            "ring_rank_launch_only_ms": ring_launch_ms, "ring_rank_step_launches_ms": ring_steps_ms,
            "ring_rank_fused_share_ms": att / N,
            "ring_overhead_vs_fused_share": ring_ms / (att / N) - 1.0,
            "ring_fetch_cost": ring_ms / ring_launch_ms - 1.0,
            "ring_fetch_bytes": (N - 1) * 2 * blk,
            "ring_parts": plan.ring_parts(),
            "ring_note": f"rank 0 of {N} on one GPU: fill + one cooperative launch whose copy warps fetch the "
                         f"other {N - 1} K/V blocks ({(N - 1) * 2 * blk >> 20} MiB; here from local HBM, on N "
                         "GPUs over NVLink) while its units compute (first half of the steps one unit per step, "
                         "then one unit per query pair), + merge of the parts; launch_only = blocks resident; "
                         "step_launches = one launch per ring step; fused_share = the fused launch / N",
        },
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms, "pipelined": "uploads, step and read-backs of consecutive steps overlap "
                                                  "on two copy streams and the compute stream"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tf, rows, dt, cores = oracle_sample_rate(w, max_rows=4096, budget_s=15.0)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"{rows} seeded sampled query rows of {WORKLOAD} in {dt:.1f} s "
                                          f"(fp64 NumPy); FLOPs counted as 4*D*(allowed keys) per row"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    plan.close()
    if ws > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
