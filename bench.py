"""Benchmark of context-parallel attention on B200: one JSON line on rank 0.

A step is one pass of the hot path over one batch of a workload (default: the
32k zigzag workload, B=1, H=32, S=32768, D=128, 8 virtual ranks, causal),
starting from its inputs resident in HBM:
  contiguous / zigzag: Q, K, V in natural [B, S, H, D] layout;
    1. layout map: Q, K, V natural -> rank-major (index-mapped copy kernel);
    2. fused context-parallel attention (ring-order key walk, online-softmax
       merge, causal tile skipping) writing O and lse;
    3. layout map: O rank-major -> natural.
  Ulysses: Q, K, V as N sequence shards [N, B, S/N, H, D]; one ``cp_attn_fwd``
    (shards -> head groups, attention per group, groups -> shards).
``value`` counts the metric's FLOPs (4*B*H*S^2*D, halved for causal) per step.

Every component leg (the attention kernel alone, the layout maps, RoPE, the
merge, the backward, the sequence-parallel step) is timed as K back-to-back
launches between one pair of CUDA events on the launching stream, with inputs
larger than L2, and divided by K; a background NVML thread samples the SM clock
during each leg, so that every figure carries the clock it ran at. Legs whose
inputs fit in L2 (small workloads, one ring rank) flush L2 before every launch
instead and time each launch between its own events, the flush enqueued ahead
so that no host latency falls inside a pair.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                       [--workload NAME] [--mode ring|replica]
Under torchrun (N > 1) the default mode is the context-parallel ring itself:
rank r holds chunk r of the workload's sequence (its zigzag or contiguous
share), the N ranks run the ring forward over CUDA IPC (``ring.IpcRing``: each
rank fetches the other ranks' K/V blocks over NVLink inside its one-launch
forward), and the line reports the whole problem's FLOPs over the slowest
rank's time (strong scaling: the total work is fixed). ``--mode replica``
instead runs an independent replica of the one-GPU problem per rank (weak
scaling). Rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal CP-attention fwd TFLOP/s and % of B200 BF16 dense peak, 1 GPU"
DEFAULT_WORKLOAD = "zigzag_32k"
NOMINAL_BF16_TFLOPS = 2250.0
# Dense bf16 tensor-core work per SM per clock (tcgen05, kind::f16) and the SM count:
# the tensor pipe's own rate at a sampled clock is SMS * this * MHz.
TENSOR_FLOP_PER_CLK_SM = 8192
B200_SMS = 148
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


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


def config_of(w, layout=None) -> dict:
    """The ``config`` object of a workload's JSON line (the same for both arms)."""
    layout = layout or w.layout
    if layout == "ulysses":
        step = "cp_attn_fwd on sequence shards: shards -> head groups, attention per group, groups -> shards"
        l2 = "inputs larger than L2" if 3 * w.B * w.S * w.H * w.D * 2 > L2_BYTES else "L2 flushed between steps"
    else:
        step = "permute Q,K,V natural->rank-major; fused CP attention; permute O back"
        per = w.B * w.S * w.H * w.D * 2
        l2 = (f"inputs larger than L2 (3 x {per >> 20} MiB of Q/K/V read per step)" if per > L2_BYTES
              else "L2 flushed between steps")
    return {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "N": w.N, "causal": w.causal,
            "layout": layout, "flops_per_step": w.flops, "l2": l2, "step": step}


# ----------------------------------------------------------------------------- clocks

_REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                ("sw_power_cap", 0x4))


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every ``period`` seconds on
    a background thread (NVML; ``nvidia-smi`` if NVML is unavailable) while the
    benchmark runs. ``window(t0, t1)`` summarises the samples of one leg."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period: float = 0.01):
        self.gpu, self.period = gpu_index, period
        self.samples = []          # (wall time, sm MHz, max MHz, power W, {reason names})
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self._path = None
        self.source = None

    def _handle(self, nv):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:  # noqa: BLE001 - fall back to the CUDA index
            return nv.nvmlDeviceGetHandleByIndex(self.gpu)

    def _nvml_loop(self, nv, h):
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                names = {n for n, b in _REASON_BITS if bits & b}
                self.samples.append((time.time(), sm, mx, pw, names))
            except Exception:  # noqa: BLE001 - a failed sample is skipped
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._thread.start()
            self.source = "nvml"
        except Exception:  # noqa: BLE001
            fd, self._path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi"
            except OSError:
                self._proc = None
        time.sleep(0.05)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            t_end = time.time()
            rows = []
            for ln in open(self._path):
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
            os.unlink(self._path)
            # nvidia-smi rows carry no time stamp: spread them over the run
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            for i, r in enumerate(rows):
                pw = float(r[3]) if r[3].replace(".", "").isdigit() else 0.0
                rs = {n for j, n in enumerate(names) if r[5 + j].lower() == "active"}
                self.samples.append((t_end - 0.1 * (len(rows) - i), float(r[1]), float(r[2]), pw, rs))

    def window(self, t0=None, t1=None) -> dict:
        s = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        mx = max(x[2] for x in s)
        sm = [x[1] for x in s]
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        reasons = sorted(set().union(*[x[4] for x in s]))
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons, "samples": len(s),
                "power_w_max": max(x[3] for x in s), "source": self.source}


# ----------------------------------------------------------------------------- timing legs

class Legs:
    """Timing of component legs on one stream, each with the clock it ran at."""

    def __init__(self, torch, dev, stream, clk):
        self.torch, self.dev, self.stream, self.clk = torch, dev, stream, clk
        self._flush = None

    def back_to_back(self, fn, reps: int, warm: int = 2):
        """``reps`` launches of ``fn`` between one event pair (inputs larger than
        L2; no synchronise inside the pair): (ms per call, clock summary)."""
        torch = self.torch
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(self.dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        a0.record(self.stream)
        for _ in range(reps):
            fn()
        a1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        t1 = time.time()
        return a0.elapsed_time(a1) / reps, self.clk.window(t0, t1)

    def flushed(self, fn, reps: int, warm: int = 2):
        """Each launch after an L2 flush, between its own events; the flush is
        enqueued ahead of the first event, so the host's launch latency is hidden
        behind it. (median ms per call, clock summary)."""
        torch = self.torch
        if self._flush is None:
            self._flush = torch.empty(256 << 20, dtype=torch.uint8, device=self.dev)
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(self.dev)
        evs = []
        t0 = time.time()
        for _ in range(reps):
            self._flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(self.stream)
            fn()
            a1.record(self.stream)
            evs.append((a0, a1))
        torch.cuda.synchronize(self.dev)
        t1 = time.time()
        return statistics.median(a.elapsed_time(b) for a, b in evs), self.clk.window(t0, t1)


def tensor_pipe_tflops(mhz):
    return None if not mhz else B200_SMS * TENSOR_FLOP_PER_CLK_SM * mhz * 1e6 / 1e12


# ----------------------------------------------------------------------------- CPU oracle

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
    w = WORKLOADS[args.workload]
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
        "data": "synthetic", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"up to 4096 seeded sampled query rows per step, {per_step:.0f} s budget; "
                                   f"throughput counted as 4*D*(allowed keys) per row"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA arm

def traffic_record(name: str, files):
    """DRAM bytes of one launch from an ncu capture under profiles/, valid only
    for the source it was taken on (null once a listed file changed)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(prof):
        return None
    csrc = os.path.join(ROOT, "context_long_sequence_cp_b200", "csrc")
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    with open(prof) as f:
        rec = json.load(f)
    return rec.get("dram_bytes_per_launch") if rec.get("source_sha256_16") == h.hexdigest()[:16] else None


def profile_mode(args, cp, torch, plan, w, dev, q, k, v, qz, kz, vz, oz, lse, q_h):
    """Launch one kernel warmup+steps times (for ncu captures); prints a status line."""
    N, D, S = w.N, w.D, w.S
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
        rslots_k, rslots_v = torch.empty_like(kz), torch.empty_like(vz)
        rslots_k[0].copy_(kz[0])
        rslots_v[0].copy_(vz[0])
        r_arr = torch.zeros(N, dtype=torch.int32, device=dev)
        r_src = ([kz[j].data_ptr() for j in range(N)], [vz[j].data_ptr() for j in range(N)])
    if args.profile == "sp":
        sp = sp_inputs(torch, dev, S)
    for _ in range(args.warmup + args.steps):
        if args.profile == "ring":
            cp.attn_fwd_ring(plan, 0, qz[0], rslots_k, rslots_v, r_src[0], r_src[1], r_arr)
        elif args.profile == "bwd":
            cp.attn_bwd(plan, qz, kz, vz, oz, lse, dod, gq, gk, gv, bws)
        elif args.profile == "attn":
            cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
        elif args.profile == "merge":
            cp.merge_partials(op, lp, o_out=om, lse_out=lm)
        elif args.profile == "rope":
            cp.rope_permute(plan, q, out=qz)
        elif args.profile == "sp":
            sp_call(cp, sp)
        else:
            cp.layout_permute(plan, q, 0, out=qz)
    st = cp.check(plan)
    print(json.dumps({"profile": args.profile, "launches": args.warmup + args.steps, "status": st}))
    return 0 if st == 0 else 1


def sp_inputs(torch, dev, rows):
    """The sequence-parallel step's inputs: 8 bf16 partials of rows x 4096, dropout 0.1."""
    from workloads import make_keep_bits
    sp_h, sp_n, sp_p = 4096, 8, 0.1
    gsp = torch.Generator().manual_seed(5)
    d = {"parts": torch.randn(sp_n, rows, sp_h, generator=gsp).to(torch.bfloat16).to(dev),
         "res": torch.randn(rows, sp_h, generator=gsp).to(torch.bfloat16).to(dev),
         "gamma": torch.ones(sp_h, device=dev), "beta": torch.zeros(sp_h, device=dev),
         "bits": make_keep_bits(rows, sp_h, sp_p, seed=5)[1].to(dev), "p": sp_p, "n": sp_n, "h": sp_h,
         "rows": rows}
    d["z"] = torch.empty(rows, sp_h, dtype=torch.bfloat16, device=dev)
    d["y"] = torch.empty_like(d["z"])
    return d


def sp_call(cp, d):
    cp.sp_rs_dropout_add_ln(d["parts"], d["bits"], d["p"], d["res"], d["gamma"], d["beta"], z=d["z"], y=d["y"])


def components_32k(cp, torch, plan, w, dev, stream, legs, peaks, q, q_h, qz, kz, vz, oz, lse, reps):
    """Component legs on the 32k zigzag workload: layout map, RoPE, backward,
    sequence-parallel step, unfused partials + merge, one ring rank."""
    N, D, S = w.N, w.D, w.S
    hbm = float(peaks["hbm_gbs"])
    comp = {}
    elem_bytes = 2 * q.numel() * 2   # 2 bytes read + 2 written per element

    perm, c = legs.back_to_back(lambda: cp.layout_permute(plan, q, 0, out=qz), 4 * reps)
    comp.update(permute_ms=perm, permute_gbs=elem_bytes / (perm * 1e-3) / 1e9, permute_clock=c)
    comp["permute_frac_hbm"] = comp["permute_gbs"] / hbm
    rope, c = legs.back_to_back(lambda: cp.rope_permute(plan, q, out=qz), 4 * reps)
    comp.update(rope_permute_ms=rope, rope_permute_gbs=elem_bytes / (rope * 1e-3) / 1e9, rope_permute_clock=c)
    comp["rope_permute_frac_hbm"] = comp["rope_permute_gbs"] / hbm
    cp.layout_permute(plan, q, 0, out=qz)

    # backward (dQ, dK, dV) on the same inputs; dO seeded like the inputs
    from workloads import make_dout
    dod = torch.empty_like(qz)
    cp.layout_permute(plan, make_dout(q_h.shape, w.seed).to(dev), 0, out=dod)
    cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse)
    gq, gk, gv = (torch.empty_like(qz) for _ in range(3))
    bws = torch.empty(plan.bwd_workspace_bytes(), dtype=torch.uint8, device=dev)
    bwd, c = legs.back_to_back(lambda: cp.attn_bwd(plan, qz, kz, vz, oz, lse, dod, gq, gk, gv, bws),
                               max(3, reps // 4))
    if cp.check(plan) != 0:
        raise RuntimeError("backward failed")
    comp.update(bwd_ms=bwd, bwd_tflops_useful=2.5 * w.flops / (bwd * 1e-3) / 1e12,
                bwd_tflops_executed=3.5 * w.flops / (bwd * 1e-3) / 1e12, bwd_clock=c,
                bwd_flops_note="useful = 2.5x the forward's FLOPs (5 tile products); executed = 3.5x "
                               "(S and dP recomputed by the dQ kernel, no atomics)")
    comp["bwd_frac_useful"] = comp["bwd_tflops_useful"] / float(peaks["bf16_tflops"])
    del gq, gk, gv, dod, bws

    # sequence-parallel step after a tensor-parallel region (HBM-bound)
    sp = sp_inputs(torch, dev, S)
    sp_t, c = legs.back_to_back(lambda: sp_call(cp, sp), 2 * reps)
    sp_bytes = (sp["n"] + 1 + 2) * sp["rows"] * sp["h"] * 2 + sp["rows"] * sp["h"] // 8 + 2 * sp["h"] * 4
    comp.update(sp_step_ms=sp_t, sp_step_gbs=sp_bytes / (sp_t * 1e-3) / 1e9, sp_step_clock=c,
                sp_step_shape="8 partials x 32768 tokens x H 4096 bf16, dropout 0.1, residual, LayerNorm")
    comp["sp_step_frac_hbm"] = comp["sp_step_gbs"] / hbm
    del sp

    # unfused path: per-step partials + merge kernel
    op = torch.empty(N, plan.rows, D, dtype=torch.float32, device=dev)
    lp = torch.empty(N, plan.rows, dtype=torch.float32, device=dev)
    om = torch.empty(plan.rows, D, dtype=torch.bfloat16, device=dev)
    lm = torch.empty(plan.rows, dtype=torch.float32, device=dev)
    part_ms, c = legs.back_to_back(lambda: cp.attn_fwd_partials(plan, qz, kz, vz, o_parts=op, lse_parts=lp),
                                   max(3, reps // 2))
    merge_ms, mc = legs.back_to_back(lambda: cp.merge_partials(op, lp, o_out=om, lse_out=lm), 2 * reps)
    nonempty = int(torch.isfinite(lp).sum().item())
    merge_bytes = nonempty * (4 * D + 4) + (N * plan.rows - nonempty) * 4 + plan.rows * (2 * D + 4)
    comp.update(partials_ms=part_ms, merge_ms=merge_ms, merge_gbs=merge_bytes / (merge_ms * 1e-3) / 1e9,
                merge_clock=mc, unfused_tflops=w.flops / ((part_ms + merge_ms) * 1e-3) / 1e12)
    comp["merge_frac_hbm"] = comp["merge_gbs"] / hbm
    del op, lp, om, lm
    if cp.check(plan) != 0:
        raise RuntimeError("component runs failed")
    return comp


def ring_components(cp, torch, plan, w, dev, stream, legs, qz, kz, vz, oz, att_ms):
    """One rank of the multi-GPU ring on its own GPU: rank 0 of N, the other ranks'
    own K/V blocks read from the layout tensors, standing in for their slot
    buffers (on N GPUs: their memory over NVLink). The ring driver runs as on N
    GPUs: fill of the own slot, one host barrier, ONE cooperative launch whose
    copy warps fetch the other blocks in ring order while its units compute, then
    the merge. Compared with the same launch on resident blocks (no fetch), with
    one launch per ring step, and with 1/N of the fused launch. L2 is flushed
    before every timed call (one rank's blocks fit in L2)."""
    from context_long_sequence_cp_b200 import ring as R
    N, D = w.N, w.D

    class _OneRank(R.RingRank):
        def pull_sources(self, c):
            return [kz[j].data_ptr() for j in range(N)], [vz[j].data_ptr() for j in range(N)]

    blk = kz[0].numel() * 2
    q0 = qz[0]
    ro = torch.empty(plan.rows // N, D, dtype=torch.bfloat16, device=dev)
    rl = torch.empty(plan.rows // N, dtype=torch.float32, device=dev)
    rr = _OneRank(plan, 0, barrier=lambda: None)
    rr.connect([0] * N)
    for _ in range(2):                    # both slot sets
        r_o, _ = rr.forward(q0, kz[0], vz[0], stream)
        torch.cuda.synchronize(dev)
        ring_err = (r_o.float() - oz[0].float()).abs().max().item()
        if cp.check(plan) != 0 or not ring_err <= 2e-2:
            raise RuntimeError(f"ring rank 0 disagrees with the fused forward: {ring_err}")
    ring_ms, c = legs.flushed(lambda: rr.forward(q0, kz[0], vz[0], stream), 15)
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

    ring_launch_ms, _ = legs.flushed(launch_only, 15)
    ring_steps_ms, _ = legs.flushed(step_launches, 15)
    # The fused launch under the ring calls' own protocol (each call after an L2
    # flush, short enough to run at burst clocks), so that the share compares like
    # with like; the back-to-back figure of the attention leg runs under the power
    # cap and would flatter the ring.
    lse_f = torch.empty(w.B, w.H, w.S, dtype=torch.float32, device=dev)
    fused_ms, fused_clock = legs.flushed(lambda: cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=lse_f), 7)
    if cp.check(plan) != 0:
        raise RuntimeError("ring runs failed")
    rr.close()
    return {
        "ring_rank_ms": ring_ms, "ring_rank_tflops": w.flops / N / (ring_ms * 1e-3) / 1e12,
        "ring_rank_launch_only_ms": ring_launch_ms, "ring_rank_step_launches_ms": ring_steps_ms,
        "ring_rank_fused_share_ms": fused_ms / N, "ring_overhead_vs_fused_share": ring_ms / (fused_ms / N) - 1.0,
        "ring_fused_clock": fused_clock, "ring_fused_share_back_to_back_ms": att_ms / N,
        "ring_fetch_cost": ring_ms / ring_launch_ms - 1.0, "ring_fetch_bytes": (N - 1) * 2 * blk,
        "ring_parts": plan.ring_parts(), "ring_clock": c,
        "ring_note": f"rank 0 of {N} on one GPU: fill + one cooperative launch whose copy warps fetch the "
                     f"other {N - 1} K/V blocks ({(N - 1) * 2 * blk >> 20} MiB; here from local HBM, on N "
                     "GPUs over NVLink) while its units compute, + merge of the parts; launch_only = blocks "
                     "resident; step_launches = one launch per ring step; fused_share = the fused launch / N "
                     "timed the same way; L2 flushed before each call",
    }


# ----------------------------------------------------------------------------- ring mode (N > 1)

def timed_ring_steps(step, barrier, events, steps: int, warmup: int) -> float:
    """``warmup`` untimed steps, then ``steps`` steps between one pair of events,
    bracketed by ``barrier()`` (host barrier of all ranks + device synchronise)
    on both sides; returns this rank's milliseconds per step. ``events()``
    returns a (start, end) pair with ``record()`` and ``elapsed_time(end)``."""
    for _ in range(warmup):
        step()
    barrier()
    e0, e1 = events()
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    barrier()
    return e0.elapsed_time(e1) / steps


def ring_line(w, n, steps, warmup, job_ms, ring_ms_rank0, fused_ms, e2e_ms, h2d, d2h, clocks, peak, peak_src):
    """The JSON line of the ring mode: the whole problem's FLOPs over the slowest
    rank's step time (strong scaling)."""
    value = w.flops / (job_ms * 1e-3) / 1e12
    cfg = config_of(w)
    cfg.update(N=n, ranks="one process per GPU, CUDA IPC slot buffers, gloo host barrier",
               step="ring forward of every rank: fill own slot, one host barrier, one cooperative launch "
                    "fetching the other ranks' K/V blocks over NVLink while computing, merge of the parts")
    achieved = w.flops / n / (ring_ms_rank0 * 1e-3) / 1e12
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": n, "steps": steps, "warmup": warmup,
        "ms_per_step": job_ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": cfg,
        "roofline": {"kernel": "attn_fwd_kernel<128,true> ring launch + merge, rank 0", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": f"{peak_src} bf16_tflops (burst)", "ms": ring_ms_rank0},
        "components": {"fused_one_gpu_ms": fused_ms,
                       "ring_overhead_vs_fused_share": None if not fused_ms else job_ms / (fused_ms / n) - 1.0,
                       "note": "fused_one_gpu_ms: the one-GPU fused forward of the whole problem on rank 0's GPU; "
                               "the overhead compares the ring step with 1/N of it"},
        "e2e": {"value": w.flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "note": "every rank uploads its own Q/K/V chunk from pinned memory and reads back its O and lse "
                        "each step; bytes summed over the ranks"},
        "gpu_launches": 2 * n * steps,
        "clocks": clocks,
    }


def ring_main(args, ws, rank, local):
    """bench.py --gpus N under torchrun: the ring over N GPUs (see the module doc)."""
    import datetime

    import torch
    import torch.distributed as dist

    import context_long_sequence_cp_b200 as cp
    from context_long_sequence_cp_b200 import ring as R
    from workloads import WORKLOADS, make_qkv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = WORKLOADS[args.workload]
    if args.layout:
        w = w.with_layout(args.layout)
    if w.layout == "ulysses":
        raise SystemExit("the ring mode runs the contiguous and zigzag layouts")
    B, H, S, D, N = w.B, w.H, w.S, w.D, ws
    plan = cp.Plan(B, H, S, D, N, w.causal, w.layout)
    nat = make_qkv(w)
    # this rank's chunk in the layout's local order, through the library's layout map
    chunks = []
    for x in nat:
        y = cp.layout_permute(plan, x.to(dev), 0).view(N, B, S // N, H, D)
        chunks.append(y[rank].contiguous())
        del y
    q, k, v = chunks
    ring = R.IpcRing(plan)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()

    def barrier():
        dist.barrier(group=ring.group)
        torch.cuda.synchronize(dev)

    def events():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        class _E:
            def __init__(self, e):
                self.e = e

            def record(self):
                self.e.record(stream)

            def elapsed_time(self, other):
                return self.e.elapsed_time(other.e)
        return _E(a), _E(b)

    with ClockSampler(local) as clk:
        t0 = time.time()
        local_ms = timed_ring_steps(lambda: ring.forward(q, k, v, stream), barrier, events, args.steps, args.warmup)
        clocks = clk.window(t0, time.time())
        st = cp.check(plan)
        if st != 0:
            raise RuntimeError(f"ring forward failed on rank {rank}: {cp.status_string(st)}")
        job_ms, _ = job_throughput(local_ms, w.flops / N, ws, dev)
        # end to end: each rank's chunk from pinned host memory, result read back
        q_p, k_p, v_p = (x.cpu().pin_memory() for x in (q, k, v))
        o_p = torch.empty_like(q_p).pin_memory()
        l_p = torch.empty(B * (S // N) * H, dtype=torch.float32).pin_memory()
        qi, ki, vi = (torch.empty_like(x) for x in (q, k, v))

        def e2e_step():
            qi.copy_(q_p, non_blocking=True)
            ki.copy_(k_p, non_blocking=True)
            vi.copy_(v_p, non_blocking=True)
            o, lse = ring.forward(qi, ki, vi, stream)
            o_p.copy_(o.view(o_p.shape), non_blocking=True)
            l_p.copy_(lse, non_blocking=True)

        e_local = timed_ring_steps(e2e_step, barrier, events, max(3, min(args.steps, 10)), 2)
        e_ms, _ = job_throughput(e_local, w.flops / N, ws, dev)
        # the one-GPU fused forward of the whole problem, on rank 0's GPU only
        fused_ms = None
        if rank == 0:
            p1 = cp.Plan(B, H, S, D, w.N, w.causal, w.layout)
            full = [cp.layout_permute(p1, x.to(dev), 0) for x in nat]
            o1 = torch.empty_like(full[0])
            l1 = torch.empty(B, H, S, dtype=torch.float32, device=dev)
            legs = Legs(torch, dev, stream, clk)
            fused_ms, _ = legs.back_to_back(lambda: cp.attn_fwd(p1, *full, o=o1, lse=l1), 10)
            del full, o1, l1
            p1.close()
        barrier()
    if rank == 0:
        per_rank = q.numel() * 2
        line = ring_line(w, N, args.steps, args.warmup, job_ms, local_ms, fused_ms, e_ms, 3 * per_rank * N,
                         (per_rank + B * (S // N) * H * 4) * N, clocks, float(peaks["bf16_tflops"]), peak_src)
        print(json.dumps(line), flush=True)
    ring.close()
    plan.close()
    dist.destroy_process_group()
    return 0


def main():
    from workloads import WORKLOADS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS),
                    help="workload of the step (default: the 32k zigzag headline)")
    ap.add_argument("--layout", default=None, help="override the workload's layout (long_128k: contiguous|zigzag)")
    ap.add_argument("--mode", choices=["ring", "replica"], default="ring",
                    help="under torchrun: the ring over the N GPUs (default) or N independent replicas")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-components", action="store_true", help="skip the component legs (32k workload)")
    ap.add_argument("--profile", choices=["attn", "merge", "permute", "rope", "sp", "bwd", "ring"], default=None,
                    help="only launch one kernel warmup+steps times (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    ws, rank, local = dist_env()
    if ws > 1 and args.mode == "ring" and not args.profile:
        return ring_main(args, ws, rank, local)

    import torch
    import torch.distributed as dist

    import context_long_sequence_cp_b200 as cp
    from workloads import make_qkv

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = WORKLOADS[args.workload]
    if args.layout:
        w = w.with_layout(args.layout)
    B, H, S, D, N = w.B, w.H, w.S, w.D, w.N
    uly = w.layout == "ulysses"
    plan = cp.Plan(B, H, S, D, N, w.causal, w.layout)
    q_h, k_h, v_h = make_qkv(w)                       # natural, bf16, host
    if uly:   # the inputs are the N sequence shards (the natural tensor split along S)
        q_h, k_h, v_h = (x.reshape(B, N, S // N, H, D).transpose(0, 1).contiguous() for x in (q_h, k_h, v_h))
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    if uly:
        qz, kz, vz = q, k, v
        oz = torch.empty_like(q)
        ws_buf = torch.empty(plan.workspace_bytes(False), dtype=torch.uint8, device=dev)
    else:
        qz, kz, vz, oz = (torch.empty_like(q).view(N, B, S // N, H, D) for _ in range(4))
        ws_buf = None
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    small = 3 * q.numel() * 2 <= 2 * L2_BYTES   # inputs (nearly) fit in L2: flush between launches

    if args.profile:
        return profile_mode(args, cp, torch, plan, w, dev, q, k, v, qz, kz, vz, oz, lse, q_h)

    def attention(qi=None, ki=None, vi=None, oi=None, li=None):
        if uly:
            cp.attn_fwd(plan, qi if qi is not None else q, ki if ki is not None else k,
                        vi if vi is not None else v, o=oi if oi is not None else o,
                        lse=li if li is not None else lse, workspace=ws_buf)
        else:
            cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=li if li is not None else lse)

    att_events = []   # (start, end) around the attention launch of each timed step

    def step(qi=q, ki=k, vi=v, oi=o, li=lse, mark=False):
        if mark:
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if uly:
            if mark:
                a0.record(stream)
            attention(qi, ki, vi, oi, li)
            if mark:
                a1.record(stream)
                att_events.append((a0, a1))
            return
        cp.layout_permute(plan, qi, 0, out=qz)
        cp.layout_permute(plan, ki, 0, out=kz)
        cp.layout_permute(plan, vi, 0, out=vz)
        if mark:
            a0.record(stream)
        cp.attn_fwd(plan, qz, kz, vz, o=oz, lse=li)
        if mark:
            a1.record(stream)
            att_events.append((a0, a1))
        cp.layout_permute(plan, oz, 1, out=oi)

    launches_per_step = 5   # 3 layout maps + attention + inverse map (Ulysses: the same inside cp_attn_fwd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if small else None

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    peaks, peak_src = load_peaks()
    # The attention kernel is timed inside the timed step loop (hundreds of ms at
    # full load, under the power cap): the sustained bf16 figure is its peak.
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    peak_burst = float(peaks["bf16_tflops"])
    with ClockSampler(local) as clk:
        legs = Legs(torch, dev, stream, clk)
        for _ in range(args.warmup):
            step()
        st = cp.check(plan)
        if st != 0:
            raise RuntimeError(f"warm-up failed: {cp.status_string(st)}")

        barrier()
        t0 = time.time()
        if small:
            # per-step events after an L2 flush enqueued ahead (inputs fit in L2)
            evs = []
            for _ in range(args.steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                step(mark=True)
                e1.record(stream)
                evs.append((e0, e1))
            barrier()
            local_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
        else:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(args.steps):
                step(mark=True)
            ev1.record(stream)
            barrier()
            local_ms = ev0.elapsed_time(ev1) / args.steps
        step_clock = clk.window(t0, time.time())
        # the dominant kernel's duration inside the timed steps (events on its stream)
        att_in_step = sum(a.elapsed_time(b) for a, b in att_events) / len(att_events)
        st = cp.check(plan)
        if st != 0:
            raise RuntimeError(f"timed run failed: {cp.status_string(st)}")
        ms, value = job_throughput(local_ms, w.flops, ws, dev)

        # --- the attention kernel alone (dominant kernel)
        if not uly:
            for x, y in ((q, qz), (k, kz), (v, vz)):
                cp.layout_permute(plan, x, 0, out=y)
        reps = max(20, args.steps // 2)
        if uly:
            # the Ulysses call is 3 maps + attention + 1 map, timed whole
            att_fn = attention
            att_kernel = "cp_attn_fwd (Ulysses: 3 maps + attn_fwd_kernel<128,false> + 1 map)"
        else:
            att_fn = attention
            att_kernel = f"attn_fwd_kernel<{D},false>"
        att_alone, att_alone_clock = (legs.flushed(att_fn, reps) if small else legs.back_to_back(att_fn, reps))
        att, att_clock = att_in_step, step_clock
        att_tflops = w.flops / (att * 1e-3) / 1e12
        st = cp.check(plan)
        if st != 0:
            raise RuntimeError(f"attention leg failed: {cp.status_string(st)}")

        comp = {"attention_in_step_ms": att, "attention_in_step_tflops": att_tflops,
                "attention_alone_ms": att_alone, "attention_alone_tflops": w.flops / (att_alone * 1e-3) / 1e12,
                "attention_alone_clock": att_alone_clock,
                "attention_alone_note": f"{reps} launches of the attention call alone after the timed steps "
                                        "(back to back, or each after an L2 flush for inputs that fit in L2)"}
        if w.name == DEFAULT_WORKLOAD and not args.no_components:
            comp.update(components_32k(cp, torch, plan, w, dev, stream, legs, peaks, q, q_h, qz, kz, vz, oz, lse,
                                       reps))
            for x, y in ((q, qz), (k, kz), (v, vz)):
                cp.layout_permute(plan, x, 0, out=y)
            attention()
            comp.update(ring_components(cp, torch, plan, w, dev, stream, legs, qz, kz, vz, oz, att_alone))

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
                step(qi, ki, vi, oi, li)
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

    traffic = None
    if w.name == DEFAULT_WORKLOAD:
        traffic = traffic_record("attn_fwd_zigzag_32k_traffic.json", ("attn_fwd.cu", "sm100.cuh", "geometry.h",
                                                                       "api.cu"))
    att_mhz = att_clock.get("sm_mhz")
    pipe = tensor_pipe_tflops(att_mhz)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w),
        "roofline": {"kernel": att_kernel, "bound": "tensor", "achieved": att_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops_sustained (the kernel is timed inside the timed "
                                    "step loop, at the loop's power-capped clocks)",
                     "frac_of_burst_peak": att_tflops / peak_burst, "burst_peak": peak_burst,
                     "frac_of_nominal_2250": att_tflops / NOMINAL_BF16_TFLOPS, "ms": att,
                     "timing": f"mean of one event pair around the attention launch in each of the {args.steps} "
                               "timed steps (its stream), i.e. at the step's own clocks",
                     "sm_mhz": att_mhz, "clock_reasons": att_clock.get("reasons"),
                     "mcycles_per_launch": None if not att_mhz else att * 1e-3 * att_mhz,
                     "frac_of_tensor_pipe_at_clock": None if not pipe else att_tflops / pipe,
                     "tensor_pipe_note": f"{B200_SMS} SMs x {TENSOR_FLOP_PER_CLK_SM} dense bf16 FLOP/clk x the "
                                         "leg's median SM clock"},
        "components": comp,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms, "pipelined": "uploads, step and read-backs of consecutive steps overlap "
                                                  "on two copy streams and the compute stream"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": step_clock,
    }

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tf, rows, dt, cores = oracle_sample_rate(w, max_rows=4096, budget_s=15.0)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"{rows} seeded sampled query rows of {w.name} in {dt:.1f} s "
                                          f"(fp64 NumPy); FLOPs counted as 4*D*(allowed keys) per row"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    plan.close()
    if ws > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
