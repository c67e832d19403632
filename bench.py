#!/usr/bin/env python
"""Benchmark of exact block-sparse attention, forward + backward, on B200.

Metric: useful-pair TFLOP/s.  A useful pair is an allowed (query, key) pair
of the sparse graph; the forward is credited 4*D flops per useful pair and
forward+backward 10*D (the headline ``value``).  The FlashAttention-style
14*D count is reported beside it, labelled.

One step = spattn_fwd + spattn_bwd over one batch of seeded synthetic inputs
that are already resident in HBM.  Default workload: partial-block 3D STA,
21x45x80 latent grid in 4x4x4 tiles, clamped 3x5x5 tile window, 40 heads,
D=128 (each input tensor is 0.94 GB, far above the 126 MB L2, so no flush is
needed between steps; smaller workloads flush L2 between steps and time each
step with its own events).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (torchrun), every rank runs an independent replica of the
workload (heads and batch entries are independent; there is no data-path
collective) and ``value`` counts the useful pairs of all ranks over the
slowest rank's time.
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
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import configs as W  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_TEXT = {
    "partial": "partial-block 3D STA: 21x45x80 grid, 4x4x4 tiles (1440 blocks, 92160 slots, 75600 valid), clamped 3x5x5 tile window",
    "full": "full-occupancy STA: 16x32x32 grid, 4x4x4 tiles (256 blocks, all valid), clamped 3x3x3 tile window",
    "vsa": "VSA-style dynamic blocks: 21x45x80 grid, 4x4x4 tiles, own tile + 31 random tiles per query tile and head",
    "svg2": "independent Q/K partitions: 75600 tokens, 100 Q / 500 K clusters, 64 K clusters per Q cluster and head",
    "tiny": "tiny STA: 5x6x10 grid, 4x4x4 tiles, clamped 3x3x3 window",
}
KERNEL_FLOPS_PER_PAIR_D = {"fwd": 4, "dkdv": 8, "dq": 6}  # algorithmic GEMM flops per useful pair / D
KERNEL_SOURCES = ["sm100.cuh", "tile.cuh", "fwd.cu", "bwd.cu", "plan.cpp"]  # kernels and the lists they walk


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_attention_bwd_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
        r = rec.get(f"{kernel}/{workload}")
        if r and r.get("kernel_source_sha") == kernel_source_hash():
            return float(r["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_id):
        self.device_id = device_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.device_id], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        with open(self.path) as fh:
            out = self.parse(fh)
        os.unlink(self.path)
        return out

    @classmethod
    def parse(cls, lines):
        """Median SM clock, max clock and the throttle reasons seen active in
        `nvidia-smi --query-gpu=FIELDS --format=csv,noheader,nounits` lines."""
        sm, mx, reasons, n = [], None, set(), 0
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            n += 1
            for name, val in zip(cls.REASONS, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": n}


# ----------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(p, t_cpu, budget_s, rng):
    """Time the oracle on whole Q blocks (forward + dQ) and 64-slot key blocks (dK/dV).

    Returns the extrapolated fwd+bwd seconds for the whole workload and a description.
    """
    import torch
    import oracle

    n_qb = -(-p.q_slots // 64)
    n_kb = -(-p.kv_slots // 64)
    t_fwd = t_dq = t_kv = 0.0
    u_rows = u_keys = 0
    nq = nk = 0
    start = time.perf_counter()
    heads_cache = {}

    def head(h):
        if h not in heads_cache:
            heads_cache.clear()
            heads_cache[h] = tuple(t_cpu[n][0, h].to(torch.float64).numpy() for n in ("q", "k", "v", "do"))
        return heads_cache[h]

    while True:
        h = int(rng.integers(p.heads))
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        q, k, v, do = head(h)
        qb = int(rng.integers(n_qb))
        rows = np.arange(64 * qb, min(64 * qb + 64, p.q_slots))
        rows = rows[p.q_group[rows] >= 0]
        if rows.size:
            u_rows += int(oracle.token_mask(p.q_group, p.kv_group, A, rows).sum())
            t0 = time.perf_counter()
            oracle.forward_rows(q, k, v, p.q_group, p.kv_group, A, rows, p.scale)
            t1 = time.perf_counter()
            oracle.dq_rows(q, k, v, do, p.q_group, p.kv_group, A, rows, p.scale)
            t2 = time.perf_counter()
            t_fwd += t1 - t0
            t_dq += t2 - t1
            nq += 1
        if nq >= 2 * (nk + 1) or time.perf_counter() - start > budget_s * 0.5:
            kb = int(rng.integers(n_kb))
            keys = np.arange(64 * kb, min(64 * kb + 64, p.kv_slots))
            keys = keys[p.kv_group[keys] >= 0]
            if keys.size:
                kg = p.kv_group[keys]
                qv = p.q_group >= 0
                cnt = 0
                for g in np.unique(kg):
                    att = qv & A[np.where(qv, p.q_group, 0), g]
                    cnt += int(att.sum()) * int((kg == g).sum())
                u_keys += cnt
                t0 = time.perf_counter()
                oracle.dkdv_keys(q, k, v, do, p.q_group, p.kv_group, A, keys, p.scale)
                t_kv += time.perf_counter() - t0
                nk += 1
        if time.perf_counter() - start > budget_s and nq > 0 and nk > 0:
            break
    return dict(t_fwd=t_fwd, t_dq=t_dq, t_kv=t_kv, u_rows=u_rows, u_keys=u_keys, n_qblocks=nq, n_kblocks=nk,
                wall=time.perf_counter() - start)


def oracle_rates(p, U, s):
    """Extrapolated oracle seconds for the whole workload, from a sample."""
    t_fwd_all = s["t_fwd"] / max(s["u_rows"], 1) * U
    t_bwd_all = (s["t_dq"] / max(s["u_rows"], 1) + s["t_kv"] / max(s["u_keys"], 1)) * U
    return t_fwd_all, t_bwd_all


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        n = [d.get("num_threads") for d in info if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def useful_pairs(p):
    import oracle

    return oracle.useful_pairs_closed_form(p.q_group, p.kv_group, p.row_ptr, p.kv_groups, p.n_q_groups,
                                           p.n_kv_groups, p.heads, p.batch)


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------
def reduce_max(values, dist, device):
    """Element-wise max of `values` over all ranks: a multi-rank job takes as
    long as its slowest rank.  Without a process group, the values as given."""
    if dist is None:
        return [float(v) for v in values]
    import torch

    tt = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return tt.tolist()


def workload_config(p, args, world):
    """The `config` object of a bench line (the same keys for both arms)."""
    tensor_bytes = p.batch * p.heads * p.q_slots * p.head_dim * 2
    flush = tensor_bytes < 2 * L2_BYTES
    return {"workload": WORKLOAD_TEXT.get(args.workload, args.workload)
            + (f" (first {p.heads} heads only)" if args.heads else ""), "batch": p.batch, "heads": p.heads,
            "head_dim": p.head_dim, "q_slots": p.q_slots, "kv_slots": p.kv_slots,
            "valid_tokens": int((p.q_group >= 0).sum()),
            "l2": "flushed between steps" if flush else f"inputs larger than L2 ({tensor_bytes / 1e9:.2f} GB per tensor)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    p = W.make_problem(args.workload)
    if args.heads:
        p = W.with_heads(p, args.heads)
    t_cpu = W.make_tensors(p)
    U = useful_pairs(p)
    D = p.head_dim
    rng = np.random.default_rng(7)
    rates, samples = [], []
    budget = args.ref_step_seconds
    walls = []
    for i in range(args.warmup + args.steps):
        s = oracle_sample(p, t_cpu, budget, rng)
        if i >= args.warmup:
            walls.append(s["wall"])
        tf, tb = oracle_rates(p, U, s)
        if i >= args.warmup:
            rates.append(10 * D * U / (tf + tb) / 1e12)
            samples.append(s)
    value = statistics.mean(rates)
    cores = blas_threads()
    desc = (f"each step: the oracle on {samples[0]['n_qblocks']}+ Q blocks (forward + dQ) and "
            f"{samples[0]['n_kblocks']}+ 64-slot key blocks (dK/dV) of random heads, ~{budget:.0f} s of CPU work, "
            f"extrapolated to all {U} useful pairs")
    line = {
        "impl": "reference", "metric": "useful-pair TFLOP/s fwd+bwd (10*D per useful pair)", "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 10 * D * U / (value * 1e12) * 1e3,
        "ms_per_step_kind": ("extrapolated: the oracle's time for one whole step of the workload, from the timed "
                             "sample of each step"),
        "measured_ms_per_step": statistics.mean(walls) * 1e3,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(p, args, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def device_plan_ms(plan, p, dev, reps=5):
    """Median wall time of re-planning the workload's graph on the device
    (spattn_plan_set_graph_device, one stream synchronisation included).
    It switches the plan to slot-order tiles, so it runs after the timed
    steps."""
    import torch

    rp = torch.from_numpy(np.ascontiguousarray(p.row_ptr, dtype=np.int64)).to(dev)
    cols = torch.from_numpy(np.ascontiguousarray(p.kv_groups, dtype=np.int32)).to(dev)
    plan.set_graph_device(rp, cols)  # first call allocates the planner's device state
    times = []
    for _ in range(reps):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        plan.set_graph_device(rp, cols)
        torch.cuda.synchronize()
        times.append((time.perf_counter() - t0) * 1e3)
    return statistics.median(times)


def measure_fwd_fp8(plan, x, out, U, D, steps, peak_burst, flush, scratch):
    """The FP8 forward on the same plan and inputs: Q and K quantised once
    to E4M3 (timed on its own), then `steps` timed spattn_fwd_fp8 calls
    (CUDA events on the launch stream, L2 flushed between calls when the
    inputs fit in it).  Reported against the mixed peak of its two products:
    S at the fp8 rate (2x the measured bf16 burst, the nominal ratio) and
    P V at the bf16 rate."""
    import torch

    import block_sparse_attention_bwd_b200 as sp

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        q8, qds = sp.quantize_fp8(x["q"])
        k8, kds = sp.quantize_fp8(x["k"])
    torch.cuda.synchronize()
    e0.record(stream)
    q8, qds = sp.quantize_fp8(x["q"])
    k8, kds = sp.quantize_fp8(x["k"])
    e1.record(stream)
    torch.cuda.synchronize()
    quant_ms = e0.elapsed_time(e1)
    for _ in range(3):
        sp.spattn_fwd_fp8(q8, k8, qds, kds, x["v"], plan, o=out["o"], lse=out["lse"])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        if flush:
            scratch.zero_()
        a.record(stream)
        sp.spattn_fwd_fp8(q8, k8, qds, kds, x["v"], plan, o=out["o"], lse=out["lse"])
        b.record(stream)
    torch.cuda.synchronize()
    sp.spattn_check(plan)
    t = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    tflops = 4 * D * U / (t / 1e3) / 1e12
    peak_mixed = 2.0 / (1.0 / (2.0 * peak_burst) + 1.0 / peak_burst)
    return {"value": tflops, "unit": "TFLOP/s", "ms_per_step": t, "steps": steps, "quantize_q_k_ms": quant_ms,
            "dtype": "e4m3 Q, K (S = Q K^T on kind::f8f6f4); bf16 P, V, O",
            "peak_mixed": peak_mixed, "frac_of_mixed_peak": tflops / peak_mixed,
            "pct_of_bf16_peak": 100 * tflops / peak_burst}


def measure_workload(name, steps, warmup, dev, peak_burst):
    """fwd and fwd+bwd useful-pair TFLOP/s of one workload on resident inputs
    (CUDA events on the launch stream, L2 flushed between steps when the
    inputs fit in it), with the SM clocks sampled during the timed steps."""
    import torch

    import block_sparse_attention_bwd_b200 as sp

    p = W.make_problem(name)
    t_cpu = W.make_tensors(p)
    x = {k: v.to(dev) for k, v in t_cpu.items()}
    del t_cpu
    plan = sp.Plan.from_problem(p)
    st = plan.stats()
    U, D = st["useful_pairs"], p.head_dim
    out = {"o": torch.empty_like(x["q"]), "lse": torch.empty(x["q"].shape[:3], dtype=torch.float32, device=dev),
           "dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"])}
    flush = x["q"].numel() * 2 < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    stream = torch.cuda.current_stream()

    def fwd():
        return sp.spattn_fwd(x["q"], x["k"], x["v"], plan, o=out["o"], lse=out["lse"])

    def bwd(o, lse):
        sp.spattn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], plan, dq=out["dq"], dk=out["dk"], dv=out["dv"])

    for _ in range(warmup):
        bwd(*fwd())
    torch.cuda.synchronize()
    sp.spattn_check(plan)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    time.sleep(0.3)
    for i in range(steps):
        if flush:
            scratch.zero_()
        ev[i][0].record(stream)
        o, lse = fwd()
        ev[i][1].record(stream)
        bwd(o, lse)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    sp.spattn_check(plan)
    t_fwd = sum(a.elapsed_time(b) for a, b, _ in ev) / 1e3
    t_bwd = sum(b.elapsed_time(c) for _, b, c in ev) / 1e3
    fwd_tf = 4 * D * U * steps / t_fwd / 1e12
    all_tf = 10 * D * U * steps / (t_fwd + t_bwd) / 1e12
    res = {"workload": WORKLOAD_TEXT.get(name, name), "steps": steps, "warmup": warmup,
           "fwd_tflops": fwd_tf, "fwd_pct_of_bf16_burst": 100 * fwd_tf / peak_burst,
           "fwd_bwd_tflops": all_tf, "fwd_bwd_pct_of_bf16_burst": 100 * all_tf / peak_burst,
           "fwd_ms": t_fwd / steps * 1e3, "bwd_ms": t_bwd / steps * 1e3,
           "useful_pairs": U, "useful_over_physical_fwd": U / st["physical_pairs_fwd"],
           "useful_over_physical_dkdv": U / st["physical_pairs_dkdv"], "useful_over_bsa_64x64": U / st["bsa_pairs"],
           "plan_ms": st["plan_ms"], "sm_mhz": clk["sm_mhz"], "clock_reasons": clk["reasons"],
           "l2": "flushed between steps" if flush else "inputs larger than L2"}
    res["device_plan_ms"] = device_plan_ms(plan, p, dev)
    plan.close()
    del x, out, scratch
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch

    import block_sparse_attention_bwd_b200 as sp

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    peaks, peak_kind = load_peaks()

    p = W.make_problem(args.workload)
    if args.heads:
        p = W.with_heads(p, args.heads)
    t_cpu = W.make_tensors(p)
    x = {k: v.to(dev) for k, v in t_cpu.items()}
    plan = sp.Plan.from_problem(p)
    st = plan.stats()
    U = st["useful_pairs"]
    D = p.head_dim
    tensor_bytes = x["q"].numel() * 2
    flush = tensor_bytes < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    stream = torch.cuda.current_stream()

    def step():
        o, lse = sp.spattn_fwd(x["q"], x["k"], x["v"], plan, o=out["o"], lse=out["lse"])
        sp.spattn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], plan, dq=out["dq"], dk=out["dk"], dv=out["dv"])

    out = {"o": torch.empty_like(x["q"]), "lse": torch.empty(x["q"].shape[:3], dtype=torch.float32, device=dev),
           "dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"])}
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sp.spattn_check(plan)

    # ---------------- timed region ----------------
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    dev_uuid = None
    try:
        dev_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        dev_uuid = str(local)
    clocks = ClockSampler(dev_uuid)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    plan.profile(True)
    for i in range(args.steps):
        if flush:
            scratch.zero_()
        a, b, c = ev[i]
        a.record(stream)
        o, lse = sp.spattn_fwd(x["q"], x["k"], x["v"], plan, o=out["o"], lse=out["lse"])
        b.record(stream)
        sp.spattn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], plan, dq=out["dq"], dk=out["dk"], dv=out["dv"])
        c.record(stream)
    torch.cuda.synchronize()
    kt = plan.profile_read()
    plan.profile(False)
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    t_fwd = sum(a.elapsed_time(b) for a, b, _ in ev) / 1e3
    t_bwd = sum(b.elapsed_time(c) for _, b, c in ev) / 1e3
    t_total = t_fwd + t_bwd
    t_total, t_fwd, t_bwd = reduce_max([t_total, t_fwd, t_bwd], dist, dev)
    sp.spattn_check(plan)
    K = args.steps
    value = 10 * D * U * world * K / t_total / 1e12
    fwd_tflops = 4 * D * U * world * K / t_fwd / 1e12

    # ---------------- dominant kernel roofline ----------------
    kern = {}
    for name in ("fwd", "dkdv", "dq"):
        ms, n = kt[name]
        if n:
            avg = ms / n
            flops = KERNEL_FLOPS_PER_PAIR_D[name] * D * U
            kern[name] = {"avg_ms": avg, "launches": n, "tflops": flops / (avg / 1e3) / 1e12}
    dom = max(kern, key=lambda n: kern[n]["avg_ms"] * kern[n]["launches"])
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = kern[dom]["tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                "frac": achieved / peak_burst, "frac_of_sustained_peak": achieved / peak_sus,
                "peak_kind": f"{peak_kind} burst bf16 (the timed region is well under a second)",
                "traffic": traffic_record(dom, args.workload),
                "algorithmic_flops_per_launch": KERNEL_FLOPS_PER_PAIR_D[dom] * D * U}

    # ---------------- end to end through the public API with host buffers ----------------
    # Every step copies its four inputs from pinned host memory and its five
    # outputs back, inside the timed region.  Two device buffer sets and three
    # streams pipeline the steps the way a training loop would: step i's
    # uploads overlap step i-1's kernels and step i-2's downloads (the plan
    # runs on one stream only, as its workspace requires).
    e2e = None
    if args.e2e_steps > 0:
        host_in = {k: v.pin_memory() for k, v in t_cpu.items()}
        host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in out.items()}
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
        d2h = sum(v.numel() * v.element_size() for v in host_out.values())
        xs = [x, {k: torch.empty_like(v) for k, v in x.items()}]
        outs = [out, {k: torch.empty_like(v) for k, v in out.items()}]
        s_up, s_run, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(2)]
        run_done = [torch.cuda.Event() for _ in range(2)]
        out_free = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                xb, ob = xs[b], outs[b]
                with torch.cuda.stream(s_up):
                    if i >= 2:
                        s_up.wait_event(run_done[b])      # step i-2's kernels no longer read xb
                    for k, v in host_in.items():
                        xb[k].copy_(v, non_blocking=True)
                    in_ready[b].record(s_up)
                with torch.cuda.stream(s_run):
                    s_run.wait_event(in_ready[b])
                    if i >= 2:
                        s_run.wait_event(out_free[b])     # step i-2's outputs have been copied out
                    o, lse = sp.spattn_fwd(xb["q"], xb["k"], xb["v"], plan, o=ob["o"], lse=ob["lse"], stream=s_run)
                    sp.spattn_bwd(xb["q"], xb["k"], xb["v"], o, lse, xb["do"], plan, dq=ob["dq"], dk=ob["dk"],
                                  dv=ob["dv"], stream=s_run)
                    run_done[b].record(s_run)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(run_done[b])
                    for k, v in ob.items():
                        host_out[k].copy_(v, non_blocking=True)
                    out_free[b].record(s_down)

        e2e_steps(2)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_up)
        s_run.wait_stream(s_up)
        s_down.wait_stream(s_up)
        e2e_steps(args.e2e_steps)
        s_down.wait_stream(s_run)
        s_down.wait_stream(s_up)
        b.record(s_down)
        torch.cuda.synchronize()
        te = reduce_max([a.elapsed_time(b) / 1e3], dist, dev)[0]
        e2e = {"value": 10 * D * U * world * args.e2e_steps / te / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "pipelined": "two buffer sets, upload / kernels / download streams"}

    # ---------------- CPU baseline: the oracle on a bounded sample ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        s = oracle_sample(p, t_cpu, args.cpu_seconds, np.random.default_rng(11))
        tf, tb = oracle_rates(p, U, s)
        cpu = {"value": 10 * D * U / (tf + tb) / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"the fp64 oracle on {s['n_qblocks']} random Q blocks (forward + dQ rows) and "
                          f"{s['n_kblocks']} random 64-slot key blocks (dK/dV), {s['wall']:.1f} s of CPU work, "
                          f"extrapolated linearly by useful pairs to the whole workload"),
               "fwd_value": 4 * D * U / tf / 1e12}

    fp8 = None
    if rank == 0 and world == 1 and D == 128 and args.fp8_steps > 0:
        fp8 = measure_fwd_fp8(plan, x, out, U, D, args.fp8_steps, peak_burst, flush, scratch)

    dplan_ms = device_plan_ms(plan, p, dev) if rank == 0 else None

    # ---------------- every other large workload, measured the same way ----------------
    workloads = None
    if rank == 0 and world == 1 and args.other_workloads:
        workloads = {}
        for name in args.other_workloads.split(","):
            if name and name != args.workload:
                workloads[name] = measure_workload(name, args.other_steps, 3, dev, peak_burst)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "useful-pair TFLOP/s fwd+bwd (10*D per useful pair)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": t_total / K * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": workload_config(p, args, world),
        "fwd": {"value": fwd_tflops, "unit": "TFLOP/s", "ms_per_step": t_fwd / K * 1e3,
                "pct_of_bf16_peak": 100 * fwd_tflops / world / peak_burst},
        "bwd_ms_per_step": t_bwd / K * 1e3,
        "fwd_fp8": fp8,
        "fwd_bwd_14D_value": 14 * D * U * world * K / t_total / 1e12,
        "pct_of_bf16_peak": 100 * value / world / peak_burst,
        "pairs": {"useful": U, "physical_fwd": st["physical_pairs_fwd"], "physical_dkdv": st["physical_pairs_dkdv"],
                  "physical_dq": st["physical_pairs_dq"], "bsa_64x64": st["bsa_pairs"],
                  "useful_over_physical_fwd": U / st["physical_pairs_fwd"]},
        "kernels": kern,
        "plan_ms": st["plan_ms"],
        "device_plan_ms": dplan_ms,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int((st["launches_fwd"] + st["launches_bwd"]) * K),
        "clocks": clk,
        "peaks": {"bf16_tflops": peak_burst, "bf16_tflops_sustained": peak_sus, "kind": peak_kind},
        "workloads": workloads,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="partial", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--other-workloads", default="vsa,svg2,full",
                    help="after the headline, measure these workloads too (comma list; empty = none)")
    ap.add_argument("--other-steps", type=int, default=8)
    ap.add_argument("--fp8-steps", type=int, default=10,
                    help="timed calls of the FP8 (E4M3 Q/K) forward on the same workload; 0 skips it")
    ap.add_argument("--heads", type=int, default=0,
                    help="profile a slice: keep the layout, use the graph of the first N heads only")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
