"""Benchmark of one DraftAttention2 attention call on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload video] [--impl ours|reference]

A step is one whole call — da2_prepare (reorder, pool, quantise), da2_draft_rank
(draft map, ranking, assignment) and da2_attention (mixed-precision attention,
output restored to token order) — on the 118,800-token (33x45x80 latent),
24-head, d=128 bf16 workload with budget skip/4/8/16 = 85/0/7.5/7.5 and
lambda = 0.5, seeded synthetic blob + noise + outlier inputs resident in HBM.
Each input tensor (730 MB) is larger than L2, so no flush is needed.

Printed on rank 0, one JSON line: effective (dense-equivalent) TFLOP/s of the
whole job, ms per call, the roofline of the attention kernel, the own dense
bf16 kernel on the same inputs, an end-to-end figure through host buffers,
SM clocks sampled during the timed region, and the CPU oracle as a reported
baseline.  ``--impl reference`` times the CPU oracle alone (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "attention-call ms + effective TFLOP/s (118.8K tok, 24 heads) vs own dense bf16"
UNIT = "TFLOP/s (dense-equivalent)"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return PEAK_FALLBACK, "fallback"


def phase_flops(wl, info):
    """Executed MMA FLOPs per phase: 4 * 64 * 64 * d per retained block pair."""
    per_pair = 4.0 * 64 * 64 * wl.d
    bh = wl.B * wl.H
    return {16: per_pair * info.n16 * bh, 8: per_pair * info.n8 * bh, 4: per_pair * info.n4 * bh}


def prep_bytes(wl, info):
    """Algorithmic bytes of the preparation stage: read Q, K, V (bf16) once;
    write the pooled descriptors (avg and max of Q and K, fp32) and only the
    formats the budget uses — INT8: Q/K codes of every 64-token block slot,
    one fp32 scale per block, V codes and one fp32 scale per channel; NVFP4:
    Q/K/V codes (4 bits), one e4m3 scale per 16 elements, V's fp32 channel
    scale."""
    bh, nb, d, S = wl.B * wl.H, info.nb, wl.d, 64
    b = 3 * bh * wl.N * d * 2 + 4 * bh * nb * d * 4
    if info.n8:
        b += 2 * (bh * nb * S * d + bh * nb * 4) + bh * nb * d * S + bh * d * 4
    if info.n4:
        b += 3 * (bh * nb * S * d // 2 + bh * nb * S * d // 16) + bh * d * 4
    return b


# XU-pipe work per retained 64x64 block pair in the attention kernel: one ex2
# per score, plus the F2FP conversions that issue to the same pipe (16-bit: one
# bf16x2 per two probabilities; 4-bit: one e2m1x2 per two and one e4m3 per
# sixteen; INT8 codes are formed on the FMA pipe).  The pipe retires 16 lanes
# per clock per SM (4,096 ex2 per sub-partition took ~1,030 cycles in a probe).
XU_PER_PAIR = {16: 64 * 64 * 1.5, 8: 64 * 64 * 1.0, 4: 64 * 64 * (1.5 + 1.0 / 16)}
XU_LANES_PER_CLK_SM = 16
SMS = 148


def roofline(wl, info, attn_ms, call_ms, pk, pk_kind, mhz):
    """The path's roofline, as the method's measurement defines it: each
    phase's executed MMA FLOPs at its format's peak (bf16 the measured burst
    cuBLAS figure, INT8 x2, NVFP4 x4 — the nominal ratios) plus the
    preparation's algorithmic bytes at the measured HBM bandwidth.

    ``frac`` is the attention kernel's tensor fraction: its phase-weighted
    floor over its measured time (achieved = executed FLOPs / time against the
    phase-weighted peak).  ``whole_call`` divides the whole floor (tensor +
    prep bytes) by the whole call.  ``xu_floor_ms`` is an extra, labelled
    bound: the softmax's work on the XU pipe (ex2 and F2FP conversions) at 16
    lanes per clock per SM at the sampled clock."""
    bf16 = pk["bf16_tflops"]
    pf = phase_flops(wl, info)
    f_tot = sum(pf.values())
    t_tensor = pf[16] / (bf16 * 1e12) + pf[8] / (2 * bf16 * 1e12) + pf[4] / (4 * bf16 * 1e12)
    pb = prep_bytes(wl, info)
    t_prep = pb / (pk["hbm_gbs"] * 1e9)
    bh = wl.B * wl.H
    xu_ops = bh * (info.n16 * XU_PER_PAIR[16] + info.n8 * XU_PER_PAIR[8] + info.n4 * XU_PER_PAIR[4])
    xu_peak = XU_LANES_PER_CLK_SM * SMS * mhz * 1e6
    achieved = f_tot / (attn_ms * 1e-3) / 1e12
    peak_blend = f_tot / t_tensor / 1e12 if t_tensor > 0 else bf16
    return {
        "bound": "tensor", "kernel": "attn_tc_kernel", "achieved": achieved, "peak": peak_blend,
        "unit": "TFLOP/s", "frac": achieved / peak_blend,
        "peak_note": (f"phase-weighted: bf16 {bf16:.1f} TFLOP/s (burst, {pk_kind}), int8 x2, nvfp4 x4; "
                      f"executed FLOPs 16/8/4 = {pf[16] / 1e12:.2f}/{pf[8] / 1e12:.2f}/{pf[4] / 1e12:.2f} T"),
        "floor_ms": {"tensor": t_tensor * 1e3, "prep_hbm": t_prep * 1e3},
        "whole_call": {"floor_ms": (t_tensor + t_prep) * 1e3, "ms": call_ms,
                       "frac": (t_tensor + t_prep) * 1e3 / call_ms, "prep_bytes": pb,
                       "hbm_gbs": pk["hbm_gbs"]},
        "xu_floor_ms": xu_ops / xu_peak * 1e3,
    }


def max_over_ranks(x, device, world):
    """The largest of the ranks' values; every rank takes the same collective."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, flops_per_rank, ms):
    """Whole-job throughput (TFLOP/s): every rank's work over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def launches_per_call(info, d):
    """Kernels this library launches per call (its own kernels only)."""
    v = 1 if (info.n8 or info.n4) else 0  # the V preparation (absmax and codes in one kernel)
    prep = 1 + v
    draft = 2  # logits + mix (mix carries the first ranking histogram)
    rank = 1 + 8 + 7 + 1  # init, 8 selects, 7 histogram passes, assign
    pairs = 1  # merged key lists of the query-block pairs
    attn = 1  # the tensor-core attention kernel
    return prep + draft + rank + pairs + attn


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        else:
            self.lines = []

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except (ValueError, IndexError):
                continue
            for n, val in zip(names, f[3:7]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"]}
        # samples under load: the upper half of the readings
        load = sorted(sm)[len(sm) // 2:]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_sample(wl, frames=4, seed=0):
    """Time the CPU oracle on a bounded sample and extrapolate to one whole call.

    The sample is the same workload cut to its first ``frames`` latent frames
    and one head (same grid, regions, d, budget, lambda), run through every
    stage in full.  Each stage is scaled to the full workload by its own
    complexity: prep by tokens, draft by region pairs, ranking by pairs x
    log(pairs), attention by kept block pairs, and all by the head count.
    Returns (seconds per call, cores, description)."""
    import math
    import numpy as np
    import torch
    from oracle import draft as ODR, geometry as OG, prep as OP, rank as OR, attention as OA
    from oracle.problem import Problem as OProblem
    from mixed_precision_block_b200.synth import make_qkv

    small = wl.with_(H=1, B=1, T=min(frames, wl.T))
    q, k, v = make_qkv(small, "cpu", seed=seed)
    op = OProblem.from_workload(small)
    full = OProblem.from_workload(wl)
    qh, kh, vh = (x[0, 0].float().numpy().astype(np.float64) for x in (q, k, v))
    t0 = time.perf_counter()
    table = OG.block_tokens(op)
    pr = OP.prepare_head(op, qh, kh, vh, table)
    t1 = time.perf_counter()
    D = ODR.draft_scores(pr["q_avg"], pr["k_avg"], pr["q_max"], pr["k_max"], op.lam, op.d)
    t2 = time.perf_counter()
    n16, n8, n4, _ = OG.budget_counts(op)
    pmap = OR.assign(D, n16, n8, n4)
    t3 = time.perf_counter()
    OA.head_attention(pr, pmap, op.d, "emulate")
    t4 = time.perf_counter()
    P_s, P_f = op.nb ** 2, full.nb ** 2
    f16, f8, f4, _ = OG.budget_counts(full)
    kept_s, kept_f = n16 + n8 + n4, f16 + f8 + f4
    head_s = ((t1 - t0) * full.N / op.N + (t2 - t1) * P_f / P_s
              + (t3 - t2) * (P_f * math.log(P_f)) / (P_s * math.log(P_s))
              + (t4 - t3) * kept_f / max(kept_s, 1))
    call_s = head_s * wl.B * wl.H
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = torch.get_num_threads()
    desc = (f"oracle (numpy fp64) on 1 head of the first {small.T} of {wl.T} frames "
            f"({op.N} tokens, {op.nb} regions): prep {t1 - t0:.2f} s, draft {t2 - t1:.2f} s, "
            f"rank {t3 - t2:.2f} s, attention {t4 - t3:.2f} s; scaled per stage by tokens, pairs, "
            f"pairs*log(pairs), kept pairs, and x{wl.B * wl.H} heads")
    return call_s, cores, desc


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mixed_precision_block_b200.synth import dense_flops
    flops = dense_flops(wl)
    times, cores, desc = [], 1, ""
    for i in range(args.warmup + args.steps):
        s, cores, desc = cpu_oracle_sample(wl, frames=args.ref_frames, seed=i)
        if i >= args.warmup:
            times.append(s)
    sec = statistics.mean(times)
    val = flops / sec / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, args),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, args):
    return {"workload": f"{wl.name}: B={wl.B} H={wl.H} grid {wl.T}x{wl.Hh}x{wl.Ww} "
                        f"({wl.N} tokens) d={wl.d} regions {wl.rh}x{wl.rw}",
            "budget_skip_4_8_16": list(wl.budget), "lambda": wl.lam, "seed": wl.seed,
            "inputs": "bf16 blob+noise+outlier, each tensor larger than L2 (no flush)",
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}


def traffic_record(kernel, kernel_src, workload):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, or None if the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    return rec.get("dram_bytes_per_launch") if rec.get("source_sha256") == h else None


def run_ours(args, wl):
    import torch
    import torch.distributed as dist
    from mixed_precision_block_b200 import da2
    from mixed_precision_block_b200.synth import make_qkv, dense_flops

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    q, k, v = make_qkv(wl, dev)
    p = da2.Problem.from_workload(wl)
    info = da2.da2_plan(p)
    ws = da2.workspace(p, dev)
    out = torch.empty_like(q)
    st = torch.cuda.Stream(dev)
    flops = dense_flops(wl)

    def barrier():
        if world > 1:
            dist.barrier()

    def step(ev=None):
        if ev is not None:
            ev[0].record(st)
        da2.da2_prepare(p, q, k, v, ws, st)
        if ev is not None:
            ev[1].record(st)
        da2.da2_draft_rank(p, ws, st)
        if ev is not None:
            ev[2].record(st)
        da2.da2_attention(p, q, k, v, ws, out, st)
        if ev is not None:
            ev[3].record(st)

    with torch.cuda.stream(st):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(st)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(st)
        torch.cuda.synchronize(dev)
    barrier()
    ms = t_start.elapsed_time(t_end) / args.steps
    stage = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j in range(3)]
    ms = max_over_ranks(ms, dev, world)
    value = whole_job_value(world, flops, ms)

    # own dense bf16 kernel on the same inputs
    dense_ms = None
    if args.dense_steps > 0:
        dense_out = torch.empty_like(q)
        with torch.cuda.stream(st):
            da2.da2_dense_attention(q, k, v, dense_out, st)
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(st)
            for _ in range(args.dense_steps):
                da2.da2_dense_attention(q, k, v, dense_out, st)
            d1.record(st)
        torch.cuda.synchronize(dev)
        dense_ms = d0.elapsed_time(d1) / args.dense_steps
        del dense_out

    # end to end through host buffers: pinned H2D of Q/K/V, the call, D2H of O
    e2e = None
    if not args.no_e2e:
        # the public host-buffer call: chunks of heads, the copies of one chunk
        # overlapped with the kernels of another, synchronous
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hbuf = da2.host_buffer(p, args.e2e_chunk, dev)

        def e2e_step():
            da2.da2_forward_host(p, hq, hk, hv, hout, hbuf, args.e2e_chunk, st)

        with torch.cuda.stream(st):
            e2e_step()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(st)
            for _ in range(args.e2e_steps):
                e2e_step()
            a1.record(st)
        torch.cuda.synchronize(dev)
        e_ms = a0.elapsed_time(a1) / args.e2e_steps
        e_ms = max_over_ranks(e_ms, dev, world)
        nbytes = q.numel() * q.element_size()
        e2e = {"value": whole_job_value(world, flops, e_ms), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "call": f"da2_forward_host on pinned host tensors, chunks of {args.e2e_chunk} (batch, head) slices"}
        del hq, hk, hv, hout, hbuf

    traffic = traffic_record("attn_tc_kernel", os.path.join(ROOT, "mixed_precision_block_b200", "csrc", "attn_tc.cu"),
                             wl.name)
    clocks = clk.summary()
    pk, pk_kind = peaks()
    roof = roofline(wl, info, stage[2], ms, pk, pk_kind, (clocks or {}).get("sm_mhz") or 1965.0)
    roof["traffic"] = traffic

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu:
            s, cores, desc = cpu_oracle_sample(wl, frames=args.cpu_frames)
            cpu = {"value": flops / s / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16+int8+nvfp4 (fp32 accumulate)", "data": "synthetic",
            "config": config_of(wl, args),
            "stages_ms": {"prepare": stage[0], "draft_rank": stage[1], "attention": stage[2]},
            "dense_bf16": None if dense_ms is None else {
                "ms": dense_ms, "tflops": flops / (dense_ms * 1e-3) / 1e12,
                "speedup_of_sparse_call": dense_ms / ms},
            "roofline": roof,
            "e2e": e2e, "gpu_launches": launches_per_call(info, wl.d) * args.steps, "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


SWEEP_BUDGETS = [  # skip / 4-bit / 8-bit / 16-bit percentages
    (95, 0, 0, 5), (90, 0, 0, 10), (85, 0, 0, 15), (80, 0, 0, 20), (70, 0, 0, 30),
    (90, 0, 10, 0), (85, 0, 15, 0), (80, 0, 20, 0), (70, 0, 30, 0),
    (90, 10, 0, 0), (85, 15, 0, 0), (80, 20, 0, 0), (70, 30, 0, 0),
    (85, 0, 7.5, 7.5), (80.7, 14.4, 4.8, 0), (80, 10, 5, 5), (70, 20, 8, 2),
]
SWEEP_LAMBDAS = [0.0, 0.25, 0.5, 0.75, 1.0]


def run_sweep(args, wl):
    """Fidelity against latency on one GPU: for a grid of budgets (the Pareto
    view of the method's allocation) and for lambda at the workload's budget
    (average-only versus average + max drafting), the call time (CUDA events,
    median of a few calls) and the relative L2 error of the output against the
    own dense bf16 attention on the same inputs.  One JSON line per point."""
    import torch
    from mixed_precision_block_b200 import da2
    from mixed_precision_block_b200.synth import make_qkv

    dev = torch.device("cuda", 0)
    q, k, v = make_qkv(wl, dev)
    ref = torch.empty_like(q)
    da2.da2_dense_attention(q, k, v, ref)
    torch.cuda.synchronize()
    ref32 = ref.float()
    ref_norm = float(ref32.norm())
    out = torch.empty_like(q)
    points = [(b, wl.lam) for b in SWEEP_BUDGETS] + [(tuple(wl.budget), lam) for lam in SWEEP_LAMBDAS]
    for budget, lam in points:
        p = da2.Problem.from_workload(wl, budget=budget, lam=lam)
        ws = da2.workspace(p, dev)
        times = []
        for it in range(1 + args.sweep_calls):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record()
            da2.da2_prepare(p, q, k, v, ws)
            da2.da2_draft_rank(p, ws)
            e[1].record()
            da2.da2_attention(p, q, k, v, ws, out)
            e[2].record()
            torch.cuda.synchronize()
            if it:
                times.append((e[0].elapsed_time(e[2]), e[1].elapsed_time(e[2])))
        times.sort()
        call_ms, attn_ms = times[len(times) // 2]
        err = float((out.float() - ref32).norm()) / ref_norm
        print(json.dumps({"sweep": wl.name, "budget_skip_4_8_16": list(budget), "lambda": lam,
                          "call_ms": call_ms, "attention_ms": attn_ms, "rel_l2_vs_own_dense": err}), flush=True)
        del ws


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="video")
    ap.add_argument("--lam", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None, help="run only this many heads (profiling captures)")
    ap.add_argument("--dense-steps", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunk", type=int, default=3, help="(batch, head) slices per chunk of the host-buffer call")
    ap.add_argument("--ref-frames", type=int, default=2, help="frames per CPU oracle sample (reference arm)")
    ap.add_argument("--cpu-frames", type=int, default=8, help="frames of the CPU-baseline oracle sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="budget and lambda sweep: call time and error against the own dense kernel")
    ap.add_argument("--sweep-calls", type=int, default=3)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # fewer warm-up steps would not give a valid number
    from mixed_precision_block_b200.synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.lam is not None:
        wl = wl.with_(lam=args.lam)
    if args.heads is not None:
        wl = wl.with_(H=args.heads)
    if args.sweep:
        run_sweep(args, wl)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
