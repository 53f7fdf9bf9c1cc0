#!/usr/bin/env python
"""Throughput of exact tiled attention (forward + backward) on B200.

One step is one pass of the whole path over one batch: the forward kernel
(O, LSE) followed by the backward pass (preprocess, dK/dV, dQ) on the default
workload B=2 H=16 N=2048 d=128, bf16, causal, inputs drawn N(0, 1) from a
fixed seed.  The metric is algorithmic TFLOP/s: 4*B*H*N^2*d forward plus
10*B*H*N^2*d backward, both halved under the causal mask.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same workload on its own GPU (independent
problems, no collective on the data path: weak scaling); the step time is the
maximum over ranks.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_35_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "attention fwd/bwd TFLOP/s (bf16) and % of B200 dense BF16 tensor peak"
DEFAULT_WORKLOAD = "fwdbwd_b2h16n2048d128_causal"
FWD_TARGET_WORKLOAD = "fwd_b2h32n4096d128_causal"
L2_FLUSH_BYTES = 256 << 20


def algorithmic_flops(w, backward=None):
    backward = w.backward if backward is None else backward
    half = 0.5 if w.causal else 1.0
    base = w.B * w.H * w.N * w.N * w.d * half
    fwd = 4.0 * base
    bwd = 10.0 * base if backward else 0.0
    return fwd, bwd


KERNEL_SOURCES = {
    "fwd::fwd_kernel<128>": ["exact_tiled_attention_35_b200/csrc/fa_device.cuh",
                             "exact_tiled_attention_35_b200/csrc/fa_fwd_sm100.cu"],
    "bwd::main_kernel<128>": ["exact_tiled_attention_35_b200/csrc/fa_device.cuh",
                              "exact_tiled_attention_35_b200/csrc/fa_bwd_sm100.cu"],
}


def kernel_source_hash(kernel):
    import hashlib

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/traffic.json,
    or None when absent or captured from other sources of that kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get("kernels", {}).get(kernel)
    if not entry or entry.get("workload") != workload:
        return None
    if entry.get("source_sha256") != kernel_source_hash(kernel):
        return None
    return entry.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]), "hbm_gbs": float(p["hbm_gbs"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons for one GPU while running."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", "GPU-" + self.uuid if not self.uuid.startswith("GPU-") else self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append((float(parts[2]), float(parts[3]), float(parts[4]), parts[5:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        loaded = [r for r in rows if r[2] > 300.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ distributed


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- CPU oracle


def oracle_sample(w, budget_s, seed=0):
    """Times the fp64 oracle on whole heads of the workload until budget_s passes.

    Returns (flops done, seconds, heads, cores)."""
    from oracle import attention_bwd_ref, attention_fwd_ref

    q, k, v, do = make_inputs(1, 1, w.N, w.d, dtype=w.dtype, seed=seed, qk_gain=w.qk_gain, with_do=True)
    q, k, v, do = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    fwd, bwd = algorithmic_flops(w)
    per_head = (fwd + bwd) / (w.B * w.H)
    done, t0 = 0, time.perf_counter()
    while True:
        attention_fwd_ref(q, k, v, w.scale, w.causal)
        if w.backward:
            attention_bwd_ref(q, k, v, do, w.scale, w.causal)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= w.B * w.H:
            break
    cores = len(os.sched_getaffinity(0))
    return per_head * done, el, done, cores


def run_reference(args, w, world, rank):
    """The oracle as it stands, on this host's cores: each step one bounded sample."""
    if rank != 0:
        return
    fwd, bwd = algorithmic_flops(w)
    for _ in range(args.warmup):
        oracle_sample(w, 0.0)
    times, flops = [], 0.0
    for _ in range(args.steps):
        f, el, heads, cores = oracle_sample(w, 0.0)
        times.append(el)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                                        "causal": w.causal, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle",
                         "sample": f"one (b,h) head of {w.name} per step ({'fwd+bwd' if w.backward else 'fwd'} "
                                   f"fp64, full N x N)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm


def run_ours(args, w, world, rank, local):
    import exact_tiled_attention_35_b200 as fa

    dev = torch.device("cuda", torch.cuda.current_device())
    fa.load_library()
    fwd_flops, bwd_flops = algorithmic_flops(w)
    step_flops = fwd_flops + bwd_flops
    q, k, v, do = make_inputs(w.B, w.H, w.N, w.d, dtype=w.dtype, seed=rank, qk_gain=w.qk_gain, with_do=True)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(max(fa.workspace_size(w.B, w.H, w.N, w.d), 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        fa.forward(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
        if w.backward:
            fa.backward(qd, kd, vd, o, dod, lse, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                        workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    fa.check_device_status()
    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    clocks = ClockSampler(dev)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for i in range(n):
        if not args.keep_l2:
            flush.zero_()  # L2 (126 MB) flushed between timed steps
        ev[i][0].record()
        fa.forward(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
        ev[i][1].record()
        if w.backward:
            fa.backward(qd, kd, vd, o, dod, lse, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                        workspace=ws)
        ev[i][2].record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    fa.check_device_status()
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
    step_ms = statistics.mean(a + b for a, b in zip(fwd_ms, bwd_ms))
    step_ms = max_over_ranks(step_ms, world)
    value = world * step_flops / (step_ms * 1e-3) / 1e12

    # end to end through the public API: pinned host inputs in, results back out
    hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
    ho, hlse, hdq, hdk, hdv = (torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                               for t in (o, lse, dq, dk, dv))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdq, hdk, hdv))
    if not w.backward:
        h2d -= hdo.numel() * hdo.element_size()
        d2h = ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size()

    def e2e_step():
        qd.copy_(hq, non_blocking=True)
        kd.copy_(hk, non_blocking=True)
        vd.copy_(hv, non_blocking=True)
        if w.backward:
            dod.copy_(hdo, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)
        if w.backward:
            hdq.copy_(dq, non_blocking=True)
            hdk.copy_(dk, non_blocking=True)
            hdv.copy_(dv, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    barrier(world)
    fa.check_device_status()

    # forward alone on the long causal workload (the tensor-peak target)
    fw = WORKLOADS[FWD_TARGET_WORKLOAD]
    fwd_only = None
    if not args.skip_fwd_target:
        fq, fk, fv = (t.to(dev) for t in make_inputs(fw.B, fw.H, fw.N, fw.d, seed=rank))
        fo = torch.empty_like(fq)
        flse = torch.empty((fw.B, fw.H, fw.N), dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            fa.forward(fq, fk, fv, causal=True, out=fo, lse=flse)
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        torch.cuda.synchronize()
        for i in range(n):
            flush.zero_()
            fev[i][0].record()
            fa.forward(fq, fk, fv, causal=True, out=fo, lse=flse)
            fev[i][1].record()
        torch.cuda.synchronize()
        fa.check_device_status()
        f_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in fev), world)
        ff = algorithmic_flops(fw, backward=False)[0]
        fwd_only = {"workload": fw.name, "ms": f_ms, "tflops": ff / (f_ms * 1e-3) / 1e12}
        del fq, fk, fv, fo, flse

    peaks = measured_peaks()
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms) if w.backward else 0.0
    if bwd_avg > fwd_avg:
        dom = {"kernel": "bwd::main_kernel<%d>" % w.d, "flops": bwd_flops, "ms": bwd_avg,
               "timed": "fa_backward as a whole: preprocess + main + dQ convert launches (the main kernel is ~83% of them in the ncu launch list), so achieved is a lower bound for the main kernel"}
    else:
        dom = {"kernel": "fwd::fwd_kernel<%d>" % w.d, "flops": fwd_flops, "ms": fwd_avg,
               "timed": "fa_forward: one launch"}
    achieved = dom["flops"] / (dom["ms"] * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": dom["kernel"], "timed": dom["timed"], "achieved": achieved,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "peak_source": peaks["source"] + " bf16 burst (MEASURED_PEAKS.json)",
            "traffic": profiled_traffic(dom["kernel"], w.name)}
    if fwd_only is not None:
        fwd_only["frac_of_peak"] = fwd_only["tflops"] / peaks["bf16_tflops"]
        fwd_only["roofline"] = {
            "bound": "tensor", "kernel": "fwd::fwd_kernel<128>", "achieved": fwd_only["tflops"],
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": fwd_only["frac_of_peak"],
            "peak_source": peaks["source"] + " bf16 burst (MEASURED_PEAKS.json)",
            "traffic": profiled_traffic("fwd::fwd_kernel<128>", fw.name)}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        f, el, heads, cores = oracle_sample(w, args.cpu_budget)
        cpu = {"value": f / el / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{heads} (b,h) head(s) of {w.name}, {'fwd+bwd' if w.backward else 'fwd'} in fp64 "
                         f"with the full N x N matrix, {el:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": n,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "global_batch": world * w.B, "seq_len": w.N, "parallelism": f"replicas{world}",
                       "l2": ("kept between timed steps (--keep-l2, a diagnostic: inputs may stay "
                              "L2-resident)" if args.keep_l2 else "flushed between timed steps (256 MB write)")},
            "breakdown_ms": {"forward": fwd_avg, "backward": bwd_avg},
            "frac_of_peak": value / world / peaks["bf16_tflops"],
            "roofline": roof,
            "forward_target": fwd_only,
            "cpu_baseline": cpu,
            "e2e": {"value": world * step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": n * (1 + (3 if w.backward else 0)),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle CPU work")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-fwd-target", action="store_true")
    ap.add_argument("--keep-l2", action="store_true",
                    help="do not flush L2 between timed steps (diagnostic for the small workloads; "
                         "the default flushes)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
