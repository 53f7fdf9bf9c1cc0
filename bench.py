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
    """Samples nvidia-smi clocks and throttle reasons for one GPU while running.

    Rows carry nvidia-smi's timestamp, so the samples of a time window (for
    example the timed steps and the soak right before them) can be picked out."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device, interval_ms=50):
        self.proc = None
        self.path = None
        self.interval_ms = interval_ms
        self.rows = []
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", str(self.interval_ms)]
            if self.uuid:
                cmd += ["-i", "GPU-" + self.uuid if not self.uuid.startswith("GPU-") else self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        import datetime

        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    self.rows.append((ts, float(parts[2]), float(parts[3]), float(parts[4]), parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)

    def summary(self, t0=None, t1=None, what=""):
        """Clock record of the samples taken between host times t0 and t1."""
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for name, flag in zip(self.REASONS, r[4]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        loaded = [r for r in rows if r[3] > 300.0] or rows
        return {"sm_mhz": statistics.median(r[1] for r in loaded), "sm_max_mhz": max(r[2] for r in rows),
                "power_w_max": max(r[3] for r in rows), "samples": len(rows),
                "samples_under_load": len([r for r in rows if r[3] > 300.0]),
                "window_s": round(rows[-1][0] - rows[0][0], 3), "reasons": sorted(reasons),
                "covers": what}


# ------------------------------------------------------------ distributed


def dist_setup(backend=None):
    """One process per GPU from torchrun's environment; NCCL on GPUs (gloo when
    asked, for host-only runs of the same plumbing).  Returns (world, rank, local)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
    if world > 1:
        import datetime

        import torch.distributed as dist

        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
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

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
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


def _vp(t):
    import ctypes

    return ctypes.c_void_p(t.data_ptr())


class Problem:
    """Device buffers of one workload plus pre-marshalled C-ABI argument lists, so
    the timed loops call the library with no per-call Python checks."""

    def __init__(self, w, dev, seed, lib, stream):
        import ctypes

        self.w = w
        ts = make_inputs(w.B, w.H, w.N, w.d, dtype=w.dtype, seed=seed, qk_gain=w.qk_gain,
                         with_do=w.backward)
        q, k, v = ts[:3]
        do = ts[3] if w.backward else None
        self.host = list(ts)
        self.q, self.k, self.v = (t.to(dev) for t in (q, k, v))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        st = ctypes.c_void_p(stream.cuda_stream)
        causal = int(w.causal)
        self.fwd_fn = lib.fa_forward if w.dtype == torch.bfloat16 else lib.fa_forward_fp32
        if w.backward and w.dtype != torch.bfloat16:
            raise ValueError("the timed backward runs the bf16 path")
        self.fwd_args = (_vp(self.q), _vp(self.k), _vp(self.v), _vp(self.o), _vp(self.lse), w.B, w.H, w.N,
                         w.d, w.scale, causal, st)
        if w.backward:
            self.do = do.to(dev)
            self.dq, self.dk, self.dv = (torch.empty_like(t) for t in (self.q, self.k, self.v))
            ws_bytes = int(lib.fa_backward_workspace_size(w.B, w.H, w.N, w.d))
            self.ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
            self.bwd_fn = lib.fa_backward_stages
            self.bwd_args = [_vp(t) for t in (self.q, self.k, self.v, self.o, self.do, self.lse, self.dq,
                                               self.dk, self.dv, self.ws)]
            self.bwd_tail = (self.ws.numel(), w.B, w.H, w.H, w.N, w.N, w.d, w.scale, causal)
            self.stream = st

    def forward(self):
        return self.fwd_fn(*self.fwd_args)

    def backward(self, stages):
        return self.bwd_fn(*self.bwd_args, *self.bwd_tail, stages, self.stream)


def _check_codes(codes, fa):
    bad = [c for c in codes if c != 0]
    if bad:
        raise fa.FAError(bad[0], "bench launch")


def time_forward(prob, flush, steps, warmup, fa, keep_l2=False):
    """Mean device time (ms) of one forward launch over `steps` launches, L2
    flushed before each (unless keep_l2)."""
    codes = []
    for _ in range(warmup):
        flush.zero_()
        codes.append(prob.forward())
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        if not keep_l2:
            flush.zero_()
        e0.record()
        codes.append(prob.forward())
        e1.record()
    torch.cuda.synchronize()
    _check_codes(codes, fa)
    fa.check_device_status()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def run_ours(args, w, world, rank, local):
    import exact_tiled_attention_35_b200 as fa

    dev = torch.device("cuda", torch.cuda.current_device())
    lib = fa.load_library()
    stream = torch.cuda.current_stream(dev)
    peaks = measured_peaks()
    fwd_flops, bwd_flops = algorithmic_flops(w)
    step_flops = fwd_flops + bwd_flops
    prob = Problem(w, dev, rank, lib, stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    codes = []

    def step(i=None, ev=None):
        # forward, then the backward's three stages; events (when given) mark
        # the boundaries on the launching stream
        if ev is not None:
            ev[0].record()
        codes.append(prob.forward())
        if ev is not None:
            ev[1].record()
        if w.backward:
            for s_i, stage in enumerate((fa.STAGE_PREPROCESS, fa.STAGE_MAIN, fa.STAGE_DQ_CONVERT)):
                codes.append(prob.backward(stage))
                if ev is not None:
                    ev[2 + s_i].record()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    _check_codes(codes, fa)
    fa.check_device_status()

    # Clock soak: the same step, untimed, for about a second right before the
    # timed steps, so the clock sampler sees the GPU under this load.
    clocks = ClockSampler(dev)
    clocks.start()
    t_soak = time.time()
    while time.time() - t_soak < args.soak_s:
        for _ in range(20):
            flush.zero_()
            step()
        torch.cuda.synchronize()
    n = args.steps
    nev = 5 if w.backward else 2
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(n):
        if not args.keep_l2:
            flush.zero_()  # L2 (126 MB) flushed between timed steps
        step(i, ev[i])
    torch.cuda.synchronize()
    barrier(world)
    t_timed_end = time.time()
    _check_codes(codes, fa)
    fa.check_device_status()
    seg = [[e[j].elapsed_time(e[j + 1]) for e in ev] for j in range(nev - 1)]
    fwd_ms = statistics.mean(seg[0])
    step_ms = statistics.mean(e[0].elapsed_time(e[nev - 1]) for e in ev)
    step_ms = max_over_ranks(step_ms, world)
    value = world * step_flops / (step_ms * 1e-3) / 1e12
    breakdown = {"forward": fwd_ms}
    if w.backward:
        breakdown.update({"bwd_preprocess": statistics.mean(seg[1]), "bwd_main": statistics.mean(seg[2]),
                          "bwd_dq_convert": statistics.mean(seg[3])})
        breakdown["backward"] = breakdown["bwd_preprocess"] + breakdown["bwd_main"] + breakdown["bwd_dq_convert"]

    # the dominant kernel of the step and its roofline (tensor-bound: FLOPs)
    if w.backward and breakdown["bwd_main"] > fwd_ms:
        dom = {"kernel": "bwd::main_kernel<%d>" % w.d, "flops": bwd_flops, "ms": breakdown["bwd_main"],
               "timed": "the backward main kernel alone: CUDA events around its launch on the launching stream"}
    else:
        dom = {"kernel": "fwd::fwd_kernel<%d>" % w.d, "flops": fwd_flops, "ms": fwd_ms,
               "timed": "the forward kernel alone: CUDA events around its launch on the launching stream"}
    achieved = dom["flops"] / (dom["ms"] * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": dom["kernel"], "timed": dom["timed"], "achieved": achieved,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
            else "fallback bf16 burst (no MEASURED_PEAKS.json)",
            "traffic": profiled_traffic(dom["kernel"], w.name)}

    # the deterministic backward on the same workload (separate dQ pass), its
    # three stages timed the same way
    extras = {}
    if w.backward and not args.skip_extras:
        det = fa.STAGE_DETERMINISTIC
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for _ in range(args.warmup):
            flush.zero_()
            for stage in (fa.STAGE_PREPROCESS, fa.STAGE_MAIN, fa.STAGE_DQ_CONVERT):
                codes.append(prob.backward(stage | det))
        torch.cuda.synchronize()
        for e in ev2:
            flush.zero_()
            e[0].record()
            for s_i, stage in enumerate((fa.STAGE_PREPROCESS, fa.STAGE_MAIN, fa.STAGE_DQ_CONVERT)):
                codes.append(prob.backward(stage | det))
                e[s_i + 1].record()
        torch.cuda.synchronize()
        _check_codes(codes, fa)
        fa.check_device_status()
        seg2 = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev2) for j in range(3)]
        tot = max_over_ranks(sum(seg2), world)
        extras["backward_deterministic"] = {
            "workload": w.name, "ms": tot, "tflops": bwd_flops / (tot * 1e-3) / 1e12,
            "breakdown_ms": {"preprocess": seg2[0], "main_dk_dv": seg2[1], "dq_pass": seg2[2]},
            "note": "fa_backward_deterministic's three launches; TFLOP/s on the same algorithmic "
                    "10*B*H*N^2*d/2 as the single-pass backward (it executes 14 instead of 10)"}

    # the other workloads, forward alone, each timed the same way
    if not args.skip_extras:
        for key, name in (("forward_target", FWD_TARGET_WORKLOAD), ("short_seq_forward", "fwd_b4h16n1024d64"),
                          ("long_context_forward", "fwd_b1h8n32768d128_causal_x4")):
            ew = WORKLOADS[name]
            ep = Problem(ew, dev, rank, lib, stream)
            t0 = time.time()
            ms = max_over_ranks(time_forward(ep, flush, n, args.warmup, fa), world)
            ff = algorithmic_flops(ew, backward=False)[0]
            tf = ff / (ms * 1e-3) / 1e12
            rec = {"workload": name, "ms": ms, "tflops": tf, "frac_of_peak": tf / peaks["bf16_tflops"],
                   "roofline": {"bound": "tensor", "kernel": f"fwd::fwd_kernel<{ew.d}>", "achieved": tf,
                                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": tf / peaks["bf16_tflops"],
                                "traffic": profiled_traffic(f"fwd::fwd_kernel<{ew.d}>", name)}}
            if key == "short_seq_forward":
                hbm = (4 * ew.N * ew.d * 2 + 4 * ew.N) * ew.B * ew.H  # Q, K, V in; O, LSE out
                rec["hbm_gbs_algorithmic"] = hbm / (ms * 1e-3) / 1e9
                rec["hbm_frac"] = rec["hbm_gbs_algorithmic"] / peaks["hbm_gbs"]
            extras[key] = rec
            del ep
        t_extras_end = time.time()
    else:
        t_extras_end = t_timed_end

    # End to end through the public Python API: every step copies its inputs in
    # from pinned host memory, runs the forward (and backward) and copies every
    # result back to pinned host memory.  Steps are pipelined as an input
    # pipeline would run them: two sets of device buffers, uploads on one
    # stream, the kernels on another and downloads on a third, so step s+1's
    # uploads overlap step s's downloads (PCIe carries both directions at once).
    hq, hk, hv = (t.pin_memory() for t in prob.host[:3])
    hdo = prob.host[3].pin_memory() if w.backward else None
    hins = [hq, hk, hv] + ([hdo] if w.backward else [])

    def dev_set():
        ins = [torch.empty_like(prob.q), torch.empty_like(prob.k), torch.empty_like(prob.v)]
        if w.backward:
            ins.append(torch.empty_like(prob.do))
        outs_ = [torch.empty_like(prob.o), torch.empty_like(prob.lse)]
        if w.backward:
            outs_ += [torch.empty_like(prob.dq), torch.empty_like(prob.dk), torch.empty_like(prob.dv)]
        return ins, outs_

    sets = [dev_set(), dev_set()]
    houts = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in sets[0][1]]
    h2d = sum(t.numel() * t.element_size() for t in hins)
    d2h = sum(t.numel() * t.element_size() for t in houts)
    s_up, s_run, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in_ready", "in_free", "out_ready", "out_free")}
    used = [False, False]

    def e2e_step(s_idx):
        b = s_idx % 2
        ins, outs_ = sets[b]
        with torch.cuda.stream(s_up):
            if used[b]:
                s_up.wait_event(ev["in_free"][b])  # the kernels of step s-2 are done with these inputs
            for dst, src in zip(ins, hins):
                dst.copy_(src, non_blocking=True)
            ev["in_ready"][b].record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev["in_ready"][b])
            if used[b]:
                s_run.wait_event(ev["out_free"][b])  # step s-2's results have been copied out
            q_, k_, v_ = ins[:3]
            fa.forward(q_, k_, v_, causal=w.causal, scale=w.scale, out=outs_[0], lse=outs_[1])
            if w.backward:
                fa.backward(q_, k_, v_, outs_[0], ins[3], outs_[1], causal=w.causal, scale=w.scale,
                            dq=outs_[2], dk=outs_[3], dv=outs_[4], workspace=prob.ws)
            ev["in_free"][b].record(s_run)
            ev["out_ready"][b].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["out_ready"][b])
            for h, d_ in zip(houts, outs_):
                h.copy_(d_, non_blocking=True)
            ev["out_free"][b].record(s_down)
        used[b] = True

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the timed region: from before the first upload to after the last download
    e0.record(s_up)
    s_run.wait_event(e0)
    s_down.wait_event(e0)
    for i in range(n):
        e2e_step(i)
    e1.record(s_down)
    torch.cuda.synchronize()
    # every step had the same inputs: the last step's downloaded results must be
    # those of the kernel-only runs (dQ, summed by reduce-adds in a varying
    # order, to fp32 rounding), or the pipeline's ordering is wrong
    ref_outs = [prob.o, prob.lse] + ([prob.dq, prob.dk, prob.dv] if w.backward else [])
    for name, h, d_ in zip(("O", "LSE", "dQ", "dK", "dV"), houts, ref_outs):
        ref_h = d_.cpu()
        if name == "dQ":
            rel = float((h.float() - ref_h.float()).norm() / ref_h.float().norm().clamp_min(1e-30))
            ok_e2e = rel < 1e-3
        else:
            ok_e2e = torch.equal(h, ref_h)
        if not ok_e2e:
            raise RuntimeError(f"end-to-end {name} differs from the kernel-only result")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    barrier(world)
    fa.check_device_status()
    clocks.stop()
    clk = clocks.summary(t_soak, t_extras_end,
                         f"{args.soak_s:.1f} s soak of the step right before the timed steps, the timed "
                         "steps, and the forward-only workloads after them")

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
                              "L2-resident)" if args.keep_l2 else "flushed between timed steps (256 MB write)"),
                       "calls": "C ABI: fa_forward, then fa_backward_stages for the preprocess, main and dQ "
                                "convert stages (fa_backward runs the same three launches in one call)"},
            "breakdown_ms": breakdown,
            "frac_of_peak": value / world / peaks["bf16_tflops"],
            "roofline": roof,
            **extras,
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
    ap.add_argument("--skip-extras", action="store_true",
                    help="skip the forward-only timings of the other workloads")
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="seconds of untimed steps right before the timed ones (clock sampling)")
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
