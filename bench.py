"""Benchmark of the MoDA (mixture-of-depths attention) hot path on B200.

One step is one pass of the whole operator over one batch of seeded synthetic input: the
fused forward (moda_forward) followed by the recompute-based backward (moda_backward),
through the library's C ABI.  The default workload is the long-context problem the
headline metric is quoted on: B=1, T=65536, Hq=16, Hkv=4, d=128, L=32, bf16, inputs
i.i.d. N(0,1).  The FLOP count is the algorithmic one, 4*B*Hq*d*(T^2/2 + T*L) for the
forward and 2.5x that for the backward (five matmul-shaped products instead of two).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl moda|reference]
Under torchrun (N > 1) every rank runs an independent replica of the workload (the
operator needs no exchange between GPUs), and the job value is the sum of the ranks'
FLOPs over the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle (the only reference implementation that
exists for this operator) on bounded samples of the same workload and reports it in the
same metric.  The oracle is imported only by that arm and by the cpu_baseline leg.
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
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "MoDA fwd(+bwd) TFLOP/s, % bf16 peak & HBM GB/s at T=64K; ratio to L=0 causal"
UNIT = "TFLOP/s"
BWD_FLOP_FACTOR = 2.5
PROFILES = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = [os.path.join(ROOT, "depth_aware_attention_b200", "csrc", f)
                  for f in ("moda_fwd.cu", "moda_bwd.cu", "sm100.cuh", "moda_internal.h")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["moda", "reference"], default="moda")
    ap.add_argument("--workload", default="long-64k", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--fwd-only", action="store_true",
                    help="time the forward alone (not the headline step)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--kvwrite", action="store_true",
                    help="time the fused depth-stream write for the workload's tokens")
    ap.add_argument("--decode", action="store_true",
                    help="time single-token decode against a cache of the workload's length")
    ap.add_argument("--decode-batch", type=int, default=8)
    ap.add_argument("--fda", action="store_true",
                    help="time depth-only attention (forward, backward) on --workload")
    ap.add_argument("--sweep", action="store_true",
                    help="forward efficiency sweep over T x L (not the headline step)")
    return ap.parse_args()


def peaks():
    """Measured denominators (generated file), else the machine's fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(bf16=float(p["bf16_tflops"]), bf16_sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


def kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel sources (profiles/traffic.json: {kernel: {workload: {bytes, source_hash}}})."""
    try:
        with open(os.path.join(PROFILES, "traffic.json")) as f:
            rec = json.load(f)[kernel][workload]
    except (OSError, KeyError, ValueError):
        return None
    return float(rec["bytes"]) if rec.get("source_hash") == kernel_hash() else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout=5.0):
        """Block until the first sample arrived, so the timed region is covered."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.05)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local))
    elif n > 1:
        print(json.dumps({"warning": f"--gpus {n} without torchrun: running one replica"}),
              file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank scalar over all ranks (the slowest rank's time sets the job's)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(step_flops_per_rank, world, ms_max):
    """Whole-job throughput in TFLOP/s: every rank runs one replica of the step, so the
    job does world x the step's FLOPs in the slowest rank's time."""
    return step_flops_per_rank * world / (ms_max * 1e-3) / 1e12


def step_flops(cfg, fwd_only):
    f = workloads.forward_flops(**cfg)
    return f if fwd_only else f * (1.0 + BWD_FLOP_FACTOR)


def forward_bytes(cfg):
    """Algorithmic bytes of one forward: every input read once, every output written once."""
    B, Hq, Hkv, T, L, d = (cfg[n] for n in ("B", "Hq", "Hkv", "T", "L", "d"))
    return (2 * B * Hq * T * d * 2              # q read, out written (bf16)
            + 2 * B * Hkv * T * d * 2           # k, v
            + workloads.depth_bytes(**cfg)      # kd, vd
            + B * Hq * T * 4)                   # lse


def kernel_roofline(name, cfg, avg_ms, pk, workload):
    """Roofline entry for one kernel: algorithmic work per launch over its average
    CUDA-event duration, against the measured sustained peak (every kernel here runs
    inside a step of back-to-back launches)."""
    B, Hq, Hkv, T, L, d = (cfg[n] for n in ("B", "Hq", "Hkv", "T", "L", "d"))
    rows = B * Hq * T
    if name == "moda_fwd_kernel":
        # the bound is whichever side takes longer at the measured peaks: the FLOPs at
        # tensor speed, or the algorithmic bytes (inputs read once, outputs written once)
        # at HBM speed -- the depth cache dominates the bytes when L is large
        flops = workloads.forward_flops(**cfg)
        fbytes = forward_bytes(cfg)
        if fbytes / (pk["hbm"] * 1e9) > flops / (pk["bf16_sustained"] * 1e12):
            bound, work = "hbm", fbytes
            what = "bytes: q, k, v, kd, vd read once; out, lse written once"
        else:
            bound, work = "tensor", flops
            what = "4*B*Hq*d*(T^2/2 + T*L) FLOPs"
    elif name in ("moda_bwd_seq_kernel", "moda_bwd_seq_h_kernel"):
        bound, work = "tensor", BWD_FLOP_FACTOR * 4.0 * B * Hq * d * T * T / 2.0
        what = "2.5 x 4*B*Hq*d*T^2/2 FLOPs (sequence part of the backward)"
    elif name == "moda_bwd_depth_kernel":
        bound = "hbm"
        work = (2 * workloads.depth_bytes(**cfg)           # kd, vd read; dkd, dvd written
                + 3 * rows * d * 2 + rows * d * 4 + rows * 8)  # q, dout, out; dq acc; lse, D
        what = "bytes: kd+vd read, dkd+dvd written, q/dout/out read, fp32 dq written, lse/D"
    else:
        bound, work = "hbm", rows * d * (4 + 2)
        what = "bytes: fp32 dq read, bf16 dq written"
    if bound == "tensor":
        achieved, peak, unit = work / (avg_ms * 1e-3) / 1e12, pk["bf16_sustained"], "TFLOP/s"
        peak_kind = f"{pk['source']} bf16 dense, sustained"
    else:
        achieved, peak, unit = work / (avg_ms * 1e-3) / 1e9, pk["hbm"], "GB/s"
        peak_kind = f"{pk['source']} HBM copy bandwidth"
    return {"kernel": name, "bound": bound, "achieved": round(achieved, 1), "peak": peak,
            "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": recorded_traffic(name, workload), "peak_kind": peak_kind,
            "algorithmic_work_per_launch": work, "work_counted": what,
            "avg_launch_ms": round(avg_ms, 4)}


# ----------------------------------------------------------------------------- GPU arm
def run_moda(args, world, rank, local):
    import depth_aware_attention_b200 as moda

    cfg = workloads.CONFIGS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    scale = workloads.default_scale(cfg["d"])
    x = workloads.make_inputs(cfg, workloads.SEED_BASE[args.workload] + 7919 * rank, dev,
                              with_dout=True)
    q, k, v, kd, vd, dout = (x[n] for n in ("q", "k", "v", "kd", "vd", "dout"))
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device=dev, dtype=torch.float32)
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], cfg["L"]
    ws_bytes = moda.moda_backward_workspace_size(B, Hq, Hkv, T, L, d)
    ws = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    grads = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                 dkd=torch.empty_like(kd) if L else None,
                 dvd=torch.empty_like(vd) if L else None)
    stream = torch.cuda.current_stream(dev)
    # Every launch of the step is bracketed by CUDA events on the launching stream: the
    # forward kernel, then the backward's three stages (row terms + depth part, sequence
    # part, dq convert), each launched on its own through moda_backward_stages.
    # the sequence stage runs the half-tile kernel at d = 128, the plain one at d = 64
    seq_kernel = "moda_bwd_seq_h_kernel" if d == 128 else "moda_bwd_seq_kernel"
    names = ["moda_fwd_kernel"] + ([] if args.fwd_only else
                                   ["moda_bwd_depth_kernel", seq_kernel,
                                    "moda_dq_convert_kernel"])
    events = {n: [] for n in names}

    def timed(name, fn, record):
        if not record:
            fn()
            return
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        events[name].append((e0, e1))

    def step(record=False):
        timed("moda_fwd_kernel",
              lambda: moda.forward(q, k, v, kd, vd, scale, True, out=out, lse=lse), record)
        if not args.fwd_only:
            for name, stage in zip(names[1:], (1, 2, 4)):
                timed(name, lambda st=stage: moda.backward(
                    q, k, v, kd, vd, out, lse, dout, scale, True, workspace=ws, grads=grads,
                    stages=st), record)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    moda.check_device_errors()

    barrier(world)
    torch.cuda.synchronize(dev)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        clocks.wait_first()
        t_start.record(stream)
        for _ in range(args.steps):
            step(record=True)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    moda.check_device_errors()
    ms_local = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms_local, world)
    value = job_value(step_flops(cfg, args.fwd_only), world, ms)
    launches_per_step = len(names)
    kernel_ms = {n: statistics.mean(a.elapsed_time(b) for a, b in ev) for n, ev in events.items()}

    pk = peaks()
    fwd_flops = workloads.forward_flops(**cfg)
    dominant = max(kernel_ms, key=kernel_ms.get)
    roofline = kernel_roofline(dominant, cfg, kernel_ms[dominant], pk, args.workload)

    # Extras the metric names: the L=0 causal ratio and the depth stream's HBM rate.
    extras = {}
    if args.workload.startswith("long-64k") and L > 0:
        fwd_ms = interleaved_ms(
            {"L": lambda: moda.forward(q, k, v, kd, vd, scale, True, out=out, lse=lse),
             "L0": lambda: moda.forward(q, k, v, None, None, scale, True, out=out, lse=lse)},
            stream, dev, rounds=7)
        ms_l, ms_0 = fwd_ms["L"], fwd_ms["L0"]
        cfg0 = dict(cfg, L=0)
        tf_l = fwd_flops / (ms_l * 1e-3) / 1e12
        tf_0 = workloads.forward_flops(**cfg0) / (ms_0 * 1e-3) / 1e12
        dbytes = workloads.depth_bytes(**cfg)
        extras["l0_ratio"] = {"fwd_ms_L": round(ms_l, 3), "fwd_ms_L0": round(ms_0, 3),
                              "time_ratio_L0_over_L": round(ms_0 / ms_l, 4),
                              "tflops_ratio_L_over_L0": round(tf_l / tf_0, 4)}
        extra_ms = ms_l - ms_0
        extras["depth_stream"] = {
            "bytes": dbytes,
            "gbs_from_time_difference": (round(dbytes / (extra_ms * 1e-3) / 1e9, 1)
                                         if extra_ms > 0.02 * ms_l else "hidden"),
            "hbm_peak_gbs": pk["hbm"]}
        extras["fwd_pct_bf16_peak"] = {
            "of_measured_burst": round(tf_l / pk["bf16"], 4),
            "of_measured_sustained": round(tf_l / pk["bf16_sustained"], 4),
            "of_spec_2250": round(tf_l / 2250.0, 4)}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, moda, cfg, x, scale, dev, stream, world)

    del x, q, k, v, kd, vd, dout, out, lse, ws, grads
    torch.cuda.empty_cache()
    extras["kernels_ms"] = {n: round(t, 4) for n, t in kernel_ms.items()}
    return dict(ms=ms, value=value, clocks=clocks.summary(), roofline=roofline,
                launches=launches_per_step * args.steps, extras=extras, e2e=e2e)


def run_e2e(args, moda, cfg, x, scale, dev, stream, world):
    """Same metric through the public API from pinned HOST buffers: every step copies its
    inputs host->device, runs the operator and reads every result back to the host.

    The steps are pipelined on three streams with two device buffer sets: while step i
    runs its kernels, step i+1's inputs are uploaded into the other set and step i-1's
    results are read back (the two copy directions use separate copy engines).  A set's
    inputs are overwritten only after the kernels that read them finished, and its
    outputs only after their read-back finished.  The timed region covers K steps
    including the pipeline's fill and drain."""
    names = ["q", "k", "v", "kd", "vd"] + ([] if args.fwd_only else ["dout"])
    host = {n: torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=True)
            for n in names if x[n] is not None}
    for n, h in host.items():
        h.copy_(x[n])
    h2d = sum(h.numel() * h.element_size() for h in host.values())
    B, Hq, T, d = x["q"].shape
    Hkv, L = x["k"].shape[1], cfg["L"]
    res_names = ["out", "lse"] + ([] if args.fwd_only else
                                  ["dq", "dk", "dv"] + (["dkd", "dvd"] if L else []))
    like = dict(out=x["q"], dq=x["q"], dk=x["k"], dv=x["v"], dkd=x["kd"], dvd=x["vd"])
    res_h = {}
    for n in res_names:
        if n == "lse":
            res_h[n] = torch.empty((B, Hq, T), dtype=torch.float32, pin_memory=True)
        else:
            res_h[n] = torch.empty(like[n].shape, dtype=torch.bfloat16, pin_memory=True)
    d2h = sum(r.numel() * r.element_size() for r in res_h.values())
    sets = []
    for _ in range(2):
        ins = {n: torch.empty_like(x[n]) for n in host}
        outs = {n: torch.empty(r.shape, dtype=r.dtype, device=dev) for n, r in res_h.items()}
        sets.append((ins, outs))
    ws = None if args.fwd_only else torch.empty(
        moda.moda_backward_workspace_size(B, Hq, Hkv, T, L, d), device=dev, dtype=torch.uint8)
    s_up, s_run, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    ran = [torch.cuda.Event() for _ in range(2)]   # kernels that read set i finished
    read = [torch.cuda.Event() for _ in range(2)]  # set i's results are on the host
    for e in ran + read:
        e.record(stream)

    def step(i):
        ins, outs = sets[i % 2]
        up = torch.cuda.Event()
        with torch.cuda.stream(s_up):
            s_up.wait_event(ran[i % 2])
            for n, h in host.items():
                ins[n].copy_(h, non_blocking=True)
            up.record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(up)
            s_run.wait_event(read[i % 2])
            moda.forward(ins["q"], ins["k"], ins["v"], ins.get("kd"), ins.get("vd"), scale,
                         True, out=outs["out"], lse=outs["lse"])
            if not args.fwd_only:
                grads = {n: outs.get(n) for n in ("dq", "dk", "dv", "dkd", "dvd")}
                moda.backward(ins["q"], ins["k"], ins["v"], ins.get("kd"), ins.get("vd"),
                              outs["out"], outs["lse"], ins["dout"], scale, True,
                              workspace=ws, grads=grads)
            ran[i % 2].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ran[i % 2])
            for n, r in res_h.items():
                r.copy_(outs[n], non_blocking=True)
            read[i % 2].record(s_down)

    def run(k):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (s_up, s_run, s_down):
            st.wait_event(e0)
        for i in range(k):
            step(i)
        for st in (s_up, s_run, s_down):
            stream.wait_stream(st)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    run(2)  # warm-up: both buffer sets once
    barrier(world)
    steps = max(1, args.steps)
    ms = max_over_ranks(run(steps) / steps, world)
    value = job_value(step_flops(cfg, args.fwd_only), world, ms)
    del host, sets, res_h, ws
    return {"value": round(value, 2), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipeline": "three streams (upload, kernels, read-back), two device buffer sets"}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(cfg, seed_base, cpu_seconds, fwd_only):
    """Times the fp64 CPU oracle on a bounded sample of the workload.

    The sample is a window of the LAST nt query tokens (the most expensive rows of the
    causal problem) with all heads; its algorithmic FLOPs are summed row by row with the
    same per-row count as the full problem (4*d*(|visible keys| + L) forward, x2.5 for the
    backward).  nt grows until the sample takes about cpu_seconds.  ``cores`` is the number
    of threads the oracle actually ran: its forward splits rows, its backward the window's
    tokens, over the host's threads.  A second, smaller sample on one thread gives
    ``value_1_thread``.
    """
    import oracle
    g = torch.Generator().manual_seed(seed_base)
    B, Hq, Hkv, T, L, d = (cfg[n] for n in ("B", "Hq", "Hkv", "T", "L", "d"))
    scale = workloads.default_scale(d)
    k = torch.randn((B, Hkv, T, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, T, d), generator=g).to(torch.bfloat16)
    threads = oracle.default_threads()

    def sample(nt, nthreads=threads):
        t0 = T - nt
        q = torch.randn((B, Hq, nt, d), generator=g).to(torch.bfloat16)
        kd = vd = None
        if L:
            kd = torch.randn((B, Hkv, nt, L, d), generator=g).to(torch.bfloat16)
            vd = torch.randn((B, Hkv, nt, L, d), generator=g).to(torch.bfloat16)
        rows_keys = sum((t + 1) + L for t in range(t0, T)) * B * Hq
        fl = 4.0 * d * rows_keys
        start = time.perf_counter()
        if fwd_only:
            oracle.forward(q, k, v, kd, vd, scale, True, t0=t0, nthreads=nthreads)
        else:
            dout = torch.randn((B, Hq, nt, d), generator=g).to(torch.bfloat16)
            oracle.backward(q, k, v, kd, vd, dout, scale, True, t0=t0, nthreads=nthreads)
            fl *= 1.0 + BWD_FLOP_FACTOR
        return fl, time.perf_counter() - start

    nt = 1
    fl, sec = sample(nt)
    while sec < cpu_seconds / 8 and nt < T:
        nt = min(T, nt * 4)
        fl, sec = sample(nt)
    if sec < cpu_seconds / 2 and nt < T:
        nt = min(T, max(nt + 1, int(nt * cpu_seconds / max(sec, 1e-3))))
        fl, sec = sample(nt)
    used = min(threads, B * Hq * nt if fwd_only else nt)
    # one thread, on about a quarter of the time budget
    nt1 = max(1, nt // (4 * used))
    fl1, sec1 = sample(nt1, 1)
    what = "forward" if fwd_only else "forward+backward"
    return {"value": round(fl / sec / 1e12, 6), "unit": UNIT, "cores": used, "kind": "oracle",
            "seconds": round(sec, 2), "host_threads": threads, "sample_tokens": nt,
            "value_1_thread": round(fl1 / sec1 / 1e12, 6), "sample_1_thread_tokens": nt1,
            "sample": f"fp64 oracle {what} on the last {nt} query tokens (all {B * Hq} "
                      f"heads) of the {cfg['T']}-token workload, L={L}; FLOPs counted "
                      f"row by row as 4*d*(visible keys + L)"
                      + ("" if fwd_only else " x (1 + 2.5)")}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, timed on bounded samples, in the same metric."""
    cfg = workloads.CONFIGS[args.workload]
    if rank != 0:
        return None
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    oracle_sample(cfg, 1, 0.5, args.fwd_only)  # warm-up: builds and loads the library
    vals = []
    last = None
    for _ in range(args.steps):
        last = oracle_sample(cfg, 1, per_step, args.fwd_only)
        vals.append(last["value"])
    value = statistics.mean(vals)
    flops = step_flops(cfg, args.fwd_only)
    return dict(value=value, ms=flops / (value * 1e12) * 1e3, cpu=dict(last, value=value))


def interleaved_ms(fns, stream, dev, rounds, warmup=2):
    """Median CUDA-event time (ms) of one call of each function in ``fns``, the calls
    interleaved round by round with the starting function rotated each round.  On a
    power-capped GPU the clock drifts over a run, so timing one variant after another
    biases their ratio toward whichever ran first; interleaving cancels that."""
    keys = list(fns)
    for _ in range(warmup):
        for key in keys:
            fns[key]()
    torch.cuda.synchronize(dev)
    ev = {key: [] for key in keys}
    for r in range(rounds):
        for i in range(len(keys)):
            key = keys[(r + i) % len(keys)]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fns[key]()
            e1.record(stream)
            ev[key].append((e0, e1))
    torch.cuda.synchronize(dev)
    return {key: statistics.median(a.elapsed_time(b) for a, b in ev[key]) for key in keys}


def run_sweep(args):
    """Forward time over T in {4K..64K} x L in {0, 8, 32, 128} x group size G in {4, 8}
    (B=1, Hkv=4, Hq=4G, d=128; G=4 is the 1.5B-layer head shape): TFLOP/s and the ratio
    time(L=0)/time(L) per point, the shape of the pages' efficiency-scaling experiment
    (the depth overhead shrinks as T grows).  Prints one JSON line per point, then a
    markdown table."""
    import depth_aware_attention_b200 as moda
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    rows = []
    Ls = (0, 8, 32, 128)
    for G, T in [(g, t) for g in (4, 8) for t in (4096, 8192, 16384, 32768, 65536)]:
        # q, k, v are shared by every L (same seeds); each L gets its own depth cache.
        xs = {L: workloads.make_inputs(dict(B=1, T=T, Hq=4 * G, Hkv=4, d=128, L=L),
                                       900 + T // 4096, dev) for L in Ls}
        x0 = xs[0]
        out = torch.empty_like(x0["q"])
        lse = torch.empty(x0["q"].shape[:3], device=dev, dtype=torch.float32)
        fns = {L: (lambda L=L: moda.forward(x0["q"], x0["k"], x0["v"], xs[L]["kd"],
                                             xs[L]["vd"], None, True, out=out, lse=lse))
               for L in Ls}
        ms = interleaved_ms(fns, stream, dev, rounds=5 if T >= 32768 else 15)
        moda.check_device_errors()
        for L in Ls:
            cfg = dict(B=1, T=T, Hq=4 * G, Hkv=4, d=128, L=L)
            tf = workloads.forward_flops(**cfg) / (ms[L] * 1e-3) / 1e12
            row = {"G": G, "T": T, "L": L, "ms": round(ms[L], 4), "tflops": round(tf, 1),
                   "time_ratio_L0_over_L": round(ms[0] / ms[L], 4),
                   "depth_gbs_from_difference": (round(workloads.depth_bytes(**cfg) /
                                                       ((ms[L] - ms[0]) * 1e-3) / 1e9, 1)
                                                 if L and ms[L] > ms[0] * 1.02 else None)}
            print(json.dumps(row), flush=True)
            rows.append(row)
        del xs, x0, fns, out, lse
        torch.cuda.empty_cache()
    print("| G | T | L | ms | TFLOP/s | time(L=0)/time(L) |")
    print("|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r['G']} | {r['T']} | {r['L']} | {r['ms']:.3f} | {r['tflops']:.0f} | "
              f"{r['time_ratio_L0_over_L']:.3f} |")


def run_fda(args):
    """Depth-only attention (Flash Depth Attention) forward and backward on the workload's
    depth cache: average CUDA-event times and the algorithmic HBM rate of each (forward:
    q, kd, vd read, out and lse written; backward: q, kd, vd, out, dout read, dkd, dvd,
    dq written, fp32 dq accumulator written and read)."""
    import depth_aware_attention_b200 as moda
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    cfg = workloads.CONFIGS[args.workload]
    if cfg["L"] < 1:
        raise SystemExit("depth-only attention needs a workload with L >= 1")
    x = workloads.make_inputs(cfg, workloads.SEED_BASE[args.workload], dev, with_dout=True)
    B, Hq, Hkv, T, L, d = (cfg[n] for n in ("B", "Hq", "Hkv", "T", "L", "d"))
    out = torch.empty_like(x["q"])
    lse = torch.empty((B, Hq, T), device=dev, dtype=torch.float32)
    ws = torch.empty(moda.moda_backward_workspace_size(B, Hq, Hkv, T, L, d), device=dev,
                     dtype=torch.uint8)
    grads = dict(dq=torch.empty_like(x["q"]), dkd=torch.empty_like(x["kd"]),
                 dvd=torch.empty_like(x["vd"]))
    fwd = lambda: moda.depth_attention_forward(x["q"], x["kd"], x["vd"], out=out, lse=lse)
    bwd = lambda: moda.depth_attention_backward(x["q"], x["kd"], x["vd"], out, lse, x["dout"],
                                                workspace=ws, grads=grads)
    res = {}
    for name, f in (("forward", fwd), ("backward", bwd)):
        for _ in range(max(3, args.warmup)):
            f()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = e0.elapsed_time(e1) / args.steps
    moda.check_device_errors()
    rows = B * Hq * T
    dep = workloads.depth_bytes(**cfg)
    fbytes = dep + rows * d * 2 * 2 + rows * 4
    bbytes = 2 * dep + rows * d * 2 * 4 + rows * d * 4 * 2 + rows * 8
    pk = peaks()
    line = {"op": "depth-only attention", "workload": args.workload, "config": cfg,
            "forward_ms": round(res["forward"], 4),
            "forward_gbs": round(fbytes / (res["forward"] * 1e-3) / 1e9, 1),
            "backward_ms": round(res["backward"], 4),
            "backward_gbs": round(bbytes / (res["backward"] * 1e-3) / 1e9, 1),
            "hbm_peak_gbs": pk["hbm"], "steps": args.steps}
    print(json.dumps(line), flush=True)


def run_decode(args):
    """Single-token decode against a K/V cache of the workload's length T (per sequence),
    batch --decode-batch sequences: average CUDA-event time and the algorithmic HBM rate
    (K/V cache and depth entries read once, q read, out and lse written)."""
    import depth_aware_attention_b200 as moda
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    cfg = dict(workloads.CONFIGS[args.workload])
    B, Hq, Hkv, S, L, d = (args.decode_batch, cfg["Hq"], cfg["Hkv"], cfg["T"], cfg["L"],
                           cfg["d"])
    g = torch.Generator(device=dev)
    g.manual_seed(workloads.SEED_BASE[args.workload] * 1000 + 7)
    mk = lambda *sh: torch.randn(*sh, generator=g, device=dev, dtype=torch.bfloat16)
    q, k, v = mk(B, Hq, d), mk(B, Hkv, S, d), mk(B, Hkv, S, d)
    kd = mk(B, Hkv, L, d) if L else None
    vd = mk(B, Hkv, L, d) if L else None
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)
    ws = torch.empty(max(256, moda.moda_decode_workspace_size(B, Hq, Hkv, S, L, d)),
                     device=dev, dtype=torch.uint8)
    f = lambda: moda.decode(q, k, v, kd, vd, out=out, lse=lse, workspace=ws)
    for _ in range(max(3, args.warmup)):
        f()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        f()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    moda.check_device_errors()
    ms = e0.elapsed_time(e1) / args.steps
    nbytes = 2 * B * Hkv * S * d * 2 + 2 * B * Hkv * L * d * 2 + 2 * B * Hq * d * 2 + B * Hq * 4
    pk = peaks()
    print(json.dumps({"op": "decode", "workload": args.workload, "batch": B, "cache_len": S,
                      "Hq": Hq, "Hkv": Hkv, "d": d, "L": L, "ms": round(ms, 4),
                      "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "hbm_peak_gbs": pk["hbm"],
                      "steps": args.steps}), flush=True)


def run_kvwrite(args):
    """Fused depth-stream write for the workload's tokens at the 1.5B-layer projection
    shape (hidden 2048 -> K|V of Hkv x d): CUDA-event time and TFLOP/s of the fused
    kernel, beside torch's matmul followed by the copy into the depth-cache slot (the
    unfused two-step it replaces; cuBLAS, for context)."""
    import depth_aware_attention_b200 as moda
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    cfg = workloads.CONFIGS[args.workload]
    B, T, Hkv, d, L = cfg["B"], cfg["T"], cfg["Hkv"], cfg["d"], max(cfg["L"], 1)
    hidden = 2048
    g = torch.Generator(device=dev)
    g.manual_seed(workloads.SEED_BASE[args.workload] * 1000 + 8)
    x = torch.randn(B, T, hidden, generator=g, device=dev, dtype=torch.bfloat16)
    w = (torch.randn(2 * Hkv * d, hidden, generator=g, device=dev) / 45.25).to(torch.bfloat16)
    kd = torch.zeros(B, Hkv, T, L, d, device=dev, dtype=torch.bfloat16)
    vd = torch.zeros_like(kd)
    slot = L - 1

    def unfused():
        y = torch.matmul(x, w.t()).view(B, T, 2, Hkv, d)
        kd[:, :, :, slot].copy_(y[:, :, 0].transpose(1, 2))
        vd[:, :, :, slot].copy_(y[:, :, 1].transpose(1, 2))

    res = {}
    for name, f in (("fused", lambda: moda.depth_kv_write(x, w, kd, vd, slot)),
                    ("torch_matmul_then_copy", unfused)):
        for _ in range(max(3, args.warmup)):
            f()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = e0.elapsed_time(e1) / args.steps
    moda.check_device_errors()
    flops = 2.0 * B * T * hidden * 2 * Hkv * d
    pk = peaks()
    print(json.dumps({"op": "depth-stream write", "workload": args.workload, "tokens": B * T,
                      "hidden": hidden, "Hkv": Hkv, "d": d, "L": L,
                      "fused_ms": round(res["fused"], 4),
                      "fused_tflops": round(flops / (res["fused"] * 1e-3) / 1e12, 1),
                      "unfused_ms": round(res["torch_matmul_then_copy"], 4),
                      "bf16_peak_tflops": pk["bf16"], "steps": args.steps}), flush=True)


L2_BYTES = 126 * 2**20  # B200 L2 capacity


def l2_note(cfg):
    """Whether one step's tensors (q, k, v, kd, vd, out, dout in bf16; lse in fp32) exceed
    L2, so that back-to-back steps read their inputs from HBM without an L2 flush."""
    shp = workloads.shapes(**{k: cfg[k] for k in ("B", "T", "Hq", "Hkv", "d", "L")})
    n = 2 * sum(math.prod(shp[t]) for t in ("q", "k", "v", "kd", "vd", "dout"))
    n += 2 * math.prod(shp["q"]) + 4 * cfg["B"] * cfg["Hq"] * cfg["T"]
    if n > L2_BYTES:
        return "inputs larger than L2 (no flush)"
    return f"inputs of {n / 2**20:.1f} MiB fit in L2: L2-warm timing, not a headline figure"


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    if args.fda:
        run_fda(args)
        return
    if args.decode:
        run_decode(args)
        return
    if args.kvwrite:
        run_kvwrite(args)
        return
    if args.impl == "reference":
        # The reference arm is the oracle on rank 0's host cores: no device work and no
        # collective, so no process group; the other ranks exit at once.
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank, local = int(os.environ.get("RANK", "0")), 0
    else:
        world, rank, local = dist_setup(args.gpus)
    cfg = workloads.CONFIGS[args.workload]
    config = {"workload": args.workload, **{k: cfg[k] for k in ("B", "T", "Hq", "Hkv", "d", "L")},
              "causal": True, "scale": "1/sqrt(d)",
              "step": "forward" if args.fwd_only else "forward+backward",
              "l2": l2_note(cfg), "parallelism": f"replicas x{world}"}
    base = {"metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic, seeded N(0,1) bf16", "config": config}

    if args.impl == "reference":
        r = run_reference(args, world, rank)
        if rank == 0:
            line = dict(base, impl="reference", value=round(r["value"], 6),
                        ms_per_step=round(r["ms"], 3), dtype="f64",
                        cpu_baseline=r["cpu"],
                        e2e={"value": round(r["value"], 6), "unit": UNIT,
                             "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
            print(json.dumps(line), flush=True)
        return

    r = run_moda(args, world, rank, local)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(cfg, 1, args.cpu_seconds, args.fwd_only)
    if rank == 0:
        line = dict(base, value=round(r["value"], 2), ms_per_step=round(r["ms"], 3),
                    dtype="bf16", clocks=r["clocks"], roofline=r["roofline"],
                    cpu_baseline=cpu, e2e=r["e2e"], gpu_launches=r["launches"], **r["extras"])
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
