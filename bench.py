"""Benchmark of the MX block-scaled GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the hot path over one batch of pre-quantised inputs:
the scale repack and the block-scaled GEMM (``mxgemm_run``: two kernel
launches).  Quantisation is input generation and stays outside the timed
region, as in the pages' methodology (devotd.net section 2: measurements
start from already-quantised inputs).

Timing: W eager warm-up steps, then the K timed steps are replayed from one
CUDA graph bracketed by a barrier + synchronize and CUDA events on the launch
stream.  Inputs rotate over enough copies that the bytes touched between two
uses of a copy exceed twice the L2 size, so every step streams from HBM.
Multi-GPU runs are replicas (the workload does not shard): every rank runs
the full workload, time is the max over ranks and ``value`` the total work of
all ranks divided by it.

The ``reference`` arm times the CPU oracle (test infrastructure) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MX scaled-GEMM TFLOPS (MXFP8/MXFP4, NT) and % of roofline on 1 B200"
DEFAULT_WORKLOAD = "mxfp8_8192x8192x8192"
_CSRC = "microscaling_block_scaled_b200/csrc/"
# the sources each GEMM kernel is compiled from, and the planner that picks
# its tiles and their order (a recorded DRAM traffic figure is valid only
# for the source it was captured on)
KERNEL_SOURCES = {
    "one_cta": [_CSRC + f for f in ("gemm_kernel.cuh", "gemm_common.cuh", "sm100_ptx.cuh", "mx_convert.cuh",
                                    "gemm.cu")],
    "pair": [_CSRC + f for f in ("gemm_pair_kernel.cuh", "gemm_common.cuh", "sm100_ptx.cuh", "mx_convert.cuh",
                                 "gemm.cu")],
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    ap.add_argument("--reps", type=int, default=20, help="extra replays of the step graph for the spread")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--schedule", default="auto",
                    help="planner override: auto, dp, splitk:S (S K ranges per tile), streamk:W (W workers) "
                         "or ksplit:2|4 (each tile's K range over a cluster of 2 or 4 CTAs)")
    ap.add_argument("--kchunks", type=int, default=0, choices=[0, 1, 2, 4],
                    help="128-byte K chunks per ring stage (0: the planner's choice)")
    return ap.parse_args()


def parse_schedule(text):
    """(schedule, splits, workers) for mxgemm_set_schedule from --schedule."""
    from microscaling_block_scaled_b200 import mxgemm
    kind, _, arg = text.partition(":")
    if kind == "auto" and not arg:
        return mxgemm.SCHED_AUTO, 1, 0
    if kind == "dp" and not arg:
        return mxgemm.SCHED_DP, 1, 0
    if kind == "splitk" and arg.isdigit() and int(arg) >= 1:
        return mxgemm.SCHED_SPLITK, int(arg), 0
    if kind == "streamk" and arg.isdigit() and int(arg) >= 1:
        return mxgemm.SCHED_STREAMK, 1, int(arg)
    if kind == "ksplit" and arg in ("2", "4"):
        return mxgemm.SCHED_KSPLIT, int(arg), 0
    raise SystemExit("--schedule: auto, dp, splitk:S, streamk:W or ksplit:2|4, not %r" % text)


def override_label(args):
    """'' for the planner's own choice, else the override as a suffix."""
    parts = []
    if args.schedule != "auto":
        parts.append(args.schedule.replace(":", ""))
    if args.kchunks:
        parts.append("kc%d" % args.kchunks)
    return "_".join(parts)


def traffic_key(args):
    """Key of the workload's recorded DRAM traffic: plans chosen by an
    override are recorded under '<workload>@<override>'."""
    label = override_label(args)
    return args.workload + ("@" + label if label else "")


def override_config(args):
    """Config keys naming a planner override (none without one)."""
    return {"planner_override": override_label(args)} if override_label(args) else {}


def apply_overrides(h, args):
    h.set_schedule(*parse_schedule(args.schedule))
    h.set_kchunks(args.kchunks)


def workload(name):
    from microscaling_block_scaled_b200 import synth
    if name not in synth.WORKLOADS:
        raise SystemExit("unknown workload %s; one of %s" % (name, sorted(synth.WORKLOADS) +
                                                             sorted(synth.EXTRA_WORKLOADS)))
    fmt_name, M, N, K, seed, kind = synth.WORKLOADS[name]
    return fmt_name, M, N, K, seed, kind


def extra_workload(name):
    """The extension workloads (dense BF16, grouped, fused epilogue,
    quantised output): their description dict, or None."""
    from microscaling_block_scaled_b200 import synth
    w = synth.EXTRA_WORKLOADS.get(name)
    if w is None:
        return None
    w = dict(w)
    if w["op"] == "grouped":
        w["M"] = int(sum(w["groups"]))
    return w


def base_config(name):
    """The workload description both arms print, word for word."""
    w = extra_workload(name)
    if w is not None:
        cfg = {"workload": name, "op": w["op"], "fmt": w["fmt"], "M": w["M"], "N": w["N"], "K": w["K"],
               "seed": w["seed"], "inputs": "normal FP32 (torch generator, seed %d), %s, untimed" % (
                   w["seed"], "rounded to BF16" if w["fmt"] == "bf16" else "OCP MX quantised")}
        for k in ("groups", "act", "out_fmt"):
            if k in w:
                cfg[k] = list(w[k]) if k == "groups" else w[k]
        return cfg
    fmt_name, M, N, K, seed, kind = workload(name)
    return {"workload": name, "fmt": fmt_name, "M": M, "N": N, "K": K, "seed": seed,
            "inputs": "%s FP32 (torch generator, seed %d), OCP MX quantised, untimed" % (kind, seed)}


def extra_bytes_flops(w):
    """Algorithmic bytes (every input read once, every output written once)
    and flops of one extension step."""
    M, N, K = w["M"], w["N"], w["K"]
    fl = 2.0 * M * N * K
    if w["op"] == "bf16":
        return 2 * M * K + 2 * N * K + 2 * M * N, fl
    fmt = 0 if w["fmt"] == "mxfp8" else 1
    rb = K if fmt == 0 else K // 2
    if w["op"] == "grouped":
        live = sum(1 for g in w["groups"] if g > 0)
        return M * (rb + K // 32) + live * N * (rb + K // 32) + 2 * M * N, fl
    base = M * (rb + K // 32) + N * (rb + K // 32)
    if w["op"] == "fused":
        return base + 2 * N + 2 * M * N + 2 * M * N, fl        # bias, residual read, C written
    orb = N if w["out_fmt"] == 0 else N // 2
    return base + M * (orb + N // 32), fl                      # codes + scales written


def flops(M, N, K):
    return 2.0 * M * N * K


def algorithmic_bytes(fmt, M, N, K):
    """A + B + both scale arrays read once, C written once (BF16)."""
    rb = K if fmt == 0 else K // 2
    return M * rb + N * rb + (M + N) * (K // 32) + 2 * M * N


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_hash(kind):
    """Hash of the sources of one GEMM kernel ("one_cta" or "pair")."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name, kind):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on the current source of that kernel."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload_name)
    if not e or e.get("kernel_hash") != kernel_hash(kind):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.002):
        self.samples = []
        self.period = period
        self.active = False
        self._stop = False
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            # NVML and CUDA may enumerate GPUs differently: find the CUDA
            # device's NVML handle by PCI address, else fall back to the index
            try:
                import torch
                pr = torch.cuda.get_device_properties(index)
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self.t = threading.Thread(target=self._loop, daemon=True)

    def sample_now(self):
        """One sample from the calling thread (the bench takes one while the
        timed graph is executing, after its end event has been queued)."""
        if not self.ok:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.samples.append((mhz, rs))
        except Exception:
            pass

    def _loop(self):
        # the first sample waits one period, so the thread does not compete
        # with the launch of the timed region for the interpreter
        while not self._stop:
            time.sleep(self.period)
            if self.active and not self._stop:
                self.sample_now()

    def __enter__(self):
        self.t.start()
        return self

    def __exit__(self, *a):
        self._stop = True
        self.t.join(timeout=1)

    def summary(self):
        if not self.samples:     # no sample was taken in the region: one now
            self.sample_now()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, rs in self.samples:
            for k, bit in self.REASONS.items():
                if rs & bit and k != "gpu_idle":
                    reasons.add(k)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU arm

class OracleSampler:
    """Times the CPU oracle (as it stands) on a bounded sample of C: a block of
    sampled rows of A against a block of sampled rows of B, sized so one call
    takes about ``target_s`` seconds.  The sampled operand rows are quantised by
    the oracle's own quantiser once, outside the timing."""

    def __init__(self, fmt, M, N, K, A32, B32, seed=99):
        import numpy as np
        import torch

        import oracle
        self.oracle = oracle
        self.fmt, self.M, self.N, self.K = fmt, M, N, K
        rng = np.random.default_rng(seed)
        self.nm = min(M, 32, A32.shape[0])
        rm = np.sort(rng.choice(A32.shape[0], self.nm, replace=False))
        a = A32[torch.from_numpy(rm).to(A32.device)].float().cpu().numpy()
        self.pool = min(N, 4096, B32.shape[0])
        rn = np.sort(rng.choice(B32.shape[0], self.pool, replace=False))
        b = B32[torch.from_numpy(rn).to(B32.device)].float().cpu().numpy()
        if fmt == 2:                       # dense BF16 operands
            import ml_dtypes
            self.oa = a.astype(ml_dtypes.bfloat16).view(np.uint16)
            self.ob = b.astype(ml_dtypes.bfloat16).view(np.uint16)
            self.osa = self.osb = None
        else:
            self.oa, self.osa = oracle.quantize(fmt, a)
            self.ob, self.osb = oracle.quantize(fmt, b)
        t0 = time.perf_counter()
        nn0 = min(self.pool, 32)
        self._product(nn0)
        self.sec_per_col = max(time.perf_counter() - t0, 1e-5) / nn0

    def _product(self, nn):
        if self.fmt == 2:
            return self.oracle.gemm_bf16(self.oa, self.ob[:nn])
        return self.oracle.gemm(self.fmt, self.K, self.oa, self.osa, self.ob[:nn], self.osb[:nn])

    def run(self, target_s):
        """One timed sample: the sampled rows against as many sampled columns as
        fit ``target_s``; when the whole column pool takes less than that, the
        same product is recomputed until the time is spent."""
        nn = int(min(self.pool, max(8, target_s / self.sec_per_col)))
        reps = 0
        t0 = time.perf_counter()
        while True:
            self._product(nn)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= 0.9 * target_s or nn < self.pool:
                break
        tflops = reps * flops(self.nm, nn, self.K) / dt / 1e12
        desc = "C[%d sampled rows][%d sampled cols] of the %dx%dx%d product, computed %d time(s) (%.3g GFLOP)" % (
            self.nm, nn, self.M, self.N, self.K, reps, reps * flops(self.nm, nn, self.K) / 1e9)
        return tflops, dt, self.oracle.num_threads(), desc


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from microscaling_block_scaled_b200 import synth
    w = extra_workload(args.workload)
    if w is not None:
        # extension workloads: the oracle's product underneath the op, sampled
        fmt_name, M, N, K, seed, kind = w["fmt"], w["M"], w["N"], w["K"], w["seed"], "normal"
    else:
        fmt_name, M, N, K, seed, kind = workload(args.workload)
    fmt = 0 if fmt_name == "mxfp8" else (1 if fmt_name == "mxfp4" else 2)
    # the whole run stays within a few minutes: split the budget over the steps
    per_step = max(0.05, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    A32, B32 = synth.operands(min(M, 64), min(N, 4096), K, seed=seed, kind=kind, device="cpu")
    sampler = OracleSampler(fmt, M, N, K, A32, B32)
    times, vals = [], []
    desc = cores = None
    for i in range(args.warmup + args.steps):
        v, dt, cores, desc = sampler.run(per_step)
        if i >= args.warmup:
            times.append(dt)
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": fmt_name,
        "data": "synthetic",
        "config": base_config(args.workload),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def max_over_ranks(values, device=None):
    """Elementwise maximum of `values` over the ranks of the default process
    group (the values themselves without one): the job's time is its slowest
    rank's.  NCCL reduces device tensors, gloo host tensors."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tflops(fmt_flops, world, steps, ms):
    """Whole-job throughput: every rank runs `steps` replicas of the GEMM in
    the slowest rank's `ms` milliseconds."""
    return fmt_flops * world * steps / (ms * 1e-3) / 1e12


def run_extra(args, w):
    """Times one extension op (see extra_workload) as the step: CUDA graph of
    K steps on rotating inputs, CUDA events on the launch stream; e2e with the
    inputs copied from pinned host memory and the output copied back in every
    step."""
    import torch
    import torch.distributed as dist

    from microscaling_block_scaled_b200 import mxgemm, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    op, M, N, K = w["op"], w["M"], w["N"], w["K"]
    fmt = mxgemm.FMT_NAMES[w["fmt"]]
    Bn = N * len(w["groups"]) if op == "grouped" else N
    A32, B32 = synth.operands(M, Bn, K, seed=w["seed"], device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w["seed"] + 1000)
    if op == "bf16":
        ins = [A32.to(torch.bfloat16), B32.to(torch.bfloat16)]
    else:
        qa, sa = mxgemm.quantize(fmt, A32)
        qb, sb = mxgemm.quantize(fmt, B32)
        ins = [qa, sa, qb, sb]
    extra = []
    if op == "fused":
        extra = [torch.randn(N, generator=gen, device=dev).to(torch.bfloat16),
                 torch.randn(M, N, generator=gen, device=dev).to(torch.bfloat16)]
    if op == "grouped":
        offs = torch.tensor([0] + list(itertools.accumulate(w["groups"])), dtype=torch.int64, device=dev)
    del A32, B32
    abytes, fl = extra_bytes_flops(w)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nsets = max(2, math.ceil(2 * l2 / abytes) + 1)

    def outputs():
        if op == "quantized":
            return [torch.empty((M, mxgemm.row_bytes(w["out_fmt"], N)), dtype=torch.uint8, device=dev),
                    torch.empty((M, N // 32), dtype=torch.uint8, device=dev)]
        return [torch.empty((M, N), dtype=torch.bfloat16, device=dev)]

    sets = [([t.clone() for t in ins], [t.clone() for t in extra], outputs()) for _ in range(nsets)]
    h = mxgemm.Handle()
    h.set_prefetch_b(True)
    apply_overrides(h, args)

    def call(i_set, stream):
        x, e, o = sets[i_set % nsets]
        if op == "bf16":
            h.run_bf16(x[0], x[1], C=o[0], stream=stream)
        elif op == "grouped":
            h.run_grouped(fmt, offs, x[0], x[1], x[2].view(len(w["groups"]), N, -1), x[3], C=o[0], K=K,
                          stream=stream)
        elif op == "fused":
            h.run_fused(fmt, x[0], x[1], x[2], x[3], bias=e[0], act=w["act"], residual=e[1], C=o[0], K=K,
                        stream=stream)
        else:
            h.run_quantized(fmt, x[0], x[1], x[2], x[3], w["out_fmt"], out=(o[0], o[1]), K=K, stream=stream)

    for i in range(args.warmup):
        call(i, None)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(0, s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for i in range(args.steps):
            call(i, s)
    g.replay()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        clk.active = True
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        g.replay()
        e1.record(st)
        clk.sample_now()
        torch.cuda.synchronize()
        clk.active = False
        ms = e0.elapsed_time(e1)
    clocks = clk.summary()
    del g
    ms = max_over_ranks([ms], dev)[0]
    us = ms / args.steps * 1e3
    peaks, peak_src = measured_peaks()
    tc_peak = peaks["bf16_tflops"] * (1.0 if op == "bf16" else (2.0 if fmt == 0 else 4.0))
    hbm = peaks["hbm_gbs"]
    t_tc, t_hbm = fl / (tc_peak * 1e12), abytes / (hbm * 1e9)
    if t_hbm >= t_tc:
        ach = abytes / (us * 1e-6) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm}
    else:
        ach = fl / (us * 1e-6) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s", "frac": ach / tc_peak}
    roof.update({"traffic": recorded_traffic(traffic_key(args), "one_cta"), "peak_source": peak_src,
                 "kernel": "mx_gemm_kernel (one-CTA)", "algorithmic_bytes": abytes, "flops": fl})
    # end to end: inputs H2D from pinned memory, the op, output D2H, every step
    hx = [t.cpu().pin_memory() for t in sets[0][0] + sets[0][1]]
    ho = [t.cpu().pin_memory() for t in sets[0][2]]
    dx = sets[0][0] + sets[0][1]
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    st = torch.cuda.current_stream()
    e0.record(st)
    for _ in range(args.e2e_steps):
        for d, hsrc in zip(dx, hx):
            d.copy_(hsrc, non_blocking=True)
        call(0, None)
        for hdst, d in zip(ho, sets[0][2]):
            hdst.copy_(d, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    st_err, code = h.check_device_error()
    if st_err != mxgemm.OK:
        raise SystemExit("device error word set: %d" % code)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if rank == 0:
        line = {
            "metric": METRIC, "value": job_tflops(fl, world, args.steps, ms), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w["fmt"], "data": "synthetic",
            "config": dict(base_config(args.workload), **override_config(args), **{
                "l2": "inputs rotate over %d copies (%.1f MB each)" % (nsets, abytes / 1e6),
                "timing": "CUDA graph of K steps, CUDA events on the launch stream", "step_us": us,
                "plan": (mxgemm.mxgemm_describe_grouped_plan(sms, fmt, len(w["groups"]), M, N, K) if op == "grouped"
                         else h.describe(mxgemm.FMT_BF16, M, N, K) if op == "bf16"
                         else h.describe(fmt, M, N, K))}),
            "clocks": clocks, "roofline": roof, "cpu_baseline": None,
            "e2e": {"value": job_tflops(fl, world, args.e2e_steps, e2e_ms), "unit": "TFLOPS",
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hx),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in ho),
                    "api": "torch copies from pinned host memory around the entry point", "steps": args.e2e_steps},
            "gpu_launches": args.steps,
        }
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    from microscaling_block_scaled_b200 import mxgemm, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    fmt_name, M, N, K, seed, kind = workload(args.workload)
    fmt = mxgemm.FMT_NAMES[fmt_name]
    A32, B32 = synth.operands(M, N, K, seed=seed, kind=kind, device=dev)
    qa, sa = mxgemm.quantize(fmt, A32)
    qb, sb = mxgemm.quantize(fmt, B32)
    torch.cuda.synchronize()

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = algorithmic_bytes(fmt, M, N, K)
    nsets = max(2, math.ceil(2 * l2 / set_bytes) + 1)
    sets = [(qa.clone(), sa.clone(), qb.clone(), sb.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev))
            for _ in range(nsets)]
    h = mxgemm.Handle()
    # B (the weights) is never written by the step before: consecutive steps
    # may overlap B's stream with the previous GEMM's tail
    h.set_prefetch_b(True)
    apply_overrides(h, args)
    plan = h.describe(fmt, M, N, K)

    def step(i, stream=None):
        a, s_a, b, s_b, c = sets[i % nsets]
        h.run(fmt, a, s_a, b, s_b, C=c, K=K, stream=stream)

    def gemm_only(i, stream=None):
        a, _, b, _, c = sets[i % nsets]
        h.gemm(fmt, M, N, K, a, b, c, stream=stream)

    def repack_only(i, stream=None):
        _, s_a, _, s_b, _ = sets[i % nsets]
        h.repack(fmt, M, N, K, s_a, s_b, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn(0, s)                     # one eager call on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for i in range(n):
                fn(i, s)
        torch.cuda.synchronize()
        return g, s

    def timed(g, s, probe=None):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        launch = torch.cuda.current_stream()      # replay() launches on the current stream
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(launch)
        g.replay()
        e1.record(launch)
        if probe is not None:                     # the GPU is still running the graph
            probe()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return e0.elapsed_time(e1)

    g_step, s_step = capture(step, args.steps)
    with ClockSampler(local) as clk:     # NVML set up before the GPU's last untimed work
        g_step.replay()                  # untimed replay (graph upload)
        torch.cuda.synchronize()
        clk.active = True
        ms = timed(g_step, s_step, probe=clk.sample_now)
        clk.active = False
    clocks = clk.summary()
    # spread: the same graph replayed again (not part of `value`)
    reps = [timed(g_step, s_step) / args.steps * 1e3 for _ in range(args.reps)]
    # the GEMM-only graph reads the repacked-scale workspace (mxgemm_run on a
    # one-CTA plan converts the scales inside the GEMM and leaves none)
    h.repack(fmt, M, N, K, sets[0][1], sets[0][3])
    torch.cuda.synchronize()
    g_gemm, s_gemm = capture(gemm_only, args.steps)
    g_gemm.replay()
    with ClockSampler(local) as clk_k:
        clk_k.active = True
        ms_gemm = timed(g_gemm, s_gemm, probe=clk_k.sample_now)
        clk_k.active = False
    clocks_kernel = clk_k.summary()
    g_rep, s_rep = capture(repack_only, args.steps)
    g_rep.replay()
    ms_rep = timed(g_rep, s_rep)
    # the input generator (OCP MX quantiser) on the activation operand A,
    # timed as an op of its own: it is not part of the step
    q_out = (torch.empty_like(qa), torch.empty_like(sa))

    def quantize_only(i, stream=None):
        mxgemm.quantize(fmt, A32, stream=stream, out=q_out)

    g_q, s_q = capture(quantize_only, args.steps)
    g_q.replay()
    ms_q = timed(g_q, s_q)
    del g_q
    # the activation quantiser proper: the same A as BF16 (a layer's output)
    A16 = A32.to(torch.bfloat16)

    def quantize_bf16_only(i, stream=None):
        mxgemm.quantize_bf16(fmt, A16, stream=stream, out=q_out)

    g_q16, s_q16 = capture(quantize_bf16_only, args.steps)
    g_q16.replay()
    ms_q16 = timed(g_q16, s_q16)
    del g_q16, A16
    # graphs go before the process group
    del g_step, g_gemm, g_rep
    torch.cuda.synchronize()

    ms, ms_gemm, ms_rep, ms_q, ms_q16 = max_over_ranks([ms, ms_gemm, ms_rep, ms_q, ms_q16], dev)
    quant_us = ms_q / args.steps * 1e3
    quant_bytes = M * K * 4 + qa.numel() + sa.numel()
    quant16_us = ms_q16 / args.steps * 1e3
    quant16_bytes = M * K * 2 + qa.numel() + sa.numel()

    ms_per_step = ms / args.steps
    value = job_tflops(flops(M, N, K), world, args.steps, ms)
    gemm_us = ms_gemm / args.steps * 1e3
    # mxgemm_run on a one-CTA plan is one kernel (scale conversion fused into
    # the GEMM's scale producers): the step's kernel time is the step time.
    # CTA-pair plans run the repack and then the GEMM: their kernel is the GEMM.
    fused = "scales=fused" in plan
    kernel_us = ms / args.steps * 1e3 if fused else gemm_us
    rep_us = ms_rep / args.steps * 1e3

    # roofline of the dominant kernel (the GEMM)
    peaks, peak_src = measured_peaks()
    tc_peak = peaks["bf16_tflops"] * (2.0 if fmt == 0 else 4.0)      # dense MXFP8 = 2x, MXFP4 = 4x bf16
    hbm = peaks["hbm_gbs"]
    t_tc = flops(M, N, K) / (tc_peak * 1e12)
    t_hbm = algorithmic_bytes(fmt, M, N, K) / (hbm * 1e9)
    if t_hbm >= t_tc:
        achieved = algorithmic_bytes(fmt, M, N, K) / (kernel_us * 1e-6) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm}
    else:
        achieved = flops(M, N, K) / (kernel_us * 1e-6) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved / tc_peak}
    tr = recorded_traffic(traffic_key(args), "pair" if "pair=1" in plan else "one_cta")
    roof["traffic"] = tr
    roof["peak_source"] = "%s (%s)" % (peak_src, "hbm_gbs" if roof["bound"] == "hbm" else
                                       "bf16_tflops x %d (nominal MX/bf16 ratio)" % (2 if fmt == 0 else 4))
    if algorithmic_bytes(fmt, M, N, K) < (1 << 20):
        roof["note"] = ("latency-bound: %d bytes per launch take ~%.0f ns at HBM speed, far below a launch; "
                        "the fraction is not meaningful, the us are" % (algorithmic_bytes(fmt, M, N, K),
                                                                        algorithmic_bytes(fmt, M, N, K) / hbm))
    if roof["bound"] == "tensor" and "bf16_tflops_sustained" in peaks:
        # the same against the GPU's sustained (power-capped) bf16 rate, for
        # a kernel that runs back to back for the whole timed region
        sus = peaks["bf16_tflops_sustained"] * (2.0 if fmt == 0 else 4.0)
        roof["frac_of_sustained"] = achieved / sus
        roof["peak_sustained"] = sus
    roof["kernel_clocks"] = clocks_kernel
    roof["kernel"] = ("mx_gemm_kernel (scale conversion fused)" if fused else
                      "mx_gemm_pair_kernel" if "pair=1" in plan else "mx_gemm_kernel")
    roof["algorithmic_bytes"] = algorithmic_bytes(fmt, M, N, K)
    roof["flops"] = flops(M, N, K)

    # end to end through the public host-buffer API
    pa = qa.cpu().pin_memory()
    psa = sa.cpu().pin_memory()
    pb = qb.cpu().pin_memory()
    psb = sb.cpu().pin_memory()
    pc = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    st = torch.cuda.current_stream()
    h.run_host(fmt, M, N, K, pa, psa, pb, psb, pc)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.e2e_steps):
        h.run_host(fmt, M, N, K, pa, psa, pb, psb, pc)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks([e2e_ms], dev)[0]
    e2e_value = job_tflops(flops(M, N, K), world, args.e2e_steps, e2e_ms)
    h2d = pa.numel() + psa.numel() + pb.numel() + psb.numel()
    d2h = pc.numel() * 2

    st_err, code = h.check_device_error()
    if st_err != mxgemm.OK:
        raise SystemExit("device error word set: %d" % code)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, cores, desc = OracleSampler(fmt, M, N, K, A32, B32).run(args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc, "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": fmt_name, "data": "synthetic",
            "config": dict(base_config(args.workload), **override_config(args), **{
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": "inputs rotate over %d copies (%.1f MB each, %.0f MB > 2x L2 %.0f MB)" % (
                           nsets, set_bytes / 1e6, nsets * set_bytes / 1e6, l2 / 1e6),
                       "timing": "CUDA graph of K steps, CUDA events on the launch stream",
                       "chaining": "each step's GEMM is a programmatic dependent of the previous one; "
                                   "B is promised constant (mxgemm_set_prefetch_b), A and C wait for it",
                       "plan": plan, "kernel_us": kernel_us, "gemm_us": gemm_us, "repack_us": rep_us,
                       "quantize_A": {"us": quant_us, "bytes": quant_bytes,
                                      "GB/s": quant_bytes / (quant_us * 1e-6) / 1e9,
                                      "frac_of_hbm": quant_bytes / (quant_us * 1e-6) / 1e9 / hbm},
                       "quantize_A_bf16": {"us": quant16_us, "bytes": quant16_bytes,
                                           "GB/s": quant16_bytes / (quant16_us * 1e-6) / 1e9,
                                           "frac_of_hbm": quant16_bytes / (quant16_us * 1e-6) / 1e9 / hbm},
                       "step_us_spread": {"n": len(reps), "median": statistics.median(reps) if reps else None,
                                          "min": min(reps) if reps else None, "max": max(reps) if reps else None},
                       "step_kernels": "mx_gemm_kernel with fused scale conversion" if fused
                       else "mx_repack_kernel + " + roof["kernel"],
                       "gemm_tflops": flops(M, N, K) / (gemm_us * 1e-6) / 1e12}),
            "clocks": clocks,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "mxgemm_run_host (pinned host buffers)", "steps": args.e2e_steps},
            "gpu_launches": (1 if fused else 2) * args.steps,
        }
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    w = extra_workload(args.workload)
    if w is not None:
        return run_extra(args, w)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
