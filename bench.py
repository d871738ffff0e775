#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 linear path on B200 (one JSON line).

A step is one pass of the whole path over one batch of synthetic input:
calibration, smoothing factors + fold, weight smoothing + INT8 quantisation
(the offline rows) and fused norm + per-token quantisation, INT8 GEMM with
the dequant epilogue (the runtime rows), for every Linear of the workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle, on a bounded sample

For N > 1 launch under torchrun; every rank runs the workload on its own GPU
with its own token batch (weak scaling, no data-path collective); time is the
max over ranks.  Rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W8A8 linear TOPS & tokens/s (prefill, decode); % of INT8 tensor peak / HBM BW"
DEFAULT_WORKLOAD = "opt-prefill-rmsnorm-qkv-2048x4096x12288"
L2_FLUSH_BYTES = 256 << 20
# nominal dense INT8 : BF16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# helpers shared by both arms
# ---------------------------------------------------------------------------

class L2Flush:
    """Empties L2 of the step's data between timed steps (untimed): writes a
    buffer larger than L2, then reads a second one, so L2 ends up holding clean
    lines only -- otherwise the first kernel of the step would pay for writing
    back up to 126 MB of the flush's own dirty lines."""

    def __init__(self, dev, nbytes: int = None):
        import torch
        n = (nbytes or L2_FLUSH_BYTES) // 4
        self.w = torch.empty(n, dtype=torch.float32, device=dev)
        self.r = torch.zeros(n, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.sink)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_ops(w, M=None) -> int:
    return w.gemm_ops(M)


def gemm_bytes(M, N, K) -> int:
    """Algorithmic bytes of one W8A8 GEMM launch: INT8 operands once, both
    scale vectors, the bf16 output."""
    return M * K + N * K + 4 * M + 4 * N + 2 * M * N


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (a timing reduction only)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(w, seed: int, rank: int):
    """One data-parallel replica's inputs: weights, norm parameters and the
    calibration batch are the same on every rank; the token batch is the
    rank's own (weak scaling: a fixed batch per GPU)."""
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    return S.make_inputs(w, seed=seed, token_seed=seed + 1000003 * rank)


def aggregate(units_per_rank: float, seconds_per_rank: float, world: int, device=None):
    """Whole-job throughput: units all ranks processed over the slowest rank's time."""
    t = max_over_ranks(seconds_per_rank, world, device)
    return units_per_rank * world / t, t


# ---------------------------------------------------------------------------
# the oracle on a bounded sample (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

def _sample_rows(n, k, seed=11):
    if k >= n:
        return np.arange(n)
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False))


def oracle_sample_step(w, inp, cal_rows=512, weight_elems=48 << 20, token_rows=16):
    """One oracle step on a bounded sample: `cal_rows` calibration tokens, up
    to `weight_elems` weight elements per Linear (whole rows) and `token_rows`
    runtime tokens.  Each phase's time is scaled linearly to the full workload.
    Returns (extrapolated seconds for the full step, seconds spent, text)."""
    import oracle
    spent = 0.0
    full = 0.0
    prep = {}

    def wrows(Wl):
        n = max(1, min(Wl.shape[0], weight_elems // Wl.shape[1]))
        return _sample_rows(Wl.shape[0], n)

    for site in w.sites:
        g, b = inp.gamma[site.name], inp.beta[site.name]
        s = None
        gf, bf = g, b
        if site.smoothed:
            xc = inp.x_cal[site.name]
            cr = _sample_rows(xc.shape[0], cal_rows)
            xcs = np.ascontiguousarray(xc[cr])
            Ws, fr = [], []
            for l in w.linears_of(site.name):
                Wl = inp.W[l.name]
                r = wrows(Wl)
                Ws.append(np.ascontiguousarray(Wl[r]))
                fr.append(len(r) / Wl.shape[0])
            t0 = time.perf_counter()
            am = oracle.calibrate_absmax(xcs, site.norm, g, b, w.eps)
            t1 = time.perf_counter()
            s, _ = oracle.smooth_scales(am, Ws, w.alpha, w.clamp_eps)
            gf, bf = oracle.fold_norm(s, g, b)
            t2 = time.perf_counter()
            spent += t2 - t0
            full += (t1 - t0) * xc.shape[0] / len(cr) + (t2 - t1) / min(fr)
        prep[site.name] = (s, gf, bf)
    lin_q = {}
    for lin in w.linears:
        Wl = inp.W[lin.name]
        r = wrows(Wl)
        Wsub = np.ascontiguousarray(Wl[r])
        t0 = time.perf_counter()
        Wq, ws = oracle.quantize_weights(Wsub, prep[lin.site][0])
        dt = time.perf_counter() - t0
        spent += dt
        full += dt * Wl.shape[0] / len(r)
        lin_q[lin.name] = (Wq, ws, len(r), Wl.shape[0])
    rows = _sample_rows(w.M, token_rows)
    R = len(rows)
    t_rows = 0.0
    outs = {}
    for site in w.sites:
        src = next((l.source for l in w.linears if l.site == site.name and l.source), None)
        x = outs[src] if src else np.ascontiguousarray(inp.x[site.name][rows])
        s, gf, bf = prep[site.name]
        t0 = time.perf_counter()
        if site.act == "silu_mul":
            Xq, xs, _ = oracle.silu_mul_quant(x)
        else:
            Xq, xs = oracle.norm_quant(x, site.norm, gf, bf, w.eps)
        t_rows += time.perf_counter() - t0
        for lin in w.linears_of(site.name):
            Wq, ws, n, N = lin_q[lin.name]
            t0 = time.perf_counter()
            acc = oracle.gemm_i64(Xq, Wq)
            _, out = oracle.epilogue(acc, xs, ws, lin.relu)
            dt = time.perf_counter() - t0
            spent += dt
            t_rows += dt * N / n  # the GEMM scales with the output channels too
            if any(l.source == lin.name for l in w.linears):
                # a downstream site reads this output: it needs every channel
                if n < N:
                    out = np.concatenate([out] * ((N + n - 1) // n), axis=1)[:, :N]
                outs[lin.name] = np.ascontiguousarray(out)
    spent += t_rows
    full += t_rows * w.M / R
    desc = ("oracle on %d of %d tokens, %d of %d calibration tokens and up to %d weight "
            "elements per Linear, each phase extrapolated linearly to the full step" %
            (R, w.M, min(cal_rows, w.M_cal), w.M_cal, weight_elems))
    return full, spent, desc


def reference_sample_sizes(w, inp, steps, budget_s=150.0):
    """Sample sizes for `steps` oracle steps to fit in about `budget_s`
    seconds: a tiny probe step measures the cost, the sizes scale from it."""
    probe = dict(cal_rows=8, weight_elems=1 << 20, token_rows=1)
    _, spent, _ = oracle_sample_step(w, inp, **probe)
    per_step = max(0.05, (budget_s - spent) / max(1, steps))
    k = max(1.0, per_step / max(spent, 1e-3))
    return dict(cal_rows=int(min(w.M_cal, 8 * k)),
                weight_elems=int(min(48 << 20, (1 << 20) * k)),
                token_rows=int(max(1, min(16, k))))


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands, on the host cores."""
    import oracle
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    oracle.build()
    inp = S.make_inputs(w, seed=args.seed)
    cores = oracle.num_threads()
    sizes = reference_sample_sizes(w, inp, args.warmup + args.steps)
    times = []
    desc = ""
    for i in range(args.warmup + args.steps):
        full, spent, desc = oracle_sample_step(w, inp, **sizes)
        if i >= args.warmup:
            times.append(full)
    t = sum(times) / len(times)
    ops = workload_ops(w)
    value = ops / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
        "data": "synthetic", "config": {"workload": w.name, "tokens": w.M},
        "tokens_per_s": w.M / t,
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
               0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown",
               0x200: "display_clock_setting"}


class ClockSampler:
    """Samples the SM clock, power and clock-event reasons of one GPU through
    NVML every few milliseconds on a background thread while the timed region
    runs (the same counters nvidia-smi's clocks query reads)."""

    def __init__(self, pci_bus_id=None, period_s=0.005):
        self.period = period_s
        self.pci = pci_bus_id
        self.samples = []
        self._stop = None
        self._thr = None
        self._nvml = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            self._nvml = (pynvml, h)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nvml = None
            return
        self._stop = threading.Event()

        def loop():
            pn, h = self._nvml
            while not self._stop.is_set():
                try:
                    self.samples.append((
                        float(pn.nvmlDeviceGetClockInfo(h, pn.NVML_CLOCK_SM)),
                        pn.nvmlDeviceGetPowerUsage(h) / 1000.0,
                        int(pn.nvmlDeviceGetCurrentClocksEventReasons(h)),
                        float(pn.nvmlDeviceGetUtilizationRates(h).gpu)))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()

    def stop(self):
        if self._nvml is None:
            return None
        self._stop.set()
        self._thr.join(timeout=2)
        try:
            self._nvml[0].nvmlShutdown()
        except Exception:
            pass
        rows = self.samples
        if not rows:
            return None
        reasons = 0
        for r in rows:
            reasons |= r[2]
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(r[0] for r in rows),
                "power_w_max": max(r[1] for r in rows),
                "samples": len(rows), "source": "NVML, every 5 ms during the timed region",
                "reasons": [name for bit, name in REASON_BITS.items() if reasons & bit]}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm.cu", "sq_device.cuh"):
        with open(os.path.join(ROOT, "w8a8_int8_quantized_norm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, or None
    when no summary matches the current kernel source."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    sha = gemm_source_sha()
    pat = re.compile(r"^traffic_per_launch_bytes:\s*(\d+)\s+kernel:\s*(\S+)\s+workload:\s*(\S+)"
                     r"\s+source_sha:\s*([0-9a-f]+)", re.M)
    for f in sorted(os.listdir(d)):
        if not f.endswith((".md", ".txt")):
            continue
        for m in pat.finditer(open(os.path.join(d, f)).read()):
            if m.group(2) == kernel and m.group(3) == workload and m.group(4) == sha:
                return int(m.group(1))
    return None


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from w8a8_int8_quantized_norm_b200 import pipeline, sq
    from w8a8_int8_quantized_norm_b200 import synthetic as S

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    sq.lib()

    inp = rank_inputs(w, args.seed, rank)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
            else torch.from_numpy(a)
        return t.to(dev)

    x = {k: to_dev(v) for k, v in inp.x.items()}
    xc = {k: to_dev(v) for k, v in inp.x_cal.items()}
    W = {k: to_dev(v) for k, v in inp.W.items()}
    g = {k: to_dev(v) for k, v in inp.gamma.items()}
    b = {k: to_dev(v) for k, v in inp.beta.items()}
    blk = pipeline.Block(w, w.M, dev, args.granularity, args.format)
    flusher = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    events = []  # (kind, units, start event, end event) of every library call in a step

    def timer(kind, units, fn):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        events.append((kind, units, e0, e1))

    def step(timed):
        blk.prepare(xc, W, g, b, timer=timer if timed else None)
        blk.forward(x, timer=timer if timed else None)

    # warm-up (eager), then the step captured once as a CUDA graph: the timed
    # region replays it, each replay bracketed by events on the launching
    # stream after an untimed L2 overwrite
    enqueue_s = 0.0
    for _ in range(args.warmup):
        flusher()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        step(True)
        enqueue_s = max(enqueue_s, time.perf_counter() - t0)
        events.clear()
    graph = blk.capture(xc, W, g, b, x)
    for _ in range(args.warmup):
        flusher()
        graph.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)

    pci = None
    try:
        p = torch.cuda.get_device_properties(dev)
        pci = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        pass
    sampler = ClockSampler(pci)
    sampler.start()
    wall0 = time.perf_counter()
    step_ev = []
    for _ in range(args.steps):
        flusher()  # L2 holds nothing of the step's inputs when it starts (untimed)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        step_ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    step_ms = [a.elapsed_time(b_) for a, b_ in step_ev]

    # per-call breakdown: the same step run eagerly, each call bracketed by
    # events; every step waits behind an untimed GPU spin sized from the host's
    # enqueue time, so the queue runs ahead and no host gap enters an interval
    # (each event record still drains the stream: a few microseconds per call)
    head_cycles = int(2.0e9 * (2.0 * enqueue_s + 50e-6))
    n_calls = max(1, min(args.steps, 50))
    for i in range(n_calls):
        flusher()
        torch.cuda._sleep(head_cycles)
        step(True)
        if i % 8 == 7:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    err = sq.get_device_error()
    if err:
        raise SystemExit("device error %s during the benchmark" % sq.status_string(err))
    del graph
    kinds = {}  # kind -> [calls, units, seconds]
    for (kind, units, a, b_) in events:
        k = kinds.setdefault(kind, [0, 0.0, 0.0])
        k[0] += 1
        k[1] += units
        k[2] += a.elapsed_time(b_) / 1e3
    calls_steps = n_calls

    t_rank = sum(step_ms) / 1e3
    ops = workload_ops(w)
    tops_total, t_max = aggregate(ops * args.steps, t_rank, world, dev)
    value = tops_total / 1e12
    tokens_per_s = w.M * args.steps * world / t_max

    # per library call: CUDA events recorded around every call inside the graph
    peaks, peak_src = load_peaks()
    kernels = {}
    for kind, (n, units, secs) in kinds.items():
        if kind == "gemm":
            continue
        gbs = units / secs / 1e9
        kernels[kind] = {"calls": n // calls_steps, "ms_per_call": secs * 1e3 / n,
                         "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                         "bytes_per_call": units / n}
    # dominant kernel: the GEMM
    g_n, g_ops, g_time = kinds["gemm"]
    g_bytes = 0
    for lin in w.linears:
        g_bytes += gemm_bytes(w.M, lin.N, w.site(lin.site).K) * calls_steps
    decode = w.M <= 128
    if decode:
        achieved = g_bytes / g_time / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    else:
        achieved = g_ops / g_time / 1e12
        peak = peaks["bf16_tflops"] * INT8_PER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TOPS",
                "frac": achieved / peak,
                "peak_sustained": peaks.get("bf16_tflops_sustained", 0.0) * INT8_PER_BF16}
    fp8 = args.format == "fp8"
    roof["peak_source"] = "%s (%s)" % (peak_src, "HBM copy" if decode else
                                       "2 x bf16 cuBLAS, the nominal %s:BF16 ratio"
                                       % ("FP8" if fp8 else "INT8"))
    # FP8 GEMMs run whole-K tiles (split 1)
    plan = sq.gemm_plan(w.M, w.linears[0].N, w.site(w.linears[0].site).K, 0, 1 if fp8 else 0)
    kname = sq.GemmPlanInfo.KERNELS[plan.kernel].split(" ")[0]
    # the committed DRAM-traffic summaries cover the INT8 instantiations
    tr = None if fp8 else profile_traffic(kname, w.name)
    roof["traffic"] = None if tr is None else tr
    roof["algorithmic_per_launch"] = (g_bytes if decode else g_ops) / g_n
    roof["kernel"] = kname
    roof["plan"] = {k: v for k, v in plan.as_dict().items() if k != "kernel"}
    roof["launch_ms_mean"] = g_time * 1e3 / g_n
    roof["timing"] = ("CUDA events on the launching stream around each GEMM call, in %d eager "
                      "steps run right after the graph-timed ones (a call = the main kernel "
                      "plus its fix-up kernel when the plan has one; the interval includes "
                      "the event records' own drain)" % calls_steps)

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_max * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3" if args.format == "fp8" else "int8",
        "data": "synthetic (seeded outlier-channel activations, N(0,0.02) weights)",
        "config": {"workload": w.name, "tokens": w.M, "calib_tokens": w.M_cal, "alpha": w.alpha,
                   "linears": ["%s %dx%d" % (l.name, w.site(l.site).K, l.N) for l in w.linears],
                   "step": "calibrate + smooth scales/fold + weight quant + norm-quant + GEMM",
                   "granularity": args.granularity, "format": args.format,
                   "launch": "the whole step as one CUDA graph, replayed per timed step",
                   "l2": "flushed before every step (256 MiB written, then another 256 MiB "
                         "read so no dirty line is left to write back; not timed)",
                   "parallelism": "dp%d (independent token batches, weights replicated)" % world},
        "tokens_per_s": tokens_per_s,
        "forward_gemm_tops": g_ops / g_time / 1e12,
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": args.steps * (blk.prepare_launches() + blk.forward_launches()),
        "clocks": clocks,
        "wall_s_timed": wall,
    }

    # end to end through the public API: pinned host inputs in, results out
    if not args.no_e2e:
        line["e2e"] = e2e_leg(args, w, inp, blk, dev, stream, world)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()

    # the oracle's baseline is the per-token path (the method's default scheme)
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and args.granularity == "per_token"
            and args.format == "int8"):
        import oracle
        oracle.build()
        full, spent, desc = oracle_sample_step(w, inp)
        line["cpu_baseline"] = {"value": workload_ops(w) / full / 1e12, "unit": "TOPS",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": desc + " (%.1f s of CPU time)" % spent}
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_leg(args, w, inp, blk, dev, stream, world):
    import torch

    def pinned(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
            else torch.from_numpy(a)
        return t.pin_memory()

    hx = {k: pinned(v) for k, v in inp.x.items()}
    hxc = {k: pinned(v) for k, v in inp.x_cal.items()}
    hW = {k: pinned(v) for k, v in inp.W.items()}
    hg = {k: pinned(v) for k, v in inp.gamma.items()}
    hb = {k: pinned(v) for k, v in inp.beta.items()}
    dx = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in hx.items()}
    dxc = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in hxc.items()}
    dW = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in hW.items()}
    dg = {k: (None if v is None else torch.empty(v.shape, dtype=v.dtype, device=dev))
          for k, v in hg.items()}
    db = {k: (None if v is None else torch.empty(v.shape, dtype=v.dtype, device=dev))
          for k, v in hb.items()}
    hout = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in blk.out.items()}
    h2d = sum(t.numel() * t.element_size() for d in (hx, hxc, hW, hg, hb) for t in d.values()
              if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in hout.values())

    def step():
        for src, dst in ((hx, dx), (hxc, dxc), (hW, dW), (hg, dg), (hb, db)):
            for k, t in src.items():
                if t is not None:
                    dst[k].copy_(t, non_blocking=True)
        blk.prepare(dxc, dW, dg, db)
        out = blk.forward(dx)
        for k, t in out.items():
            hout[k].copy_(t, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    n = max(1, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / 1e3
    value, _ = aggregate(workload_ops(w) * n, t, world, dev)
    return {"value": value / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "path": "pinned host -> device copies, the six C-ABI calls, device -> pinned host"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--granularity", default="per_token",
                    choices=["per_token", "per_tensor_dynamic", "per_tensor_static"],
                    help="activation / weight scale sharing (per-token + per-channel, or the "
                         "per-tensor O2 / O3 levels)")
    ap.add_argument("--format", choices=["int8", "fp8"], default="int8",
                    help="code format: INT8 (the method as published) or FP8 e4m3 with the "
                         "same smoothing")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    if args.workload not in S.WORKLOADS:
        ap.error("unknown workload; choose from: %s" % ", ".join(S.WORKLOADS))
    w = S.WORKLOADS[args.workload]
    if args.impl == "reference":
        world, rank, _ = dist_env()
        if rank != 0:
            return 0
        run_reference(args, w)
        return 0
    run_gpu(args, w)
    return 0


if __name__ == "__main__":
    sys.exit(main())
