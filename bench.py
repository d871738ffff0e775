#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 linear path on B200 (one JSON line).

The default workload is the Llama-style decoder block (hidden 8192, 8 x 2048
tokens: RMSNorm -> QKV, o_proj, RMSNorm -> gate_up, SiLU(gate)*up -> down).
A timed step is the runtime forward of every Linear of the block: fused norm
+ per-token INT8 quantisation (or SiLU(gate)*up + quantisation), INT8 GEMM
with the dequant epilogue; ``value`` is its throughput.  The offline rows
(calibration, smoothing factors + fold, weight smoothing + INT8 quantisation)
run in the same job and are reported under ``offline_prep``; the decode
sweep (M = 1, 8, 32, 128 tokens per step on the same weights) under
``decode``.

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
DEFAULT_WORKLOAD = "llama-block-8192-prefill-16384tok"
DECODE_TOKENS = (1, 8, 32, 128)
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
    if k is None or k >= n:
        return np.arange(n)
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False))


# the oracle's sample of each workload for the CPU baseline: the two small
# workloads run in full; the larger ones run the weight rows (K2) and the
# calibration in full, K1 on 1024 tokens and the GEMMs on 16, each phase's
# time scaled to the full step
FULL_SAMPLE = dict(cal_rows=None, weight_elems=None, norm_rows=None, gemm_rows=None)
LARGE_SAMPLE = dict(cal_rows=None, weight_elems=None, norm_rows=1024, gemm_rows=16)


def cpu_sample_for(w):
    return FULL_SAMPLE if w.gemm_ops() <= 4e11 else LARGE_SAMPLE


def oracle_sample_step(w, inp, cal_rows=None, weight_elems=None, norm_rows=None, gemm_rows=None):
    """One oracle step (the offline rows, then the forward) on a sample of
    the workload: ``cal_rows`` calibration tokens, at most ``weight_elems``
    weight elements per Linear (whole rows), ``norm_rows`` tokens through the
    norm + quantisation and ``gemm_rows`` of them through the GEMMs (None =
    all).  Each phase's time is scaled linearly to the full workload.
    Returns (seconds for the full step, seconds spent, text, full)."""
    import oracle
    spent = 0.0
    est = 0.0
    prep = {}
    extrap = False

    def wrows(Wl):
        if weight_elems is None:
            return np.arange(Wl.shape[0])
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
                Ws.append(Wl if len(r) == Wl.shape[0] else np.ascontiguousarray(Wl[r]))
                fr.append(len(r) / Wl.shape[0])
            t0 = time.perf_counter()
            am = oracle.calibrate_absmax(xcs, site.norm, g, b, w.eps)
            t1 = time.perf_counter()
            s, _ = oracle.smooth_scales(am, Ws, w.alpha, w.clamp_eps)
            gf, bf = oracle.fold_norm(s, g, b)
            t2 = time.perf_counter()
            spent += t2 - t0
            est += (t1 - t0) * xc.shape[0] / len(cr) + (t2 - t1) / min(fr)
            extrap |= len(cr) < xc.shape[0] or min(fr) < 1.0
        prep[site.name] = (s, gf, bf)
    lin_q = {}
    for lin in w.linears:
        Wl = inp.W[lin.name]
        r = wrows(Wl)
        Wsub = Wl if len(r) == Wl.shape[0] else np.ascontiguousarray(Wl[r])
        t0 = time.perf_counter()
        Wq, ws = oracle.quantize_weights(Wsub, prep[lin.site][0])
        dt = time.perf_counter() - t0
        spent += dt
        est += dt * Wl.shape[0] / len(r)
        extrap |= len(r) < Wl.shape[0]
        lin_q[lin.name] = (Wq, ws, len(r), Wl.shape[0])
    nrows = _sample_rows(w.M, norm_rows)
    R = len(nrows)
    G = R if gemm_rows is None else min(R, gemm_rows)
    extrap |= R < w.M or G < w.M
    outs = {}
    for site in w.sites:
        src = next((l.source for l in w.linears if l.site == site.name and l.source), None)
        # a site fed by a Linear's output has the GEMM's rows only
        x = outs[src] if src else np.ascontiguousarray(inp.x[site.name][nrows])
        rows = x.shape[0]
        s, gf, bf = prep[site.name]
        t0 = time.perf_counter()
        if site.act == "silu_mul":
            Xq, xs, _ = oracle.silu_mul_quant(x)
        else:
            Xq, xs = oracle.norm_quant(x, site.norm, gf, bf, w.eps)
        dt = time.perf_counter() - t0
        spent += dt
        est += dt * w.M / rows
        for lin in w.linears_of(site.name):
            Wq, ws, n, N = lin_q[lin.name]
            Xg = np.ascontiguousarray(Xq[:G])
            t0 = time.perf_counter()
            acc = oracle.gemm_i64(Xg, Wq)
            _, out = oracle.epilogue(acc, xs[:G], ws, lin.relu)
            dt = time.perf_counter() - t0
            spent += dt
            est += dt * (w.M / G) * (N / n)  # the GEMM scales with tokens and channels
            if any(l.source == lin.name for l in w.linears):
                # a downstream site reads this output: it needs every channel
                if n < N:
                    out = np.concatenate([out] * ((N + n - 1) // n), axis=1)[:, :N]
                outs[lin.name] = np.ascontiguousarray(out)
    if not extrap:
        desc = "the oracle on the whole step (all %d tokens, %d calibration tokens, every weight)" % (
            w.M, w.M_cal)
    else:
        desc = ("oracle: %d of %d calibration tokens, %s weight rows, %d of %d tokens through "
                "norm + quantisation and %d through the GEMMs; each phase's time extrapolated "
                "linearly to the full step" %
                (w.M_cal if cal_rows is None else min(cal_rows, w.M_cal), w.M_cal,
                 "all" if weight_elems is None else "up to %d elements of" % weight_elems,
                 R, w.M, G))
    return est, spent, desc, not extrap


def reference_sample_sizes(w, inp, steps, budget_s=150.0):
    """Sample sizes for `steps` oracle steps to fit in about `budget_s`
    seconds: a tiny probe step measures the cost, the sizes scale from it."""
    probe = dict(cal_rows=8, weight_elems=1 << 20, norm_rows=1, gemm_rows=1)
    _, spent, _, _ = oracle_sample_step(w, inp, **probe)
    per_step = max(0.05, (budget_s - spent) / max(1, steps))
    k = max(1.0, per_step / max(spent, 1e-3))
    return dict(cal_rows=int(min(w.M_cal, 8 * k)),
                weight_elems=int(min(48 << 20, (1 << 20) * k)),
                norm_rows=int(max(1, min(w.M, 64 * k))),
                gemm_rows=int(max(1, min(16, k))))


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
        est, spent, desc, _ = oracle_sample_step(w, inp, **sizes)
        if i >= args.warmup:
            times.append(est)
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
                         "sample": desc + "; the oracle's whole step (offline rows + forward)"},
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


def _to_dev(a, dev):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
        else torch.from_numpy(a)
    return t.to(dev)


def _timed_replays(graph, n, flusher, stream):
    """Device time (ms) of each of ``n`` replays of ``graph``, every replay
    bracketed by CUDA events on the launching stream after an untimed L2
    flush."""
    import torch
    ev = []
    for _ in range(n):
        flusher()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _call_breakdown(run_step, n, flusher, stream, head_cycles, dev):
    """Per library call device times: ``n`` eager steps, every call
    bracketed by CUDA events (the ``timer`` hook of the pipeline).  Each step
    waits behind an untimed GPU spin sized from the host's enqueue time, so
    the queue runs ahead and no host gap enters an interval (each event
    record still drains the stream: a few microseconds per call).  Returns
    {kind: [calls, units, seconds]}."""
    import torch
    events = []

    def timer(kind, units, fn):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        events.append((kind, units, e0, e1))

    for i in range(n):
        flusher()
        torch.cuda._sleep(head_cycles)
        run_step(timer)
        if i % 8 == 7:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    kinds = {}
    for (kind, units, a, b_) in events:
        k = kinds.setdefault(kind, [0, 0.0, 0.0])
        k[0] += 1
        k[1] += units
        k[2] += a.elapsed_time(b_) / 1e3
    return kinds


def _row_kernels(kinds, n_steps, hbm):
    out = {}
    for kind, (n, units, secs) in kinds.items():
        if kind.startswith("gemm:"):
            continue
        gbs = units / secs / 1e9
        out[kind] = {"calls": n // n_steps, "ms_per_call": secs * 1e3 / n, "achieved_gbs": gbs,
                     "frac_hbm": gbs / hbm, "bytes_per_call": units / n}
    return out


def _gemm_calls(w, M, kinds, peaks):
    """Per-Linear GEMM call times: TOPS against the INT8 peak for prefill
    shapes, algorithmic GB/s against HBM for decode shapes (M <= 128)."""
    out = {}
    for lin in w.linears:
        K = w.site(lin.site).K
        n, ops, secs = kinds["gemm:" + lin.name]
        t = secs / n
        d = {"shape": "%dx%dx%d" % (M, lin.N, K), "ms_per_call": t * 1e3,
             "tops": 2.0 * M * lin.N * K / t / 1e12}
        if M <= 128:
            gb = gemm_bytes(M, lin.N, K)
            d.update(bytes_per_call=gb, achieved_gbs=gb / t / 1e9,
                     frac_hbm=gb / t / 1e9 / peaks["hbm_gbs"])
        else:
            d["frac_int8_peak"] = d["tops"] / (peaks["bf16_tflops"] * INT8_PER_BF16)
        out[lin.name] = d
    return out


def _forward_bytes(w, M, blk):
    """Algorithmic bytes of one forward: every GEMM's operands, scales and
    bf16 output, and every row kernel's input read, codes written, scales and
    norm parameters."""
    total = 0
    for lin in w.linears:
        total += gemm_bytes(M, lin.N, w.site(lin.site).K)
    for site in w.sites:
        nparam = (blk.gamma_f[site.name] is not None) + (blk.beta_f[site.name] is not None)
        width = 2 * site.K if site.act == "silu_mul" else site.K
        total += M * width * 2 + M * site.K + 4 * M + 4 * site.K * nparam
    return total


def decode_sweep(args, w, blk, dev, stream, flusher, peaks, seed, rank):
    """The decode configurations on the prefill block's weights: for M tokens
    per step, the runtime forward (norm + per-token quantisation, the four
    GEMMs) as one CUDA graph, timed like the main loop; plus each GEMM call's
    time from eager steps.  Weight bytes dominate: every step streams all the
    INT8 weights once."""
    import torch
    from w8a8_int8_quantized_norm_b200 import pipeline
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    res = {}
    for M in DECODE_TOKENS:
        wd = S.WORKLOADS["llama-block-8192-decode-m%d" % M]
        inp = S.make_inputs(wd, seed=seed, weights=False, token_seed=seed + 1000003 * rank)
        x = {k: _to_dev(v, dev) for k, v in inp.x.items()}
        bd = pipeline.Block(wd, M, dev, args.granularity, args.format, shared=blk)
        graph = pipeline.capture_forward(bd, x)
        for _ in range(3):
            flusher()
            graph.replay()
        n = max(10, args.steps)
        ms = _timed_replays(graph, n, flusher, stream)
        t = sum(ms) / n / 1e3
        del graph
        kinds = _call_breakdown(lambda timer: bd.forward(x, timer=timer), min(n, 20), flusher,
                                stream, int(2.0e9 * 200e-6), dev)
        gemms = _gemm_calls(wd, M, kinds, peaks)
        gb = sum(g["bytes_per_call"] for g in gemms.values())
        gt = sum(g["ms_per_call"] for g in gemms.values()) / 1e3
        fb = _forward_bytes(wd, M, bd)
        res["m%d" % M] = {
            "tokens": M, "us_per_step": t * 1e6, "tokens_per_s": M / t,
            "tops": wd.gemm_ops() / t / 1e12, "bytes_per_step": fb,
            "achieved_gbs": fb / t / 1e9, "frac_hbm": fb / t / 1e9 / peaks["hbm_gbs"],
            "gemm_calls": {"achieved_gbs": gb / gt / 1e9,
                           "frac_hbm": gb / gt / 1e9 / peaks["hbm_gbs"],
                           "per_linear": gemms},
            "row_kernels": _row_kernels(kinds, min(n, 20), peaks["hbm_gbs"]),
            "launches_per_step": bd.forward_launches(),
        }
    return res


def comparator_leg(args, w, inp, dev, stream, flusher, peaks, rank):
    """LLM.int8()'s decomposition against the W8A8 layer on one Linear of the
    block that has no norm in front (o_proj, the attention-output activations
    with their outlier channels): the runtime forward of plain per-token INT8
    (no smoothing), of LLM.int8() (tau = 6) and of SmoothQuant (alpha of the
    workload, 1/s as a per-channel multiplier: the fold with gamma = 1), each
    one CUDA graph timed like the main loop, and each one's output error on
    sampled token rows against an fp64 product of the same bf16 inputs."""
    import torch
    from w8a8_int8_quantized_norm_b200 import llmint8, pipeline, sq
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    lin = next(l for l in w.linears if l.name == "o_proj")
    site = w.site(lin.site)
    M, K, N = w.M, site.K, lin.N
    x = _to_dev(inp.x[site.name], dev)
    W = _to_dev(inp.W[lin.name], dev)
    xcal = _to_dev(S.activations(w, site.name, w.M_cal, "x_cal", args.seed), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    # plain per-token INT8 and SmoothQuant: the same two calls, with or without s
    Wq_p, ws_p = sq.smooth_quantize_weights(W, None)
    am = torch.zeros(K, **f32)
    sq.calibrate_absmax(xcal, sq.NORM_NONE, act_max=am)
    s_, gf = torch.empty(K, **f32), torch.empty(K, **f32)
    sq.compute_smooth_scales(am, [W], w.alpha, w.clamp_eps, None, None, s=s_, gamma_folded=gf)
    Wq_s, ws_s = sq.smooth_quantize_weights(W, s_)
    xq, xs = torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty(M, **f32)
    outs = {k: torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            for k in ("plain_int8", "llm_int8", "smoothquant")}

    def w8a8(mult, Wq, ws, out):
        sq.norm_smooth_quant_per_token(x, sq.NORM_NONE, mult, None, 0.0, Xq=xq, x_scale=xs)
        sq.w8a8_gemm_dequant(xq, Wq, xs, ws, "bf16", out=out)

    comp = llmint8.LLMInt8Linear(W, 6.0).prepare()
    runs = {"plain_int8": lambda: w8a8(None, Wq_p, ws_p, outs["plain_int8"]),
            "llm_int8": lambda: comp.forward(x, out=outs["llm_int8"]),
            "smoothquant": lambda: w8a8(gf, Wq_s, ws_s, outs["smoothquant"])}
    launches = {"plain_int8": 1 + sq.gemm_plan(M, N, K).launches,
                "llm_int8": comp.launches(M),
                "smoothquant": 1 + sq.gemm_plan(M, N, K).launches}
    res = {}
    for name, fn in runs.items():
        graph = pipeline.capture_graph(fn)
        for _ in range(3):
            flusher()
            graph.replay()
        n = max(5, min(args.steps, 20))
        ms = _timed_replays(graph, n, flusher, stream)
        t = sum(ms) / n / 1e3
        del graph
        res[name] = {"ms": t * 1e3, "tops": 2.0 * M * N * K / t / 1e12,
                     "launches": launches[name]}
    torch.cuda.synchronize(dev)
    # output error on sampled rows against the fp64 product of the bf16 inputs
    rows = _sample_rows(M, 64, seed=5)
    xr = inp.x[site.name][rows]
    bf = lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = bf(xr) @ bf(inp.W[lin.name]).T
    for name in runs:
        got = outs[name][torch.from_numpy(rows).to(dev)].float().cpu().numpy().astype(np.float64)
        res[name]["rel_error"] = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    res["smoothquant"]["alpha"] = w.alpha
    return {"linear": "%s %dx%dx%d (M x K x N), input: %s activations" % (
                lin.name, M, K, N, site.name),
            "tau": 6.0, "outlier_channels": int(comp.count.item()),
            "error": "relative Frobenius error of the bf16 output on %d token rows against "
                     "the fp64 product of the same bf16 x and W" % len(rows),
            "timing": "each method's runtime calls as one CUDA graph, L2 flushed before "
                      "every replay",
            **res}


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from w8a8_int8_quantized_norm_b200 import pipeline, sq

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
    x = {k: _to_dev(v, dev) for k, v in inp.x.items()}
    xc = {k: _to_dev(v, dev) for k, v in inp.x_cal.items()}
    W = {k: _to_dev(v, dev) for k, v in inp.W.items()}
    g = {k: _to_dev(v, dev) for k, v in inp.gamma.items()}
    b = {k: _to_dev(v, dev) for k, v in inp.beta.items()}
    blk = pipeline.Block(w, w.M, dev, args.granularity, args.format)
    flusher = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    # warm-up (eager), measuring the host's enqueue time of one step
    enqueue_s = 0.0
    for _ in range(args.warmup):
        flusher()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        blk.prepare(xc, W, g, b)
        blk.forward(x)
        enqueue_s = max(enqueue_s, time.perf_counter() - t0)
    # the offline rows and the runtime forward, each captured once as a graph
    prep_graph = pipeline.capture_prepare(blk, xc, W, g, b)
    fwd_graph = pipeline.capture_forward(blk, x)
    prep_graph.replay()
    for _ in range(args.warmup):
        flusher()
        fwd_graph.replay()
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
    # ---- the timed region: K forward steps (runtime rows of every Linear)
    sampler = ClockSampler(pci)
    sampler.start()
    wall0 = time.perf_counter()
    step_ms = _timed_replays(fwd_graph, args.steps, flusher, stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()

    t_rank = sum(step_ms) / 1e3
    ops = workload_ops(w)
    tops_total, t_max = aggregate(ops * args.steps, t_rank, world, dev)
    value = tops_total / 1e12
    tokens_per_s = w.M * args.steps * world / t_max
    peaks, peak_src = load_peaks()

    # ---- the offline rows, timed the same way (one-time work per weight set)
    n_prep = max(3, min(args.steps, 10))
    prep_ms = _timed_replays(prep_graph, n_prep, flusher, stream)
    prep_t = sum(prep_ms) / n_prep / 1e3
    del prep_graph, fwd_graph

    # ---- per-call breakdown from eager steps
    head_cycles = int(2.0e9 * (2.0 * enqueue_s + 50e-6))
    n_calls = max(1, min(args.steps, 20))

    def eager_step(timer):
        blk.prepare(xc, W, g, b, timer=timer)
        blk.forward(x, timer=timer)

    kinds = _call_breakdown(eager_step, n_calls, flusher, stream, head_cycles, dev)
    kernels = _row_kernels(kinds, n_calls, peaks["hbm_gbs"])
    gemms = _gemm_calls(w, w.M, kinds, peaks)
    prep_kinds = ("calibrate", "smooth_scales", "weight_quant", "static_absmax")
    prep_bytes = sum(kinds[k][1] for k in prep_kinds if k in kinds) / n_calls

    # dominant kernel: the GEMM call with the most work
    dom = max(w.linears, key=lambda l: l.N * w.site(l.site).K)
    K_dom = w.site(dom.site).K
    n_dom, _, secs_dom = kinds["gemm:" + dom.name]
    t_dom = secs_dom / n_dom
    decode = w.M <= 128
    fp8 = args.format == "fp8"
    if decode:
        alg = gemm_bytes(w.M, dom.N, K_dom)
        achieved = alg / t_dom / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    else:
        alg = 2.0 * w.M * dom.N * K_dom
        achieved = alg / t_dom / 1e12
        peak = peaks["bf16_tflops"] * INT8_PER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TOPS",
                "frac": achieved / peak,
                "peak_sustained": peaks.get("bf16_tflops_sustained", 0.0) * INT8_PER_BF16}
    roof["peak_source"] = "%s (%s)" % (peak_src, "HBM copy" if decode else
                                       "2 x bf16 cuBLAS, the nominal %s:BF16 ratio"
                                       % ("FP8" if fp8 else "INT8"))
    # FP8 GEMMs run whole-K tiles (split 1)
    plan = sq.gemm_plan(w.M, dom.N, K_dom, 0, 1 if fp8 else 0)
    kname = sq.GemmPlanInfo.KERNELS[plan.kernel].split(" ")[0]
    # the committed DRAM-traffic summaries cover the INT8 instantiations
    tr = None
    if not fp8:
        tr = profile_traffic(kname, "%s:%s" % (w.name, dom.name))
        if tr is None and len(w.linears) == 1:
            tr = profile_traffic(kname, w.name)
    roof["traffic"] = tr
    roof["algorithmic_per_launch"] = alg
    roof["kernel"] = kname
    roof["linear"] = "%s %dx%dx%d (M x N x K)" % (dom.name, w.M, dom.N, K_dom)
    roof["plan"] = {k: v for k, v in plan.as_dict().items() if k != "kernel"}
    roof["launch_ms_mean"] = t_dom * 1e3
    roof["timing"] = ("CUDA events on the launching stream around each %s GEMM call, in %d "
                      "eager steps run right after the timed ones (a call = the main kernel "
                      "plus its fix-up kernel when the plan has one; the interval includes "
                      "the event records' own drain)" % (dom.name, n_calls))

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_max * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3" if fp8 else "int8",
        "data": "synthetic (seeded outlier-channel activations, N(0,0.02) weights)",
        "config": {"workload": w.name, "tokens": w.M, "calib_tokens": w.M_cal, "alpha": w.alpha,
                   "linears": ["%s %dx%d" % (l.name, w.site(l.site).K, l.N) for l in w.linears],
                   "step": "the runtime forward of every Linear: norm + per-token quant (or "
                           "SiLU(gate)*up + quant), INT8 GEMM with the dequant epilogue; the "
                           "offline rows (calibration, smoothing factors + fold, weight "
                           "quant) are timed separately under offline_prep",
                   "granularity": args.granularity, "format": args.format,
                   "launch": "the forward as one CUDA graph, replayed per timed step",
                   "l2": "flushed before every step (256 MiB written, then another 256 MiB "
                         "read so no dirty line is left to write back; not timed)",
                   "parallelism": "dp%d (independent token batches, weights replicated)" % world},
        "tokens_per_s": tokens_per_s,
        "forward_gemm_tops": sum(kinds["gemm:" + l.name][1] for l in w.linears)
        / sum(kinds["gemm:" + l.name][2] for l in w.linears) / 1e12,
        "roofline": roof,
        "gemms": gemms,
        "kernels": kernels,
        "offline_prep": {
            "ms": prep_t * 1e3, "bytes": prep_bytes, "achieved_gbs": prep_bytes / prep_t / 1e9,
            "frac_hbm": prep_bytes / prep_t / 1e9 / peaks["hbm_gbs"],
            "launches": blk.prepare_launches(), "replays": n_prep,
            "what": "calibration (beside the weight column maxima, two streams), smoothing "
                    "factors + fold, weight smoothing + quantisation of every Linear, as one "
                    "CUDA graph; bytes = the calls' algorithmic bytes"},
        "whole_path_ms": t_max * 1e3 / args.steps + prep_t * 1e3,
        "gpu_launches": args.steps * blk.forward_launches(),
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if (not args.no_decode and not decode and w.name.startswith("llama-block-8192")
            and args.format == "int8" and args.granularity == "per_token"):
        line["decode"] = decode_sweep(args, w, blk, dev, stream, flusher, peaks, args.seed, rank)
    if (not args.no_comparator and w.name.startswith("llama-block-8192") and not decode
            and args.format == "int8"):
        line["comparator"] = comparator_leg(args, w, inp, dev, stream, flusher, peaks, rank)
    err = sq.get_device_error()
    if err:
        raise SystemExit("device error %s during the benchmark" % sq.status_string(err))

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
        est, spent, desc, full = oracle_sample_step(w, inp, **cpu_sample_for(w))
        line["cpu_baseline"] = {
            "value": workload_ops(w) / est / 1e12, "unit": "TOPS",
            "cores": oracle.num_threads(), "kind": "oracle",
            "measured": "in full" if full else "extrapolated from a sample",
            "sample": desc + " (%.1f s of CPU time; the oracle's whole step, offline rows "
                             "included)" % spent}
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_leg(args, w, inp, blk, dev, stream, world):
    """The forward through the public API with its activations in pinned host
    memory: every step copies the step's input tokens in, runs the library
    calls and copies the block's results (the outputs no later Linear of the
    block consumes) back to pinned host memory.

    The steps are pipelined the way a serving loop overlaps its transfers:
    two Blocks share the prepared weights and take the steps in turn, each
    with its own device inputs and outputs; step i's inputs go in on one copy
    stream and step i's results come out on another while the neighbouring
    steps' forwards run on the compute stream (PCIe moves both directions at
    once).  Events order each copy after the forward that last read or
    wrote its buffers.  The interval runs from the first input copy to the
    last result copy, timed by events."""
    import torch
    from w8a8_int8_quantized_norm_b200 import pipeline

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
            else torch.from_numpy(a)
        return t.pin_memory()

    hx = {k: pinned(v) for k, v in inp.x.items()}
    blks = [blk, pipeline.Block(w, blk.M, dev, blk.granularity, blk.fmt, shared=blk)]
    dxs = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in hx.items()}
           for _ in blks]
    consumed = {l.source for l in w.linears if l.source}
    results = [k for k in blk.out if k not in consumed]
    houts = [{k: torch.empty(b.out[k].shape, dtype=b.out[k].dtype).pin_memory() for k in results}
             for b in blks]
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in houts[0].values())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_fw, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        b = i % 2
        if used[b]:  # forward i - 2 read these inputs
            s_in.wait_event(ev_fw[b])
        with torch.cuda.stream(s_in):
            for k, t in hx.items():
                dxs[b][k].copy_(t, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if used[b]:  # the results of step i - 2 have left these outputs
            stream.wait_event(ev_out[b])
        with torch.cuda.stream(stream):
            out = blks[b].forward(dxs[b], stream=stream)
        ev_fw[b].record(stream)
        s_out.wait_event(ev_fw[b])
        with torch.cuda.stream(s_out):
            for k in results:
                houts[b][k].copy_(out[k], non_blocking=True)
        ev_out[b].record(s_out)
        used[b] = True

    for i in range(max(2, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    n = max(2, min(args.steps, 20))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        step(i)
    e1.record(s_out)  # after the last result copy, which follows every earlier step
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / 1e3
    value, _ = aggregate(workload_ops(w) * n, t, world, dev)
    return {"value": value / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": t / n * 1e3,
            "path": "pinned host tokens -> device, the forward's C-ABI calls (Block.forward), "
                    "the block's results -> pinned host, every step; weights prepared once "
                    "beforehand; two Blocks sharing the weights take the steps in turn so one "
                    "step's copies overlap the neighbouring steps' forwards (copy streams in "
                    "each direction, ordered by events)"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip LLM.int8()'s decomposition against the W8A8 layer on o_proj")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode sweep (M = 1, 8, 32, 128 on the Llama block weights)")
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
