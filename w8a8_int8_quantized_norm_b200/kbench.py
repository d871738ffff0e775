"""Per-kernel timing through the C ABI, one library call at a time.

    python -m w8a8_int8_quantized_norm_b200.kbench norm_quant --M 16384 --K 8192 --norm rms
    python -m w8a8_int8_quantized_norm_b200.kbench gemm --M 2048 --N 12288 --K 4096 --path 1
    python -m w8a8_int8_quantized_norm_b200.kbench calibrate --M 4096 --K 8192 --norm layer
    python -m w8a8_int8_quantized_norm_b200.kbench weight_quant --N 28672 --K 8192
    python -m w8a8_int8_quantized_norm_b200.kbench smooth_scales --N 12288 --K 4096
    python -m w8a8_int8_quantized_norm_b200.kbench quant_given --M 4096 --K 36864
    python -m w8a8_int8_quantized_norm_b200.kbench silu_mul_quant --M 16384 --K 28672
    python -m w8a8_int8_quantized_norm_b200.kbench gemm --M 4096 --N 36864 --K 9216 --rowmax
    python -m w8a8_int8_quantized_norm_b200.kbench llmint8_combine --M 16384 --N 8192 --K 8192

Each call is captured once as a CUDA graph; every timed replay is bracketed by
CUDA events on the launching stream, with L2 emptied before it (256 MiB
written, then 256 MiB of another buffer read, so only clean lines remain;
untimed): the operands come from HBM, no write-back of the flush is charged to
the call, and no host work falls inside the interval.  Prints one JSON line: mean time per call, the call's algorithmic
bytes (row kernels, GEMMs with at most 128 tokens) or integer ops (other
GEMMs), and the fraction of the measured peak.  Inputs are seeded synthetic
tensors made on the device: N(0, 1) activations with a few outlier channels
scaled by 20-100, N(0, 0.02) weights, random INT8 codes for GEMM operands.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

from . import sq

NORMS = {"none": sq.NORM_NONE, "rms": sq.NORM_RMS, "layer": sq.NORM_LAYER}
L2_FLUSH_BYTES = 256 << 20
INT8_PER_BF16 = 2  # nominal INT8 : BF16 dense tensor-core ratio


def _peaks():
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def _acts(M, K, dtype, gen, dev):
    x = torch.randn((M, K), generator=gen, device=dev, dtype=torch.float32)
    ch = torch.randperm(K, generator=gen, device=dev)[:max(1, K // 1000)]
    x[:, ch] *= torch.empty(ch.numel(), device=dev).uniform_(20, 100, generator=gen)
    return x.to(torch.bfloat16) if dtype == "bf16" else x


def _codes(R, K, gen, dev):
    return torch.randint(-127, 128, (R, K), generator=gen, device=dev, dtype=torch.int8)


class _L2Flush:
    """Writes a buffer larger than L2, then reads a second one: L2 is left
    holding clean lines only, so the timed call pays no write-back of the
    flush's own dirty lines."""

    def __init__(self, dev):
        n = L2_FLUSH_BYTES // 4
        self.w = torch.empty(n, dtype=torch.float32, device=dev)
        self.r = torch.zeros(n, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.sink)


def _time(fn, iters, warmup, flush):
    """Mean device time of one call: the call is captured once as a CUDA graph
    (no host work inside the timed interval) and each replay is bracketed by
    events, after an untimed L2 overwrite."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(iters):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        e1.synchronize()
        total += e0.elapsed_time(e1)
    del graph
    return total / iters * 1e3  # microseconds per call


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("op", choices=["norm_quant", "gemm", "calibrate", "weight_quant",
                                   "smooth_scales", "quant_given", "silu_mul_quant",
                                   "llmint8_combine"])
    ap.add_argument("--outliers", type=int, default=8,
                    help="llmint8_combine: outlier channels of x (x50, the rest N(0, 1))")
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--norm", choices=sorted(NORMS), default="rms")
    ap.add_argument("--dtype", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--path", type=int, default=0, help="GEMM path hint (0 = auto)")
    ap.add_argument("--split", type=int, default=0, help="GEMM split-K (0 = auto)")
    ap.add_argument("--epi", choices=["bf16", "bf16_relu", "i32"], default="bf16")
    ap.add_argument("--fp8", action="store_true", help="GEMM: e4m3 operands (kind::f8f6f4)")
    ap.add_argument("--rowmax", action="store_true",
                    help="GEMM: also reduce each output row's max |out| (prefill tiles)")
    ap.add_argument("--iters", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("kbench needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sq.lib()
    gen = torch.Generator(device=dev)
    gen.manual_seed(a.seed)
    flush = _L2Flush(dev)
    hbm, bf16, src = _peaks()
    M, N, K = a.M, a.N, a.K
    norm = NORMS[a.norm]
    esz = 2 if a.dtype == "bf16" else 4
    shape = {}
    if a.op == "norm_quant":
        x = _acts(M, K, a.dtype, gen, dev)
        g = torch.empty(K, device=dev).uniform_(0.5, 1.5, generator=gen) if norm else None
        b = torch.randn(K, generator=gen, device=dev) * 0.1 if norm == sq.NORM_LAYER else None
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        xs = torch.empty(M, dtype=torch.float32, device=dev)
        fn = lambda: sq.norm_smooth_quant_per_token(x, norm, g, b, 1e-5, xq, xs)
        units = M * K * (esz + 1) + 4 * M + 4 * K * ((g is not None) + (b is not None))
        shape = {"M": M, "K": K, "norm": a.norm, "dtype": a.dtype}
    elif a.op == "quant_given":
        x = _acts(M, K, a.dtype, gen, dev)
        am = x.float().abs().amax(dim=1).contiguous()
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        xs = torch.empty(M, dtype=torch.float32, device=dev)
        fn = lambda: sq.quant_per_token_given_absmax(x, am, xq, xs)
        units = M * K * (esz + 1) + 8 * M
        shape = {"M": M, "K": K, "dtype": a.dtype}
    elif a.op == "silu_mul_quant":
        # K is the width of h; the input rows hold gate and up (2K)
        gu = (torch.randn((M, 2 * K), generator=gen, device=dev) * 2.0).to(torch.bfloat16)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        xs = torch.empty(M, dtype=torch.float32, device=dev)
        fn = lambda: sq.silu_mul_quant_per_token(gu, xq, xs)
        units = M * 2 * K * 2 + M * K + 4 * M
        shape = {"M": M, "I": K, "dtype": "bf16"}
    elif a.op == "llmint8_combine":
        # LLM.int8()'s merge on [M, N] outputs of a K-deep Linear: the INT32
        # accumulator read, the 16-bit lane over the outlier channels, bf16 out
        x = torch.randn((M, K), generator=gen, device=dev)
        ch = torch.randperm(K, generator=gen, device=dev)[:a.outliers]
        x[:, ch] *= 50.0
        x = x.to(torch.bfloat16)
        W = (torch.randn((N, K), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        col = sq.weight_column_max([x])
        mask, idx, count = sq.llmint8_outliers(col, 6.0)
        acc = torch.randint(-2 ** 20, 2 ** 20, (M, N), generator=gen, device=dev,
                            dtype=torch.int32)
        xs = torch.empty(M, device=dev).uniform_(1e-3, 1e-2, generator=gen)
        wsc = torch.empty(N, device=dev).uniform_(1e-4, 1e-3, generator=gen)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fn = lambda: sq.llmint8_combine(acc, xs, wsc, x, W, idx, count, "bf16", out=out)
        units = M * N * (4 + 2) + 4 * (M + N)
        shape = {"M": M, "N": N, "K": K, "outliers": int(count.item())}
    elif a.op == "calibrate":
        x = _acts(M, K, a.dtype, gen, dev)
        g = torch.empty(K, device=dev).uniform_(0.5, 1.5, generator=gen) if norm else None
        b = torch.randn(K, generator=gen, device=dev) * 0.1 if norm == sq.NORM_LAYER else None
        am = torch.zeros(K, dtype=torch.float32, device=dev)
        # the running max starts from zero every call, as in a calibration pass
        fn = lambda: (am.zero_(), sq.calibrate_absmax(x, norm, g, b, 1e-5, act_max=am))
        units = M * K * esz + 4 * K
        shape = {"M": M, "K": K, "norm": a.norm, "dtype": a.dtype}
    elif a.op == "weight_quant":
        W = (torch.randn((N, K), generator=gen, device=dev) * 0.02)
        W = W.to(torch.bfloat16) if a.dtype == "bf16" else W
        s = torch.empty(K, device=dev).uniform_(0.25, 4.0, generator=gen)
        wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        wsc = torch.empty(N, dtype=torch.float32, device=dev)
        fn = lambda: sq.smooth_quantize_weights(W, s, Wq=wq, w_scale=wsc)
        units = N * K * (esz + 1) + 4 * N + 4 * K
        shape = {"N": N, "K": K, "dtype": a.dtype}
    elif a.op == "smooth_scales":
        W = (torch.randn((N, K), generator=gen, device=dev) * 0.02)
        W = W.to(torch.bfloat16) if a.dtype == "bf16" else W
        am = torch.empty(K, device=dev).uniform_(0.1, 60.0, generator=gen)
        g = torch.empty(K, device=dev).uniform_(0.5, 1.5, generator=gen)
        s = torch.empty(K, dtype=torch.float32, device=dev)
        gf = torch.empty(K, dtype=torch.float32, device=dev)
        fn = lambda: sq.compute_smooth_scales(am, [W], 0.5, 1e-5, g, None, s=s, gamma_folded=gf)
        units = N * K * esz + 16 * K
        shape = {"N": N, "K": K, "dtype": a.dtype}
    else:
        A, B = _codes(M, K, gen, dev), _codes(N, K, gen, dev)
        xs = torch.empty(M, device=dev).uniform_(1e-3, 1e-2, generator=gen)
        wsc = torch.empty(N, device=dev).uniform_(1e-4, 1e-3, generator=gen)
        out = torch.empty((M, N), dtype=torch.int32 if a.epi == "i32" else torch.bfloat16,
                          device=dev)
        need = sq.gemm_workspace_size(M, N, K, a.split)
        ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
        scales = (None, None) if a.epi == "i32" else (xs, wsc)
        fn = lambda: sq.w8a8_gemm_dequant(A, B, scales[0], scales[1], a.epi, out=out,
                                          path_hint=a.path, split_k=a.split, workspace=ws)
        if a.fp8:
            A8, B8 = A.view(torch.uint8) & 0x77, B.view(torch.uint8) & 0xf7  # finite e4m3 codes
            fn = lambda: sq.fp8_gemm_dequant(A8, B8, scales[0], scales[1],
                                             "f32" if a.epi == "i32" else a.epi,
                                             out=out.view(torch.float32) if a.epi == "i32" else out,
                                             path_hint=a.path, workspace=ws)
        if a.rowmax:
            rm = torch.empty(M, dtype=torch.float32, device=dev)
            fn = lambda: sq.w8a8_gemm_dequant_rowmax(A, B, xs, wsc, a.epi, out=out,
                                                     row_absmax=rm, path_hint=a.path)
        shape = {"M": M, "N": N, "K": K, "path": a.path, "split": a.split, "epi": a.epi,
                 "rowmax": a.rowmax, "fp8": a.fp8}
        units = None
    us = _time(fn, a.iters, a.warmup, flush)
    err = sq.get_device_error()
    if err:
        raise SystemExit("device error: %s" % sq.status_string(err))
    line = {"op": a.op, "shape": shape, "us_per_call": us, "iters": a.iters,
            "l2": "emptied before every call, clean (untimed)", "peak_source": src}
    if a.op == "gemm" and M > 128:
        ops = 2.0 * M * N * K
        line.update(achieved=ops / us / 1e6, unit="TOPS", peak=bf16 * INT8_PER_BF16,
                    algorithmic_ops=ops)
    else:
        if units is None:
            osz = 4 if a.epi == "i32" else 2
            units = M * K + N * K + 4 * M + 4 * N + osz * M * N
        line.update(achieved=units / us / 1e3, unit="GB/s", peak=hbm, algorithmic_bytes=units)
    line["frac"] = line["achieved"] / line["peak"]
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
