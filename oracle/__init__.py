"""CPU parity oracle for the SmoothQuant W8A8 linear layer (test infrastructure).

This package is TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.  The
product (the CUDA library and its Python binding) never imports, links or calls
anything here, and nothing here imports the product.

The arithmetic lives in ``oracle.c`` (plain C, one IEEE rounding per operator,
compiled without fast-math or FMA contraction).  This module only marshals
numpy arrays through ctypes.  Array conventions:

* ``float32`` arrays are fp32 data; ``uint16`` arrays are bf16 bit patterns.
* Weights are nn.Linear shaped ``[N, K]`` (row n = output channel, K = input
  channel), activations ``[M, K]`` (row m = token).
* Norm codes: ``NORM_NONE = 0``, ``NORM_RMS = 1``, ``NORM_LAYER = 2``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

NORM_NONE = 0
NORM_RMS = 1
NORM_LAYER = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GCC_FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", "-std=gnu11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _declare(L):
    L.oracle_exact_sum.restype = ctypes.c_double
    L.oracle_exact_sum.argtypes = [_P, _I64]
    L.oracle_norm.restype = ctypes.c_int
    L.oracle_norm.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int, _P, _P,
                              ctypes.c_float, _P, _P, _P]
    L.oracle_quantize_rows.restype = None
    L.oracle_quantize_rows.argtypes = [_P, _I64, _I64, _P, _P]
    L.oracle_calibrate_absmax.restype = ctypes.c_int
    L.oracle_calibrate_absmax.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int,
                                          _P, _P, ctypes.c_float, _P]
    L.oracle_smooth_scales.restype = ctypes.c_int
    L.oracle_smooth_scales.argtypes = [_P, _P, _P, ctypes.c_int, ctypes.c_int, _I64,
                                       ctypes.c_double, ctypes.c_float, _P, _P]
    L.oracle_fold_norm.restype = None
    L.oracle_fold_norm.argtypes = [_P, _P, _P, _I64, _P, _P]
    L.oracle_smooth_weights.restype = None
    L.oracle_smooth_weights.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P]
    L.oracle_llmint8_outliers.restype = _I64
    L.oracle_llmint8_outliers.argtypes = [_P, _I64, ctypes.c_float, _P, _P]
    L.oracle_llmint8_combine.restype = None
    L.oracle_llmint8_combine.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, _I64, _P, ctypes.c_int,
                                         _I64, _P, _I64, ctypes.c_int, _P, _P]
    L.oracle_gemm_i64.restype = None
    L.oracle_gemm_i64.argtypes = [_P, _P, _I64, _I64, _I64, _P]
    L.oracle_epilogue.restype = None
    L.oracle_epilogue.argtypes = [_P, _P, _P, _I64, _I64, ctypes.c_int, _P, _P]
    L.oracle_f32_to_bf16_bits.restype = ctypes.c_uint16
    L.oracle_f32_to_bf16_bits.argtypes = [ctypes.c_float]
    L.oracle_row_sums.restype = None
    L.oracle_row_sums.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P]
    L.oracle_absmax_all.restype = None
    L.oracle_absmax_all.argtypes = [_P, _I64, _I64, _P]
    L.oracle_step_of.restype = ctypes.c_float
    L.oracle_step_of.argtypes = [ctypes.c_float]
    L.oracle_quantize_with_step.restype = None
    L.oracle_quantize_with_step.argtypes = [_P, _I64, _I64, ctypes.c_float, _P]
    L.oracle_exp_cw.restype = None
    L.oracle_exp_cw.argtypes = [_P, _I64, _P]
    L.oracle_silu_mul.restype = None
    L.oracle_silu_mul.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P]
    L.oracle_e4m3_to_f32.restype = ctypes.c_float
    L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    L.oracle_quantize_rows_fp8.restype = None
    L.oracle_quantize_rows_fp8.argtypes = [_P, _I64, _I64, _P, _P]
    L.oracle_gemm_fp8.restype = None
    L.oracle_gemm_fp8.argtypes = [_P, _P, _I64, _I64, _I64, _P]
    L.oracle_epilogue_f32.restype = None
    L.oracle_epilogue_f32.argtypes = [_P, _P, _P, _I64, _I64, ctypes.c_int, _P, _P]
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_num_threads.argtypes = []


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError("oracle inputs are float32 or bf16 bit patterns (uint16), got %s" % a.dtype)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def exact_sum(x) -> float:
    """Correctly rounded fp64 value of the exact sum of fp64 terms."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    return float(lib().oracle_exact_sum(_ptr(x), x.size))


def norm(x: np.ndarray, norm_kind: int, gamma=None, beta=None, eps: float = 1e-5):
    """Step 4: returns (y fp32 [M,K], mu fp32 [M], r fp32 [M])."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    y = np.empty((M, K), np.float32)
    mu = np.empty(M, np.float32)
    r = np.empty(M, np.float32)
    gamma, beta = _f32(gamma), _f32(beta)
    rc = lib().oracle_norm(_ptr(x), _dtype_code(x), M, K, K, norm_kind, _ptr(gamma), _ptr(beta),
                           eps, _ptr(y), _ptr(mu), _ptr(r))
    if rc != 0:
        raise ValueError("oracle_norm rejected its arguments (%d)" % rc)
    return y, mu, r


def row_sums(x: np.ndarray):
    """Exact per-row (sum x, sum x^2, sum |x|), each rounded once to fp64."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    S1, S2, SA = (np.empty(M, np.float64) for _ in range(3))
    lib().oracle_row_sums(_ptr(x), _dtype_code(x), M, K, K, _ptr(S1), _ptr(S2), _ptr(SA))
    return S1, S2, SA


def quantize_rows(y: np.ndarray):
    """Steps 5/6: per-row symmetric absmax INT8.  Returns (q int8, step fp32)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    q = np.empty((M, K), np.int8)
    step = np.empty(M, np.float32)
    lib().oracle_quantize_rows(_ptr(y), M, K, _ptr(q), _ptr(step))
    return q, step


def absmax_all(y: np.ndarray, absmax: float = 0.0) -> np.float32:
    """Per-tensor variants: running max of |y| over every element."""
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, y.shape[-1] if y.ndim else 1)
    M, K = y.shape
    am = np.array([absmax], np.float32)
    lib().oracle_absmax_all(_ptr(y), M, K, _ptr(am))
    return am[0]


def step_of(absmax) -> np.float32:
    """fl32(absmax / 127)."""
    return np.float32(lib().oracle_step_of(float(np.float32(absmax))))


def quantize_with_step(y: np.ndarray, step) -> np.ndarray:
    """Every element with one step: clamp(rne(fl32(y / step)), +-127)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    q = np.empty((M, K), np.int8)
    lib().oracle_quantize_with_step(_ptr(y), M, K, float(np.float32(step)), _ptr(q))
    return q


def quantize_tensor(y: np.ndarray):
    """O2 on a tensor (or per-tensor weights): (q int8, step fp32)."""
    step = step_of(absmax_all(y))
    return quantize_with_step(y, step), step


def norm_quant_per_tensor(x, norm_kind, gamma_f=None, beta_f=None, eps=1e-5, absmax=None):
    """Steps 4+5 with one activation scale for the whole tensor: O2 (``absmax``
    None: the tensor's own max |y|) or O3 (``absmax`` given: the calibrated
    static max; larger values saturate).  Returns (Xq, step)."""
    y, _, _ = norm(x, norm_kind, gamma_f, beta_f, eps)
    am = absmax_all(y) if absmax is None else np.float32(absmax)
    step = step_of(am)
    return quantize_with_step(y, step), step


def norm_quant(x, norm_kind, gamma_f=None, beta_f=None, eps=1e-5):
    """Steps 4+5 (the runtime activation path): returns (Xq, x_scale)."""
    y, _, _ = norm(x, norm_kind, gamma_f, beta_f, eps)
    return quantize_rows(y)


def calibrate_absmax(x, norm_kind, gamma=None, beta=None, eps=1e-5, act_max=None):
    """Step 1: running per-channel max |norm(x)|.  ``act_max`` is updated in place."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    if act_max is None:
        act_max = np.zeros(K, np.float32)
    assert act_max.dtype == np.float32 and act_max.shape == (K,)
    gamma, beta = _f32(gamma), _f32(beta)
    rc = lib().oracle_calibrate_absmax(_ptr(x), _dtype_code(x), M, K, K, norm_kind, _ptr(gamma),
                                       _ptr(beta), eps, _ptr(act_max))
    if rc != 0:
        raise ValueError("oracle_calibrate_absmax failed (%d)" % rc)
    return act_max


def smooth_scales(act_max, weights, alpha, eps=1e-5):
    """Step 2: s (fp32) and its fp64 value before rounding, for a list of
    weights [N_l, K] that read the same norm (all of one dtype)."""
    act_max = _f32(act_max)
    ws = [np.ascontiguousarray(w) for w in weights]
    K = act_max.shape[0]
    code = _dtype_code(ws[0])
    for w in ws:
        assert w.shape[1] == K and _dtype_code(w) == code
    ptrs = (ctypes.c_void_p * len(ws))(*[w.ctypes.data for w in ws])
    ns = (ctypes.c_int64 * len(ws))(*[w.shape[0] for w in ws])
    s = np.empty(K, np.float32)
    s64 = np.empty(K, np.float64)
    rc = lib().oracle_smooth_scales(_ptr(act_max), ctypes.cast(ptrs, ctypes.c_void_p),
                                    ctypes.cast(ns, ctypes.c_void_p), len(ws), code, K,
                                    float(alpha), eps, _ptr(s), _ptr(s64))
    if rc != 0:
        raise ValueError("oracle_smooth_scales failed (%d)" % rc)
    return s, s64


def fold_norm(s, gamma=None, beta=None):
    """Step 3 (norm side): gamma' = gamma/s, beta' = beta/s (fp32)."""
    s = _f32(s)
    K = s.shape[0]
    gamma, beta = _f32(gamma), _f32(beta)
    gf = np.empty(K, np.float32)
    bf = np.empty(K, np.float32) if beta is not None else None
    lib().oracle_fold_norm(_ptr(s), _ptr(gamma), _ptr(beta), K, _ptr(gf), _ptr(bf))
    return gf, bf


def smooth_weights(W, s=None):
    """Step 3 (weight side): W-hat = W * s per input column, fp32."""
    W = np.ascontiguousarray(W)
    N, K = W.shape
    out = np.empty((N, K), np.float32)
    lib().oracle_smooth_weights(_ptr(W), _dtype_code(W), N, K, K, _ptr(_f32(s)), _ptr(out))
    return out


def quantize_weights(W, s=None):
    """Steps 3+6: (Wq int8 [N,K], w_scale fp32 [N])."""
    return quantize_rows(smooth_weights(W, s))


def quantize_weights_per_tensor(W, s=None):
    """Steps 3+6 with one weight scale for the whole matrix (the paper's
    O1-O3 weights): (Wq int8 [N,K], step fp32)."""
    return quantize_tensor(smooth_weights(W, s))


def gemm_i64(Xq, Wq):
    """Step 7: exact int64 acc[m,n] = sum_k Xq[m,k] * Wq[n,k]."""
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    M, K = Xq.shape
    N, K2 = Wq.shape
    assert K == K2
    acc = np.empty((M, N), np.int64)
    lib().oracle_gemm_i64(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc))
    return acc


def epilogue(acc, x_scale, w_scale, relu=False):
    """Step 8: (o32 fp32 [M,N], out bf16 bits uint16 [M,N])."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    M, N = acc.shape
    xs, ws = _f32(x_scale), _f32(w_scale)
    o32 = np.empty((M, N), np.float32)
    out = np.empty((M, N), np.uint16)
    lib().oracle_epilogue(_ptr(acc), _ptr(xs), _ptr(ws), M, N, int(bool(relu)), _ptr(o32), _ptr(out))
    return o32, out


def f32_to_bf16_bits(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    f = lib().oracle_f32_to_bf16_bits
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def exp_cw(t) -> np.ndarray:
    """e^t by Cody-Waite reduction and a degree-7 Taylor polynomial in fp32
    (the exponential of the SiLU step; see oracle.c)."""
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty_like(t)
    lib().oracle_exp_cw(_ptr(t), t.size, _ptr(out))
    return out


def silu_mul(gu):
    """The down projection's input from gate_up's output [M, 2I] (gate in the
    first I columns, up in the last I): h = SiLU(gate) * up in fp32, and h
    rounded to bf16.  Returns (h32 fp32 [M, I], h bf16 bits uint16 [M, I])."""
    gu = np.ascontiguousarray(gu)
    M, K2 = gu.shape
    if K2 % 2:
        raise ValueError("gate_up rows hold two halves")
    I = K2 // 2
    h32 = np.empty((M, I), np.float32)
    hb = np.empty((M, I), np.uint16)
    lib().oracle_silu_mul(_ptr(gu), _dtype_code(gu), M, I, K2, _ptr(h32), _ptr(hb))
    return h32, hb


def silu_mul_quant(gu):
    """SiLU(gate) * up stored as bf16, then per-token quantised (steps 5 on
    h, no norm).  Returns (Xq int8 [M, I], x_scale fp32 [M], h bf16 bits)."""
    _, hb = silu_mul(gu)
    Xq, xs = norm_quant(hb, NORM_NONE)
    return Xq, xs, hb


# ---- FP8 (e4m3) W8A8 (see oracle.c for the readings) ----------------------

def e4m3_decode(codes) -> np.ndarray:
    """Values of e4m3 codes (uint8) as fp32."""
    c = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_e4m3_to_f32
    table = np.array([f(i) for i in range(256)], dtype=np.float32)
    return table[c]


def e4m3_encode(x) -> np.ndarray:
    """fp32 -> e4m3 codes, nearest-even, saturating at +-448."""
    x = np.asarray(x, dtype=np.float32)
    f = lib().oracle_f32_to_e4m3
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def quantize_rows_fp8(y: np.ndarray):
    """Per-row FP8: step = fl32(max|y| / 448), code = e4m3(fl32(y * fl32(1/step))).
    Returns (q uint8 [M, K], step fp32 [M])."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    q = np.empty((M, K), np.uint8)
    step = np.empty(M, np.float32)
    lib().oracle_quantize_rows_fp8(_ptr(y), M, K, _ptr(q), _ptr(step))
    return q, step


def norm_quant_fp8(x, norm_kind, gamma_f=None, beta_f=None, eps=1e-5):
    """The norm (step 4) then per-token FP8 codes.  Returns (Xq8, x_scale)."""
    y, _, _ = norm(x, norm_kind, gamma_f, beta_f, eps)
    return quantize_rows_fp8(y)


def quantize_weights_fp8(W, s=None):
    """W-hat = fl32(W * s) per output channel in FP8.  Returns (Wq8, w_scale)."""
    return quantize_rows_fp8(smooth_weights(W, s))


def gemm_fp8(Xq8, Wq8) -> np.ndarray:
    """Exact sum of the decoded products, fp64 [M, N]."""
    Xq8 = np.ascontiguousarray(Xq8, dtype=np.uint8)
    Wq8 = np.ascontiguousarray(Wq8, dtype=np.uint8)
    M, K = Xq8.shape
    N = Wq8.shape[0]
    if K > (1 << 17):
        raise ValueError("the fp64 sum is exact for K <= 2^17")
    acc = np.empty((M, N), np.float64)
    lib().oracle_gemm_fp8(_ptr(Xq8), _ptr(Wq8), M, N, K, _ptr(acc))
    return acc


def epilogue_f32(acc32, x_scale, w_scale, relu=False):
    """Epilogue from an fp32 accumulator: (o32 [M, N], out bf16 bits [M, N])."""
    acc32 = np.ascontiguousarray(acc32, dtype=np.float32)
    M, N = acc32.shape
    xs, ws = _f32(x_scale), _f32(w_scale)
    o32 = np.empty((M, N), np.float32)
    out = np.empty((M, N), np.uint16)
    lib().oracle_epilogue_f32(_ptr(acc32), _ptr(xs), _ptr(ws), M, N, int(bool(relu)), _ptr(o32),
                              _ptr(out))
    return o32, out


def linear(x, norm_kind, gamma_f, beta_f, eps, Wq, w_scale, relu=False):
    """The whole runtime path: norm+quant, integer GEMM, epilogue.
    Returns (Xq, x_scale, acc, o32, out_bf16_bits)."""
    Xq, xs = norm_quant(x, norm_kind, gamma_f, beta_f, eps)
    acc = gemm_i64(Xq, Wq)
    o32, out = epilogue(acc, xs, w_scale, relu)
    return Xq, xs, acc, o32, out


# --------------------------------------------------------------------------
# Comparator: LLM.int8()'s mixed-precision decomposition
# --------------------------------------------------------------------------

def llmint8_outliers(col_absmax, tau: float = 6.0):
    """(mask [K] fp32: 0 on outlier channels, idx: the outlier channels
    ascending) for O = {j : col_absmax[j] >= tau}."""
    col = _f32(col_absmax)
    K = col.shape[0]
    mask = np.empty(K, np.float32)
    idx = np.empty(K, np.int32)
    n = lib().oracle_llmint8_outliers(_ptr(col), K, float(np.float32(tau)), _ptr(mask), _ptr(idx))
    return mask, idx[:n].copy()


def llmint8_combine(o32, x, W, idx, relu=False):
    """(y fp32 [M,N], out bf16 bits): the INT8 lane's o32 plus the 16-bit lane
    over the channels idx (fp64 accumulation, ascending), one fp32 add."""
    o32 = np.ascontiguousarray(o32, dtype=np.float32)
    x = np.ascontiguousarray(x)
    W = np.ascontiguousarray(W)
    M, N = o32.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    y = np.empty((M, N), np.float32)
    out = np.empty((M, N), np.uint16)
    lib().oracle_llmint8_combine(_ptr(o32), M, N, _ptr(x), _dtype_code(x), x.shape[1], _ptr(W),
                                 _dtype_code(W), W.shape[1], _ptr(idx), idx.shape[0],
                                 int(bool(relu)), _ptr(y), _ptr(out))
    return y, out


def llmint8_linear(x, Wq, w_scale, W, tau: float = 6.0, relu: bool = False):
    """The comparator layer end to end ([LLMint8] "Fix 1", "going deeper"):
    outlier channels from this batch's column maxima, per-token INT8 codes of
    the other channels, the INT8 GEMM and its epilogue, the 16-bit lane and
    the sum.  Wq / w_scale: W quantised per output channel (quantize_weights
    with no smoothing).  Returns a dict of every stage."""
    col = calibrate_absmax(x, NORM_NONE)
    mask, idx = llmint8_outliers(col, tau)
    Xq, xs = norm_quant(x, NORM_NONE, mask, None)
    acc = gemm_i64(Xq, Wq)
    o32, _ = epilogue(acc, xs, w_scale, False)
    y, out = llmint8_combine(o32, x, W, idx, relu)
    return {"col_absmax": col, "mask": mask, "idx": idx, "Xq": Xq, "x_scale": xs, "acc": acc,
            "o32": o32, "y": y, "out": out}
