"""Thin Python binding of ``libsq.so`` (include/sq.h).

Argument marshalling only: every call checks the tensors it is given, turns
them into device pointers and sizes, and calls the C ABI on the current torch
CUDA stream.  Output tensors are allocated here with torch when the caller
does not pass them; the library itself never allocates.  There is no CPU or
PyTorch fallback: if the library is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

from . import build as _build

SQ_OK = 0
STATUS_NAMES = {
    0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED", 3: "SQ_ERR_ALIGNMENT",
    4: "SQ_ERR_OVERFLOW_RISK", 5: "SQ_ERR_CUDA", 6: "SQ_ERR_PIPELINE_TIMEOUT",
    7: "SQ_ERR_WORKSPACE",
}
SQ_F32, SQ_BF16 = 0, 1
NORM_NONE, NORM_RMS, NORM_LAYER = 0, 1, 2
EPI = {"bf16": 0, "bf16_relu": 1, "i32": 2, "f32": 3}
MAX_K = 133144

# Every symbol include/sq.h declares.
EXPORTS = (
    "sq_calibrate_absmax", "sq_compute_smooth_scales", "sq_smooth_quantize_weights",
    "sq_norm_smooth_quant_per_token", "sq_w8a8_gemm_workspace_size", "sq_w8a8_gemm_dequant",
    "sq_linear_w8a8", "sq_status_string", "sq_get_device_error", "sq_set_wait_limit",
    "sq_w8a8_gemm_dequant_noalloc", "sq_w8a8_gemm_plan", "sq_norm_smooth_absmax",
    "sq_norm_smooth_quant_per_tensor", "sq_smooth_quantize_weights_per_tensor",
    "sq_w8a8_gemm_dequant_rowmax", "sq_quant_per_token_given_absmax",
    "sq_silu_mul_quant_per_token", "sq_norm_smooth_quant_per_token_fp8",
    "sq_smooth_quantize_weights_fp8", "sq_fp8_gemm_dequant", "sq_weight_column_max",
    "sq_smooth_scales_from_maxima", "sq_silu_mul_quant_per_token_fp8", "sq_row_absmax",
    "sq_dequant_i32", "sq_llmint8_outliers", "sq_llmint8_combine",
)
LLMINT8_MAX_K = 1 << 20
NOALLOC_SCRATCH_BYTES = 8 << 20


class GemmPlanInfo(ctypes.Structure):
    """sq_gemm_plan_info: what sq_w8a8_gemm_dequant runs for a shape."""
    _fields_ = [("kernel", ctypes.c_int), ("tile_m", ctypes.c_int), ("tile_n", ctypes.c_int),
                ("split_k", ctypes.c_int), ("stream_k", ctypes.c_int), ("ctas", ctypes.c_int),
                ("launches", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t)]

    KERNELS = ("w8a8_gemm_kernel", "w8a8_gemm_pair_kernel", "w8a8_gemm_kernel (decode tiles)")

    def as_dict(self):
        d = {f: getattr(self, f) for f, _ in self._fields_}
        d["kernel_name"] = self.KERNELS[self.kernel]
        return d


class SQError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__("%s failed: %s" % (call, _status_text(status)))


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load libsq.so (built in-tree); raises if it is not there."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError("libsq.so is not built (%s); run python -m "
                               "w8a8_int8_quantized_norm_b200.build" % path)
        L = ctypes.CDLL(path)
        _declare(L)
        _lib = L
    return _lib


_P, _I64, _I32, _F32, _F64, _SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                   ctypes.c_double, ctypes.c_size_t)


def _declare(L):
    L.sq_calibrate_absmax.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _F32, _P, _P]
    L.sq_compute_smooth_scales.argtypes = [_P, _P, _P, _I32, _I32, _I64, _F64, _F32, _P, _P, _P,
                                           _P, _P, _P]
    L.sq_smooth_quantize_weights.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]
    L.sq_norm_smooth_quant_per_token.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _F32,
                                                 _P, _P, _P]
    L.sq_w8a8_gemm_workspace_size.argtypes = [_I64, _I64, _I64, _I32]
    L.sq_w8a8_gemm_workspace_size.restype = _SZ
    L.sq_w8a8_gemm_dequant.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I64, _P, _SZ,
                                       _I32, _I32, _P]
    L.sq_w8a8_gemm_dequant_noalloc.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I64,
                                               _I32, _I32, _P]
    L.sq_linear_w8a8.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _F32, _P, _P, _I64,
                                 _I32, _P, _I64, _P, _P, _P, _SZ, _P]
    L.sq_status_string.argtypes = [_I32]
    L.sq_status_string.restype = ctypes.c_char_p
    L.sq_get_device_error.argtypes = [_P]
    L.sq_norm_smooth_absmax.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _F32, _P, _P]
    L.sq_norm_smooth_quant_per_tensor.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P, _F32,
                                                  _P, _P, _P, _P]
    L.sq_smooth_quantize_weights_per_tensor.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P,
                                                        _P, _P]
    L.sq_w8a8_gemm_dequant_rowmax.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I64,
                                              _P, _I32, _P]
    L.sq_quant_per_token_given_absmax.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]
    L.sq_row_absmax.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P]
    L.sq_llmint8_outliers.argtypes = [_P, _I64, _F32, _P, _P, _P, _P]
    L.sq_llmint8_combine.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _I64, _P, _I32,
                                     _I64, _I64, _P, _P, _I32, _P, _I64, _P]
    L.sq_dequant_i32.argtypes = [_P, _I64, _I64, _I64, _P, _P, _I32, _P, _I64, _P]
    L.sq_silu_mul_quant_per_token.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _I64, _P]
    L.sq_norm_smooth_quant_per_token_fp8.argtypes = [_P, _I32, _I64, _I64, _I64, _I32, _P, _P,
                                                     _F32, _P, _P, _P]
    L.sq_smooth_quantize_weights_fp8.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]
    L.sq_fp8_gemm_dequant.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _P, _I64, _P, _SZ,
                                      _I32, _P]
    L.sq_silu_mul_quant_per_token_fp8.argtypes = [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _I64,
                                                  _P]
    L.sq_weight_column_max.argtypes = [_P, _P, _I32, _I32, _I64, _P, _P]
    L.sq_smooth_scales_from_maxima.argtypes = [_P, _P, _I64, _F64, _F32, _P, _P, _P, _P, _P, _P]
    L.sq_w8a8_gemm_plan.argtypes = [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(GemmPlanInfo)]
    L.sq_set_wait_limit.argtypes = [_I64]
    L.sq_set_wait_limit.restype = None
    for name in EXPORTS:
        f = getattr(L, name)
        if f.argtypes is None:  # every call passes 64-bit sizes: no implicit int conversion
            raise RuntimeError("no argument types declared for %s" % name)
        if name not in ("sq_w8a8_gemm_workspace_size", "sq_status_string", "sq_set_wait_limit"):
            f.restype = _I32


def _status_text(status: int) -> str:
    try:
        return lib().sq_status_string(status).decode()
    except Exception:  # the library may be what failed to load
        return STATUS_NAMES.get(status, str(status))


def _check(status: int, call: str):
    if status != SQ_OK:
        raise SQError(status, call)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    if t.dtype == torch.float32:
        return SQ_F32
    raise TypeError("activations and weights are bf16 or fp32, got %s" % t.dtype)


def _rows(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dim() != 2 or (t.stride(1) != 1 and t.shape[1] > 1):
        raise ValueError("%s must be 2-D with unit column stride" % name)
    # a single row's stride is arbitrary (numpy / torch may report 0 for it)
    ld = t.stride(0) if t.shape[0] > 1 else t.shape[1]
    return t.shape[0], t.shape[1], ld


def _vec(t: Optional[torch.Tensor], K: int, name: str):
    if t is None:
        return None
    if not (t.is_cuda and t.dtype == torch.float32 and t.dim() == 1 and t.numel() == K
            and t.is_contiguous()):
        raise ValueError("%s must be a contiguous fp32 CUDA vector of length %d" % (name, K))
    return t


# ---------------------------------------------------------------------------
# the six calls of the C ABI
# ---------------------------------------------------------------------------

def calibrate_absmax(x: torch.Tensor, norm: int, gamma=None, beta=None, eps: float = 1e-5,
                     act_max: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K, ld = _rows(x, "x")
    if act_max is None:
        act_max = torch.zeros(K, dtype=torch.float32, device=x.device)
    _vec(act_max, K, "act_max")
    _check(lib().sq_calibrate_absmax(_ptr(x), _dtype_code(x), M, K, ld, norm,
                                     _ptr(_vec(gamma, K, "gamma")), _ptr(_vec(beta, K, "beta")),
                                     eps, _ptr(act_max), _stream(stream)), "sq_calibrate_absmax")
    return act_max


def compute_smooth_scales(act_max: torch.Tensor, weights: Sequence[torch.Tensor], alpha: float,
                          clamp_eps: float = 1e-5, gamma=None, beta=None, s=None,
                          gamma_folded=None, beta_folded=None, stream=None
                          ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    K = act_max.numel()
    _vec(act_max, K, "act_max")
    dt = _dtype_code(weights[0])
    for w in weights:
        _rows(w, "W")
        if not w.is_contiguous() or w.shape[1] != K or _dtype_code(w) != dt:
            raise ValueError("weights must be contiguous [N, K] of one dtype")
    ptrs = (ctypes.c_void_p * len(weights))(*[w.data_ptr() for w in weights])
    ns = (ctypes.c_int64 * len(weights))(*[w.shape[0] for w in weights])
    dev = act_max.device
    s = torch.empty(K, dtype=torch.float32, device=dev) if s is None else _vec(s, K, "s")
    gf = (torch.empty(K, dtype=torch.float32, device=dev) if gamma_folded is None
          else _vec(gamma_folded, K, "gamma_folded"))
    bf = None
    if beta is not None:
        bf = (torch.empty(K, dtype=torch.float32, device=dev) if beta_folded is None
              else _vec(beta_folded, K, "beta_folded"))
    _check(lib().sq_compute_smooth_scales(_ptr(act_max), ctypes.cast(ptrs, ctypes.c_void_p),
                                          ctypes.cast(ns, ctypes.c_void_p), len(weights), dt, K,
                                          float(alpha), clamp_eps, _ptr(_vec(gamma, K, "gamma")),
                                          _ptr(_vec(beta, K, "beta")), _ptr(s), _ptr(gf), _ptr(bf),
                                          _stream(stream)), "sq_compute_smooth_scales")
    return s, gf, bf


def weight_column_max(weights: Sequence[torch.Tensor], w_max=None, stream=None) -> torch.Tensor:
    """max over the weights and their rows of |W[n, j]|, per input column j."""
    K = weights[0].shape[1]
    dt = _dtype_code(weights[0])
    for w in weights:
        _rows(w, "W")
        if not w.is_contiguous() or w.shape[1] != K or _dtype_code(w) != dt:
            raise ValueError("weights must be contiguous [N, K] of one dtype")
    ptrs = (ctypes.c_void_p * len(weights))(*[w.data_ptr() for w in weights])
    ns = (ctypes.c_int64 * len(weights))(*[w.shape[0] for w in weights])
    if w_max is None:
        w_max = torch.empty(K, dtype=torch.float32, device=weights[0].device)
    _check(lib().sq_weight_column_max(ctypes.cast(ptrs, ctypes.c_void_p),
                                      ctypes.cast(ns, ctypes.c_void_p), len(weights), dt, K,
                                      _ptr(_vec(w_max, K, "w_max")), _stream(stream)),
           "sq_weight_column_max")
    return w_max


def smooth_scales_from_maxima(act_max: torch.Tensor, w_max: torch.Tensor, alpha: float,
                              clamp_eps: float = 1e-5, gamma=None, beta=None, s=None,
                              gamma_folded=None, beta_folded=None, stream=None):
    """s, gamma / s and beta / s from the two maxima (s may be w_max)."""
    K = act_max.numel()
    dev = act_max.device
    s = torch.empty(K, dtype=torch.float32, device=dev) if s is None else s
    gf = torch.empty(K, dtype=torch.float32, device=dev) if gamma_folded is None else gamma_folded
    bf = None
    if beta is not None:
        bf = torch.empty(K, dtype=torch.float32, device=dev) if beta_folded is None else beta_folded
    _check(lib().sq_smooth_scales_from_maxima(
        _ptr(_vec(act_max, K, "act_max")), _ptr(_vec(w_max, K, "w_max")), K, float(alpha),
        clamp_eps, _ptr(_vec(gamma, K, "gamma")), _ptr(_vec(beta, K, "beta")),
        _ptr(_vec(s, K, "s")), _ptr(_vec(gf, K, "gamma_folded")),
        _ptr(_vec(bf, K, "beta_folded")), _stream(stream)), "sq_smooth_scales_from_maxima")
    return s, gf, bf


def smooth_quantize_weights(W: torch.Tensor, s: Optional[torch.Tensor] = None, Wq=None,
                            w_scale=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    N, K, ld = _rows(W, "W")
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(lib().sq_smooth_quantize_weights(_ptr(W), _dtype_code(W), N, K, ld,
                                            _ptr(_vec(s, K, "s")), _ptr(Wq), _ptr(w_scale),
                                            _stream(stream)), "sq_smooth_quantize_weights")
    return Wq, w_scale


def norm_smooth_quant_per_token(x: torch.Tensor, norm: int, gamma_folded=None, beta_folded=None,
                                eps: float = 1e-5, Xq=None, x_scale=None, stream=None
                                ) -> Tuple[torch.Tensor, torch.Tensor]:
    M, K, ld = _rows(x, "x")
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().sq_norm_smooth_quant_per_token(
        _ptr(x), _dtype_code(x), M, K, ld, norm, _ptr(_vec(gamma_folded, K, "gamma_folded")),
        _ptr(_vec(beta_folded, K, "beta_folded")), eps, _ptr(Xq), _ptr(x_scale), _stream(stream)),
        "sq_norm_smooth_quant_per_token")
    return Xq, x_scale


def norm_smooth_absmax(x: torch.Tensor, norm: int, gamma_folded=None, beta_folded=None,
                       eps: float = 1e-5, absmax=None, stream=None) -> torch.Tensor:
    """Running max over all of |norm(x)| into a 1-element fp32 device tensor."""
    M, K, ld = _rows(x, "x")
    if absmax is None:
        absmax = torch.zeros(1, dtype=torch.float32, device=x.device)
    _check(lib().sq_norm_smooth_absmax(_ptr(x), _dtype_code(x), M, K, ld, norm,
                                       _ptr(_vec(gamma_folded, K, "gamma_folded")),
                                       _ptr(_vec(beta_folded, K, "beta_folded")), eps,
                                       _ptr(absmax), _stream(stream)), "sq_norm_smooth_absmax")
    return absmax


def norm_smooth_quant_per_tensor(x: torch.Tensor, norm: int, absmax: torch.Tensor,
                                 gamma_folded=None, beta_folded=None, eps: float = 1e-5,
                                 Xq=None, x_scale=None, stream=None):
    """Codes with the one step fl32(absmax / 127); x_scale holds it per row."""
    M, K, ld = _rows(x, "x")
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().sq_norm_smooth_quant_per_tensor(
        _ptr(x), _dtype_code(x), M, K, ld, norm, _ptr(_vec(gamma_folded, K, "gamma_folded")),
        _ptr(_vec(beta_folded, K, "beta_folded")), eps, _ptr(absmax), _ptr(Xq), _ptr(x_scale),
        _stream(stream)), "sq_norm_smooth_quant_per_tensor")
    return Xq, x_scale


def quant_per_token_given_absmax(x: torch.Tensor, row_absmax: torch.Tensor, Xq=None,
                                 x_scale=None, stream=None):
    """Per-token codes of x [M, K] with each row's max |x| given (no norm)."""
    M, K, ld = _rows(x, "x")
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().sq_quant_per_token_given_absmax(
        _ptr(x), _dtype_code(x), M, K, ld, _ptr(_vec(row_absmax, M, "row_absmax")), _ptr(Xq),
        _ptr(x_scale), _stream(stream)), "sq_quant_per_token_given_absmax")
    return Xq, x_scale


def row_absmax(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """max_k |x[m, k]| per row of x [M, K] (no norm), fp32 [M]."""
    M, K, ld = _rows(x, "x")
    if out is None:
        out = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().sq_row_absmax(_ptr(x), _dtype_code(x), M, K, ld, _ptr(_vec(out, M, "out")),
                               _stream(stream)), "sq_row_absmax")
    return out


def dequant_i32(acc: torch.Tensor, x_scale: torch.Tensor, w_scale: torch.Tensor,
                epi: str = "bf16", out=None, stream=None) -> torch.Tensor:
    """The GEMM's epilogue on an INT32 accumulator acc [M, N]: bf16 [M, N]."""
    if acc.dim() != 2 or acc.dtype != torch.int32 or (acc.shape[1] > 1 and acc.stride(1) != 1):
        raise ValueError("acc must be an int32 [M, N] tensor with unit column stride")
    M, N = acc.shape
    if epi not in ("bf16", "bf16_relu"):
        raise ValueError("epi must be bf16 or bf16_relu")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=acc.device)
    if tuple(out.shape) != (M, N) or out.dtype != torch.bfloat16 or \
            (N > 1 and out.stride(1) != 1):
        raise ValueError("out must be a bf16 [M, N] tensor with unit column stride")
    _check(lib().sq_dequant_i32(_ptr(acc), M, N, max(acc.stride(0), N),
                                _ptr(_vec(x_scale, M, "x_scale")), _ptr(_vec(w_scale, N, "w_scale")),
                                EPI[epi], _ptr(out), max(out.stride(0), N), _stream(stream)),
           "sq_dequant_i32")
    return out


def llmint8_outliers(col_absmax: torch.Tensor, tau: float = 6.0, mask=None, idx=None, count=None,
                     stream=None):
    """(mask [K] fp32, idx [K] int32, count [1] int32) of the LLM.int8()
    comparator: mask 0 on the channels with col_absmax >= tau, idx[:count] those
    channels ascending (count stays on the device)."""
    K = col_absmax.numel()
    dev = col_absmax.device
    if mask is None:
        mask = torch.empty(K, dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty(K, dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=dev)
    if idx.dtype != torch.int32 or idx.numel() < K or count.dtype != torch.int32:
        raise ValueError("idx [K] and count [1] must be int32")
    _check(lib().sq_llmint8_outliers(_ptr(_vec(col_absmax, K, "col_absmax")), K, tau,
                                     _ptr(_vec(mask, K, "mask")), _ptr(idx), _ptr(count),
                                     _stream(stream)), "sq_llmint8_outliers")
    return mask, idx, count


def llmint8_combine(acc: torch.Tensor, x_scale, w_scale, x: torch.Tensor, W: torch.Tensor, idx,
                    count, epi: str = "bf16", out=None, stream=None) -> torch.Tensor:
    """The comparator's merge: the INT8 lane's epilogue plus the 16-bit lane
    over the outlier channels, bf16 [M, N]."""
    M, N = acc.shape
    _, K, ldx = _rows(x, "x")
    _, Kw, ldw = _rows(W, "W")
    if Kw != K or W.shape[0] != N or acc.dtype != torch.int32 or \
            (N > 1 and acc.stride(1) != 1):
        raise ValueError("acc [M, N] int32, x [M, K], W [N, K]")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=acc.device)
    _check(lib().sq_llmint8_combine(_ptr(acc), M, N, max(acc.stride(0), N),
                                    _ptr(_vec(x_scale, M, "x_scale")),
                                    _ptr(_vec(w_scale, N, "w_scale")), _ptr(x), _dtype_code(x),
                                    ldx, _ptr(W), _dtype_code(W), ldw, K, _ptr(idx), _ptr(count),
                                    EPI[epi], _ptr(out), max(out.stride(0), N), _stream(stream)),
           "sq_llmint8_combine")
    return out


def silu_mul_quant_per_token(gate_up: torch.Tensor, Xq=None, x_scale=None, h_out=None,
                             stream=None, fp8: bool = False):
    """Per-token codes of h = SiLU(gate) * up from gate_up [M, 2I] (gate in the
    first I columns): INT8, or with ``fp8`` e4m3 bytes (uint8).  ``h_out``
    (bf16 [M, I]) also receives h when given."""
    M, K2, ld = _rows(gate_up, "gate_up")
    if K2 % 2:
        raise ValueError("gate_up rows hold two halves")
    I = K2 // 2
    if Xq is None:
        Xq = torch.empty((M, I), dtype=torch.uint8 if fp8 else torch.int8, device=gate_up.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=gate_up.device)
    ldh = 0
    if h_out is not None:
        if h_out.dtype != torch.bfloat16 or tuple(h_out.shape) != (M, I):
            raise ValueError("h_out must be bf16 [M, I]")
        _, _, ldh = _rows(h_out, "h_out")
    call = "sq_silu_mul_quant_per_token_fp8" if fp8 else "sq_silu_mul_quant_per_token"
    _check(getattr(lib(), call)(_ptr(gate_up), _dtype_code(gate_up), M, I, ld, _ptr(Xq),
                                _ptr(x_scale), _ptr(h_out), ldh, _stream(stream)), call)
    return Xq, x_scale


# ---- FP8 (e4m3) W8A8: codes are uint8 tensors holding e4m3 bytes ----------

def norm_smooth_quant_per_token_fp8(x: torch.Tensor, norm: int, gamma_folded=None,
                                    beta_folded=None, eps: float = 1e-5, Xq8=None, x_scale=None,
                                    stream=None):
    M, K, ld = _rows(x, "x")
    if Xq8 is None:
        Xq8 = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().sq_norm_smooth_quant_per_token_fp8(
        _ptr(x), _dtype_code(x), M, K, ld, norm, _ptr(_vec(gamma_folded, K, "gamma_folded")),
        _ptr(_vec(beta_folded, K, "beta_folded")), eps, _ptr(Xq8), _ptr(x_scale),
        _stream(stream)), "sq_norm_smooth_quant_per_token_fp8")
    return Xq8, x_scale


def smooth_quantize_weights_fp8(W: torch.Tensor, s: Optional[torch.Tensor] = None, Wq8=None,
                                w_scale=None, stream=None):
    N, K, ld = _rows(W, "W")
    if Wq8 is None:
        Wq8 = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(lib().sq_smooth_quantize_weights_fp8(_ptr(W), _dtype_code(W), N, K, ld,
                                                _ptr(_vec(s, K, "s")), _ptr(Wq8), _ptr(w_scale),
                                                _stream(stream)), "sq_smooth_quantize_weights_fp8")
    return Wq8, w_scale


def fp8_gemm_dequant(Xq8: torch.Tensor, Wq8: torch.Tensor, x_scale: Optional[torch.Tensor],
                     w_scale: Optional[torch.Tensor], epi: str = "bf16", out=None,
                     path_hint: int = 0, workspace=None, whole_k: bool = False,
                     stream=None) -> torch.Tensor:
    """e4m3 GEMM with the dequant epilogue.  Decode tiles run stream-K with a
    workspace (allocated here when not given) unless ``whole_k``."""
    M, K = Xq8.shape
    N = Wq8.shape[0]
    if Xq8.dtype != torch.uint8 or Wq8.dtype != torch.uint8 or not Xq8.is_contiguous() \
            or not Wq8.is_contiguous() or Wq8.shape[1] != K:
        raise ValueError("Xq8 [M,K] and Wq8 [N,K] must be contiguous uint8 (e4m3 bytes)")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if epi == "f32" else torch.bfloat16,
                          device=Xq8.device)
    if whole_k:
        workspace = None
    else:
        need = gemm_workspace_size(M, N, K, 0) if path_hint != 1 and path_hint != 3 else 0
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=Xq8.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().sq_fp8_gemm_dequant(_ptr(Xq8), _ptr(Wq8), _ptr(x_scale), _ptr(w_scale), M, N, K,
                                     EPI[epi], _ptr(out), out.stride(0), _ptr(workspace), wsb,
                                     path_hint, _stream(stream)), "sq_fp8_gemm_dequant")
    return out


def smooth_quantize_weights_per_tensor(W: torch.Tensor, s: Optional[torch.Tensor] = None,
                                       Wq=None, w_scale=None, w_absmax=None, stream=None):
    N, K, ld = _rows(W, "W")
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    if w_absmax is None:
        w_absmax = torch.empty(1, dtype=torch.float32, device=W.device)
    _check(lib().sq_smooth_quantize_weights_per_tensor(
        _ptr(W), _dtype_code(W), N, K, ld, _ptr(_vec(s, K, "s")), _ptr(Wq), _ptr(w_scale),
        _ptr(w_absmax), _stream(stream)), "sq_smooth_quantize_weights_per_tensor")
    return Wq, w_scale


def gemm_plan(M: int, N: int, K: int, path_hint: int = 0, split_k: int = 0) -> GemmPlanInfo:
    info = GemmPlanInfo()
    _check(lib().sq_w8a8_gemm_plan(M, N, K, path_hint, split_k, ctypes.byref(info)),
           "sq_w8a8_gemm_plan")
    return info


def gemm_workspace_size(M: int, N: int, K: int, split_k: int = 0) -> int:
    return int(lib().sq_w8a8_gemm_workspace_size(M, N, K, split_k))


def w8a8_gemm_dequant(Xq: torch.Tensor, Wq: torch.Tensor, x_scale: Optional[torch.Tensor],
                      w_scale: Optional[torch.Tensor], epi: str = "bf16", out=None,
                      path_hint: int = 0, split_k: int = 0, workspace=None, stream=None
                      ) -> torch.Tensor:
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.int8 or Wq.dtype != torch.int8 or not Xq.is_contiguous() \
            or not Wq.is_contiguous() or Wq.shape[1] != K:
        raise ValueError("Xq [M,K] and Wq [N,K] must be contiguous int8")
    code = EPI[epi]
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if epi == "i32" else torch.bfloat16,
                          device=Xq.device)
    need = gemm_workspace_size(M, N, K, split_k)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=Xq.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().sq_w8a8_gemm_dequant(_ptr(Xq), _ptr(Wq), _ptr(x_scale), _ptr(w_scale), M, N, K,
                                      code, _ptr(out), out.stride(0), _ptr(workspace), wsb,
                                      path_hint, split_k, _stream(stream)),
           "sq_w8a8_gemm_dequant")
    return out


def w8a8_gemm_dequant_rowmax(Xq: torch.Tensor, Wq: torch.Tensor, x_scale: torch.Tensor,
                             w_scale: torch.Tensor, epi: str = "bf16", out=None,
                             row_absmax=None, path_hint: int = 0, stream=None):
    """The prefill GEMM that also returns max_n |out[m, n]| per row (bf16
    epilogues only).  Returns (out, row_absmax)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.int8 or Wq.dtype != torch.int8 or not Xq.is_contiguous() \
            or not Wq.is_contiguous() or Wq.shape[1] != K:
        raise ValueError("Xq [M,K] and Wq [N,K] must be contiguous int8")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    if row_absmax is None:
        row_absmax = torch.empty(M, dtype=torch.float32, device=Xq.device)
    _check(lib().sq_w8a8_gemm_dequant_rowmax(
        _ptr(Xq), _ptr(Wq), _ptr(x_scale), _ptr(w_scale), M, N, K, EPI[epi], _ptr(out),
        out.stride(0), _ptr(_vec(row_absmax, M, "row_absmax")), path_hint, _stream(stream)),
        "sq_w8a8_gemm_dequant_rowmax")
    return out, row_absmax


def w8a8_gemm_dequant_noalloc(Xq: torch.Tensor, Wq: torch.Tensor,
                              x_scale: Optional[torch.Tensor], w_scale: Optional[torch.Tensor],
                              out: torch.Tensor, epi: str = "bf16", path_hint: int = 0,
                              split_k: int = 0, stream=None) -> torch.Tensor:
    """The GEMM for callers that cannot allocate: the caller passes every input
    and the output; split-K scratch comes from the library's own fixed array
    (see include/sq.h).  Calls that overlap on the GPU share that array."""
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.int8 or Wq.dtype != torch.int8 or not Xq.is_contiguous() \
            or not Wq.is_contiguous() or Wq.shape[1] != K:
        raise ValueError("Xq [M,K] and Wq [N,K] must be contiguous int8")
    # the C ABI cannot see the output's extent: a wrong one would be written past
    want = torch.int32 if epi == "i32" else torch.bfloat16
    if (out.dim() != 2 or tuple(out.shape) != (M, N) or out.dtype != want
            or (N > 1 and out.stride(1) != 1) or out.stride(0) < N
            or out.device != Xq.device or Wq.device != Xq.device):
        raise ValueError("out must be a [M, N] = [%d, %d] %s tensor with unit column stride "
                         "on the device of Xq" % (M, N, want))
    _check(lib().sq_w8a8_gemm_dequant_noalloc(_ptr(Xq), _ptr(Wq), _ptr(x_scale), _ptr(w_scale),
                                              M, N, K, EPI[epi], _ptr(out), out.stride(0),
                                              path_hint, split_k, _stream(stream)),
           "sq_w8a8_gemm_dequant_noalloc")
    return out


def linear_w8a8(x: torch.Tensor, norm: int, gamma_folded, beta_folded, eps: float,
                Wq: torch.Tensor, w_scale: torch.Tensor, epi: str = "bf16", out=None,
                Xq_scratch=None, xscale_scratch=None, workspace=None, stream=None) -> torch.Tensor:
    M, K, ld = _rows(x, "x")
    N = Wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if epi == "i32" else torch.bfloat16,
                          device=x.device)
    if Xq_scratch is None:
        Xq_scratch = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if xscale_scratch is None:
        xscale_scratch = torch.empty(M, dtype=torch.float32, device=x.device)
    need = gemm_workspace_size(M, N, K, 0)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().sq_linear_w8a8(_ptr(x), _dtype_code(x), M, K, ld, norm,
                                _ptr(_vec(gamma_folded, K, "gamma_folded")),
                                _ptr(_vec(beta_folded, K, "beta_folded")), eps, _ptr(Wq),
                                _ptr(w_scale), N, EPI[epi], _ptr(out), out.stride(0),
                                _ptr(Xq_scratch), _ptr(xscale_scratch), _ptr(workspace), wsb,
                                _stream(stream)), "sq_linear_w8a8")
    return out


def get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(lib().sq_get_device_error(_stream(stream)))


def set_wait_limit(polls: int) -> None:
    lib().sq_set_wait_limit(int(polls))


def status_string(status: int) -> str:
    return _status_text(status)
