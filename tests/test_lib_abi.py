"""The C-ABI library loads, exports every symbol include/sq.h declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

from w8a8_int8_quantized_norm_b200 import build as sqbuild
from w8a8_int8_quantized_norm_b200 import sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")


@pytest.fixture(scope="module")
def L():
    sqbuild.build()
    return sq.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 10
    assert set(names) == set(sq.EXPORTS)
    for n in names:
        assert getattr(L, n) is not None


def test_header_constants_match_binding():
    text = open(HEADER).read()
    for name, val in [("SQ_OK", 0), ("SQ_ERR_INVALID_ARG", 1), ("SQ_ERR_UNSUPPORTED", 2),
                      ("SQ_ERR_ALIGNMENT", 3), ("SQ_ERR_OVERFLOW_RISK", 4), ("SQ_ERR_CUDA", 5),
                      ("SQ_ERR_PIPELINE_TIMEOUT", 6), ("SQ_ERR_WORKSPACE", 7), ("SQ_F32", 0),
                      ("SQ_BF16", 1), ("SQ_NORM_NONE", 0), ("SQ_NORM_RMS", 1),
                      ("SQ_NORM_LAYER", 2), ("SQ_EPI_BF16", 0), ("SQ_EPI_BF16_RELU", 1),
                      ("SQ_EPI_I32_RAW", 2)]:
        assert re.search(r"\b%s\s*=\s*%d\b" % (name, val), text), name
    assert re.search(r"#define SQ_MAX_K %d\b" % sq.MAX_K, text)
    assert re.search(r"#define SQ_NOALLOC_SCRATCH_BYTES \(8u << 20\)", text)
    assert sq.NOALLOC_SCRATCH_BYTES == 8 << 20
    assert 127 * 127 * sq.MAX_K < 2 ** 31 <= 127 * 127 * (sq.MAX_K + 1)


def test_status_strings(L):
    for code, name in sq.STATUS_NAMES.items():
        assert L.sq_status_string(code).decode().startswith(name)
    assert b"unknown" in L.sq_status_string(99)


# Fake, never-dereferenced device addresses: every call below must be rejected
# by the host-side checks before it touches CUDA.
A16 = ctypes.c_void_p(0x10000)
A8 = ctypes.c_void_p(0x10008)


def test_rows_calls_reject_bad_arguments(L):
    f = L.sq_norm_smooth_quant_per_token
    ok_args = dict(x=A16, dt=1, M=4, K=64, ld=64, norm=1, g=None, b=None, eps=1e-5, q=A16, s=A16)

    def call(**kw):
        a = dict(ok_args, **kw)
        return f(a["x"], a["dt"], a["M"], a["K"], a["ld"], a["norm"], a["g"], a["b"], a["eps"],
                 a["q"], a["s"], None)

    assert call(dt=7) == 1
    assert call(norm=9) == 1
    assert call(M=-1) == 1
    assert call(K=0) == 1
    assert call(ld=32) == 1          # ld < K
    assert call(x=None) == 1
    assert call(q=None) == 1
    assert call(s=None) == 1
    assert call(eps=-1.0) == 1
    assert call(K=40, ld=40) == 3    # K % 16
    assert call(x=A8) == 3           # misaligned base
    assert call(ld=68) == 3          # bf16 row stride not 16-byte multiple
    assert call(q=A8) == 3
    assert call(g=A8) == 3
    assert call(K=65536 * 4, ld=65536 * 4) == 2  # row too wide for one CTA
    c = L.sq_calibrate_absmax
    assert c(A16, 1, 4, 64, 64, 1, None, None, 1e-5, None, None) == 1
    assert c(A16, 1, 4, 64, 64, 5, None, None, 1e-5, A16, None) == 1
    w = L.sq_smooth_quantize_weights
    assert w(A16, 1, 4, 64, 64, None, None, A16, None) == 1
    assert w(A16, 1, 4, 64, 64, A8, A16, A16, None) == 3


def test_smooth_scales_rejects_bad_arguments(L):
    f = L.sq_compute_smooth_scales
    ptrs = (ctypes.c_void_p * 1)(0x10000)
    ns = (ctypes.c_int64 * 1)(64)
    P = ctypes.cast(ptrs, ctypes.c_void_p)
    Nn = ctypes.cast(ns, ctypes.c_void_p)
    assert f(A16, P, Nn, 1, 1, 64, 1.5, 1e-5, None, None, A16, A16, None, None) == 1  # alpha
    assert f(A16, P, Nn, 1, 1, 64, -0.1, 1e-5, None, None, A16, A16, None, None) == 1
    assert f(A16, P, Nn, 1, 1, 64, float("nan"), 1e-5, None, None, A16, A16, None, None) == 1
    assert f(A16, P, Nn, 0, 1, 64, 0.5, 1e-5, None, None, A16, A16, None, None) == 1  # num_w
    assert f(A16, P, Nn, 1, 1, 64, 0.5, 0.0, None, None, A16, A16, None, None) == 1   # eps
    assert f(A16, None, Nn, 1, 1, 64, 0.5, 1e-5, None, None, A16, A16, None, None) == 1
    assert f(A16, P, Nn, 1, 1, 64, 0.5, 1e-5, None, None, None, A16, None, None) == 1  # s
    assert f(A8, P, Nn, 1, 1, 64, 0.5, 1e-5, None, None, A16, A16, None, None) == 3


def test_gemm_rejects_bad_arguments(L):
    f = L.sq_w8a8_gemm_dequant

    def call(Xq=A16, Wq=A16, xs=A16, ws=A16, M=16, N=64, K=64, epi=0, out=A16, ldo=64,
             wsp=None, wsb=0, path=0, split=0):
        return f(Xq, Wq, xs, ws, M, N, K, epi, out, ldo, wsp, wsb, path, split, None)

    assert call(M=-1) == 1
    assert call(K=0) == 1
    assert call(epi=5) == 1
    assert call(path=4) == 1
    assert call(split=-2) == 1
    assert call(ldo=32) == 1
    assert call(Xq=None) == 1
    assert call(out=None) == 1
    assert call(xs=None) == 1           # scales needed for the bf16 epilogue
    assert call(K=sq.MAX_K + 16) == 4   # INT32 overflow risk
    assert call(K=40) == 3
    assert call(Wq=A8) == 3
    assert call(out=ctypes.c_void_p(0x10001)) == 3  # output not element aligned
    assert call(ws=A8) == 3
    assert call(path=2, M=300) == 2     # decode tiles take at most 256 tokens
    # empty problems are valid no-ops that touch nothing
    assert call(M=0, Xq=None, xs=None, out=None) == 0
    assert call(N=0, ldo=0, Wq=None, ws=None, out=None) == 0


def test_workspace_size_is_host_only_for_empty_shapes(L):
    assert L.sq_w8a8_gemm_workspace_size(0, 10, 64, 0) == 0
    assert L.sq_w8a8_gemm_workspace_size(10, 10, 64, -1) == 0


def test_rowmax_gemm_rejects_bad_arguments(L):
    f = L.sq_w8a8_gemm_dequant_rowmax

    def call(Xq=A16, Wq=A16, xs=A16, ws=A16, M=16, N=64, K=64, epi=0, out=A16, ldo=64,
             am=A16, path=0):
        return f(Xq, Wq, xs, ws, M, N, K, epi, out, ldo, am, path, None)

    assert call(epi=2) == 1             # the INT32 epilogue has no output values to reduce
    assert call(epi=5) == 1
    assert call(path=2) == 1            # decode tiles: not supported here
    assert call(path=4) == 1
    assert call(am=None) == 1
    assert call(am=A8) == 3
    assert call(K=40) == 3
    assert call(M=-1) == 1
    assert call(M=0, Xq=None, xs=None, out=None, am=None) == 0


def test_given_absmax_quant_rejects_bad_arguments(L):
    f = L.sq_quant_per_token_given_absmax

    def call(x=A16, dt=1, M=4, K=64, ld=64, am=A16, q=A16, s=A16):
        return f(x, dt, M, K, ld, am, q, s, None)

    assert call(x=None) == 1
    assert call(dt=7) == 1
    assert call(ld=32) == 1
    assert call(am=None) == 1
    assert call(q=None) == 1
    assert call(s=None) == 1
    assert call(am=A8) == 3
    assert call(K=60) == 3              # int8 rows: K % 16
    assert call(K=48000, ld=48000) == 2  # longer rows than one CTA holds
    assert call(M=0, am=None, q=None, s=None) == 0


def test_row_split_calls_reject_bad_arguments(L):
    f = L.sq_row_absmax

    def call(x=A16, dt=1, M=4, K=64, ld=64, am=A16):
        return f(x, dt, M, K, ld, am, None)

    assert call(x=None) == 1
    assert call(dt=7) == 1
    assert call(ld=32) == 1
    assert call(am=None) == 1
    assert call(am=A8) == 3
    assert call(K=60) == 3
    assert call(K=48000, ld=48000) == 2
    assert call(M=0, am=None) == 0
    g = L.sq_dequant_i32

    def dq(acc=A16, M=4, N=8, lda=8, xs=A16, ws=A16, epi=0, out=A16, ldo=8):
        return g(acc, M, N, lda, xs, ws, epi, out, ldo, None)

    assert dq(acc=None) == 1
    assert dq(xs=None) == 1
    assert dq(ws=None) == 1
    assert dq(out=None) == 1
    assert dq(lda=4) == 1
    assert dq(ldo=4) == 1
    assert dq(epi=2) == 1               # the raw accumulator is the input, not an epilogue
    assert dq(M=-1) == 1
    assert dq(acc=ctypes.c_void_p(0x10002)) == 3
    assert dq(out=ctypes.c_void_p(0x10001)) == 3
    assert dq(M=0, acc=None, xs=None, ws=None, out=None) == 0


def test_llmint8_calls_reject_bad_arguments(L):
    f = L.sq_llmint8_outliers

    def out_(col=A16, K=64, tau=6.0, mask=A16, idx=A16, cnt=A16):
        return f(col, K, tau, mask, idx, cnt, None)

    assert out_(col=None) == 1
    assert out_(K=0) == 1
    assert out_(K=(1 << 20) + 1) == 1
    assert out_(tau=-1.0) == 1
    assert out_(tau=float("nan")) == 1
    assert out_(idx=None) == 1
    assert out_(cnt=ctypes.c_void_p(0x10002)) == 3
    g = L.sq_llmint8_combine

    def comb(acc=A16, M=4, N=8, lda=8, xs=A16, ws=A16, x=A16, xd=1, ldx=64, W=A16, wd=1,
             ldw=64, K=64, idx=A16, cnt=A16, epi=0, out=A16, ldo=8):
        return g(acc, M, N, lda, xs, ws, x, xd, ldx, W, wd, ldw, K, idx, cnt, epi, out, ldo, None)

    assert comb(acc=None) == 1
    assert comb(idx=None) == 1
    assert comb(cnt=None) == 1
    assert comb(W=None) == 1
    assert comb(ldx=32) == 1
    assert comb(ldw=32) == 1
    assert comb(lda=4) == 1
    assert comb(xd=7) == 1
    assert comb(epi=2) == 1
    assert comb(x=ctypes.c_void_p(0x10001)) == 3
    assert comb(W=ctypes.c_void_p(0x10002), wd=0) == 3
    assert comb(M=0, acc=None, out=None) == 0


def test_silu_mul_quant_rejects_bad_arguments(L):
    f = L.sq_silu_mul_quant_per_token

    def call(gu=A16, dt=1, M=4, I=64, ld=128, q=A16, s=A16, h=None, ldh=0):
        return f(gu, dt, M, I, ld, q, s, h, ldh, None)

    assert call(gu=None) == 1
    assert call(dt=7) == 1
    assert call(ld=64) == 1             # a row holds gate and up: ld >= 2I
    assert call(I=0) == 1
    assert call(M=-1) == 1
    assert call(q=None) == 1
    assert call(s=None) == 1
    assert call(h=A16, ldh=32) == 1     # ld_h < I
    assert call(dt=0) == 2              # bf16 rows only
    assert call(I=40, ld=80) == 3       # I % 16
    assert call(s=A8) == 3
    assert call(h=A8, ldh=64) == 3
    assert call(I=28944, ld=2 * 28944) == 2  # beyond one CTA's shared memory
    assert call(M=0, gu=None, q=None, s=None) == 0


def test_fp8_calls_reject_bad_arguments(L):
    g = L.sq_fp8_gemm_dequant

    def gemm(Xq=A16, Wq=A16, xs=A16, ws=A16, M=16, N=64, K=64, epi=0, out=A16, ldo=64, path=0):
        return g(Xq, Wq, xs, ws, M, N, K, epi, out, ldo, None, 0, path, None)

    assert gemm(epi=2) == 1             # INT32 output: INT8 GEMMs only
    assert gemm(epi=7) == 1
    assert gemm(path=5) == 1
    assert gemm(xs=None) == 1           # bf16 epilogues need both scales
    assert gemm(K=40) == 3
    assert gemm(M=0, Xq=None, xs=None, out=None) == 0
    q = L.sq_norm_smooth_quant_per_token_fp8
    assert q(A16, 1, 4, 64, 64, 1, None, None, 1e-5, None, A16, None) == 1
    assert q(A16, 1, 4, 64, 64, 9, None, None, 1e-5, A16, A16, None) == 1
    assert q(A16, 1, 4, 64, 64, 1, None, None, 1e-5, A8, A16, None) == 3
    assert q(A16, 1, 0, 64, 64, 1, None, None, 1e-5, None, None, None) == 0
    w = L.sq_smooth_quantize_weights_fp8
    assert w(A16, 1, 4, 64, 64, None, None, A16, None) == 1
    assert w(A16, 1, 4, 64, 64, A8, A16, A16, None) == 3


def test_split_smoothing_calls_reject_bad_arguments(L):
    ns = (ctypes.c_int64 * 1)(64)
    ws = (ctypes.c_void_p * 1)(0x10000)
    P = ctypes.cast(ws, ctypes.c_void_p)
    Nn = ctypes.cast(ns, ctypes.c_void_p)
    cm = L.sq_weight_column_max
    assert cm(None, Nn, 1, 1, 64, A16, None) == 1
    assert cm(P, Nn, 0, 1, 64, A16, None) == 1      # no weights
    assert cm(P, Nn, 1, 7, 64, A16, None) == 1      # dtype
    assert cm(P, Nn, 1, 1, 64, None, None) == 1     # w_max
    assert cm(P, Nn, 1, 1, 64, A8, None) == 3
    assert cm(P, Nn, 1, 1, 40, A16, None) == 3      # K % 16
    fm = L.sq_smooth_scales_from_maxima

    def fin(am=A16, wm=A16, K=64, alpha=0.5, eps=1e-5, g=None, b=None, s=A16, gf=A16, bf=None):
        return fm(am, wm, K, alpha, eps, g, b, s, gf, bf, None)

    assert fin(alpha=1.5) == 1
    assert fin(alpha=float("nan")) == 1
    assert fin(eps=0.0) == 1
    assert fin(K=0) == 1
    assert fin(am=None) == 1
    assert fin(wm=None) == 1
    assert fin(s=None) == 1
    assert fin(gf=None) == 1
    assert fin(wm=A8) == 3
    assert fin(g=A8) == 3
