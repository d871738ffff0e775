"""GPU (libsq.so through the C ABI) versus the CPU oracle, element by element.

Stage tests feed both sides the same seeded inputs (for a later stage, the
oracle's own upstream results); workload tests run the whole path on the GPU
and the oracle on the full tensors (small workloads) or on sampled token rows
(full-size workloads, which the GPU processes at full size in the same launch
configuration as the benchmark).
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_norm_b200 import pipeline, sq
from w8a8_int8_quantized_norm_b200 import synthetic as S

from _oracle_pipeline import forward_rows, prepare
from _parity import (bf16_bits, bf16_ulp_diff, compare_rows_quant, norm_near_tie_rows,
                     scale_near_tie_channels, to_gpu)

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(20261202)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sq.lib()
    yield
    assert sq.get_device_error() == 0


def _acts(M, K, dtype, outliers=3, scale=1.0):
    x = RNG.standard_normal((M, K)).astype(np.float32) * np.float32(scale)
    if K >= 8 and outliers:
        ch = RNG.choice(K, size=min(outliers, K), replace=False)
        x[:, ch] *= RNG.uniform(20, 100, ch.size).astype(np.float32)
    return S.to_bf16_bits(x) if dtype == "bf16" else x


# ---------------------------------------------------------------------------
# K1: fused norm + per-token quantisation
# ---------------------------------------------------------------------------

SHAPES = [(1, 16), (3, 48), (17, 64), (129, 4112), (64, 8192), (5, 28672), (3, 36864),
          (2, 40960)]
KINDS = [("none", oracle.NORM_NONE, False), ("none_mult", oracle.NORM_NONE, True),
         ("rms", oracle.NORM_RMS, True), ("rms_nogamma", oracle.NORM_RMS, False),
         ("layer", oracle.NORM_LAYER, True)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("kind", KINDS, ids=lambda k: k[0])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_quant_matches_oracle(shape, kind, dtype):
    M, K = shape
    _, norm, with_params = kind
    x = _acts(M, K, dtype)
    if M >= 3:
        x[1] = 0  # an all-zero row: scale 0, codes 0 (LayerNorm: y = beta)
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32) if with_params else None
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if (with_params and norm == oracle.NORM_LAYER) else None
    Xq_o, xs_o = oracle.norm_quant(x, norm, g, b, 1e-5)
    Xq_g, xs_g = sq.norm_smooth_quant_per_token(to_gpu(x), norm, None if g is None else to_gpu(g),
                                                None if b is None else to_gpu(b), 1e-5)
    tol = compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, xs_o,
                             norm_near_tie_rows(x, norm, 1e-5))
    assert tol == 0


@pytest.mark.parametrize("shape", [(1000, 4096), (777, 8192), (4099, 64), (300, 9216),
                                   (2048, 4096), (700, 4112), (5000, 1024), (150, 40960)],
                         ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("kind", [oracle.NORM_RMS, oracle.NORM_LAYER, oracle.NORM_NONE])
def test_norm_quant_many_rows(shape, kind):
    """More rows than resident CTAs: every CTA loops over several rows."""
    M, K = shape
    x = _acts(M, K, "bf16")
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if kind == oracle.NORM_LAYER else None
    Xq_o, xs_o = oracle.norm_quant(x, kind, g, b, 1e-5)
    Xq_g, xs_g = sq.norm_smooth_quant_per_token(to_gpu(x), kind, to_gpu(g),
                                                None if b is None else to_gpu(b), 1e-5)
    assert compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, xs_o,
                              norm_near_tie_rows(x, kind, 1e-5)) == 0


def test_quantizer_half_integer_quotients():
    """Values whose quotient by the step is a half-integer or within an ulp of
    one: the rounding must follow the exact fp32 quotient (ties to even)."""
    K = 4096
    rows = []
    for am in (100.0, 3.0, 0.1234, 77.7):
        step = np.float32(np.float32(am) / np.float32(127.0))
        k = RNG.integers(-126, 126, K).astype(np.float32)
        y = ((k + np.float32(0.5)) * step).astype(np.float32)
        y = np.nextafter(y, y + RNG.choice([-1.0, 0.0, 1.0], K).astype(np.float32) * np.float32(1e30))
        y = y.astype(np.float32)
        y[0] = am
        y[1] = -am
        y = np.clip(y, -am, am).astype(np.float32)
        rows.append(y)
    x = np.stack(rows)
    Xq_o, xs_o = oracle.norm_quant(x, oracle.NORM_NONE)
    Xq_g, xs_g = sq.norm_smooth_quant_per_token(to_gpu(x), oracle.NORM_NONE)
    assert np.array_equal(xs_g.cpu().numpy(), xs_o)
    assert np.array_equal(Xq_g.cpu().numpy(), Xq_o)


def test_norm_quant_strided_rows_and_canaries():
    M, K, ld = 33, 4096, 4096 + 64
    big = S.to_bf16_bits(RNG.standard_normal((M, ld)).astype(np.float32))
    x = np.ascontiguousarray(big[:, :K])
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    Xq_o, xs_o = oracle.norm_quant(x, oracle.NORM_RMS, g, None, 1e-5)
    xg = to_gpu(big)[:, :K]
    assert xg.stride(0) == ld
    # outputs with guard regions around them
    q_buf = torch.full((M + 2, K), 77, dtype=torch.int8, device="cuda")
    s_buf = torch.full((M + 8,), -3.0, dtype=torch.float32, device="cuda")
    Xq_g, xs_g = sq.norm_smooth_quant_per_token(xg, oracle.NORM_RMS, to_gpu(g), None, 1e-5,
                                                Xq=q_buf[1:M + 1], x_scale=s_buf[4:M + 4])
    assert torch.all(q_buf[0] == 77) and torch.all(q_buf[M + 1] == 77)
    assert torch.all(s_buf[:4] == -3.0) and torch.all(s_buf[M + 4:] == -3.0)
    compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, xs_o,
                       norm_near_tie_rows(x, oracle.NORM_RMS, 1e-5))


def test_worked_example_row_on_gpu(golden_dir):
    """The pages' 4096-wide row with outliers 45 and -60: step 60/127 on the GPU too."""
    import json, os
    g = json.load(open(os.path.join(golden_dir, "token_row_outliers.json")))
    row = RNG.uniform(-2, 2, g["row_width"]).astype(np.float32)
    for ch, v in g["outliers"].items():
        row[int(ch)] = v
    Xq, xs = sq.norm_smooth_quant_per_token(to_gpu(row[None, :]), oracle.NORM_NONE)
    assert float(xs[0]) == float(np.float32(60.0) / np.float32(127.0))
    q = Xq.cpu().numpy()[0]
    mask = np.ones(row.size, bool)
    mask[[int(c) for c in g["outliers"]]] = False
    assert q[mask].min() >= -4 and q[mask].max() <= 4


@pytest.mark.parametrize("case", [(2048, 4096, 12288, oracle.NORM_RMS, "bf16", False),
                                  (37, 4112, 1000, oracle.NORM_LAYER, "bf16", True),
                                  (5, 64, 48, oracle.NORM_RMS, "f32", False)],
                         ids=["opt-qkv-2048x4096x12288-rms", "37x4112x1000-layer-relu",
                              "5x64x48-rms-f32"])
def test_linear_w8a8_matches_oracle(case):
    """sq_linear_w8a8, the whole runtime layer in one call (norm + per-token
    quantisation into caller scratch, then the GEMM with its epilogue), against
    the oracle's linear: codes, scales and the bf16 output bit for bit; the
    output and scratch buffers have guard regions that must stay untouched."""
    M, K, N, norm, dtype, relu = case
    x = _acts(M, K, dtype)
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if norm == oracle.NORM_LAYER else None
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq_o, ws_o = oracle.quantize_weights(W, None)
    Xq_o, xs_o, _, _, out_o = oracle.linear(x, norm, g, b, 1e-5, Wq_o, ws_o, relu)
    ld = N + 24
    out_buf = torch.full((M + 2, ld), -7.0, dtype=torch.bfloat16, device="cuda")
    q_buf = torch.full((M + 2, K), 55, dtype=torch.int8, device="cuda")
    s_buf = torch.full((M + 8,), -3.0, dtype=torch.float32, device="cuda")
    out = out_buf[1:M + 1, :N]
    sq.linear_w8a8(to_gpu(x), norm, to_gpu(g), None if b is None else to_gpu(b), 1e-5,
                   to_gpu(Wq_o), to_gpu(ws_o), "bf16_relu" if relu else "bf16", out=out,
                   Xq_scratch=q_buf[1:M + 1], xscale_scratch=s_buf[4:M + 4])
    assert sq.get_device_error() == 0
    tie = norm_near_tie_rows(x, norm, 1e-5)
    assert compare_rows_quant(q_buf[1:M + 1].cpu().numpy(), s_buf[4:M + 4].cpu().numpy(), Xq_o,
                              xs_o, tie) == 0
    assert np.array_equal(bf16_bits(out), out_o)
    ob = bf16_bits(out_buf)
    assert (ob[0] == bf16_bits(torch.tensor([-7.0], dtype=torch.bfloat16))[0]).all()
    assert (ob[M + 1] == ob[0]).all() and (ob[1:M + 1, N:] == ob[0, 0]).all()
    assert torch.all(q_buf[0] == 55) and torch.all(q_buf[M + 1] == 55)
    assert torch.all(s_buf[:4] == -3.0) and torch.all(s_buf[M + 4:] == -3.0)


# ---------------------------------------------------------------------------
# K2: calibration, smoothing factors + fold, weight smoothing + quantisation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", [oracle.NORM_NONE, oracle.NORM_RMS, oracle.NORM_LAYER])
@pytest.mark.parametrize("K", [64, 4096, 9216, 16384, 28672])
def test_calibration_running_max(kind, K):
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if kind == oracle.NORM_LAYER else None
    x1, x2 = _acts(300, K, "bf16"), _acts(213, K, "bf16")
    am_o = oracle.calibrate_absmax(x1, kind, g, b)
    am_o = oracle.calibrate_absmax(x2, kind, g, b, act_max=am_o)
    gg, bb = to_gpu(g), (to_gpu(b) if b is not None else None)
    am_g = sq.calibrate_absmax(to_gpu(x1), kind, gg, bb)
    am_g = sq.calibrate_absmax(to_gpu(x2), kind, gg, bb, act_max=am_g).cpu().numpy()
    ties = norm_near_tie_rows(np.concatenate([x1, x2]), kind, 1e-5)
    if not ties.any():
        assert np.array_equal(am_g.view(np.uint32), am_o.view(np.uint32))
    else:
        assert np.all(np.abs(am_g - am_o) <= 2 * np.spacing(am_o))


@pytest.mark.parametrize("kind", [oracle.NORM_NONE, oracle.NORM_RMS, oracle.NORM_LAYER])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(3000, 4096), (1500, 4112), (2, 8192)],
                         ids=lambda s: "%dx%d" % s)
def test_calibration_many_rows(kind, dtype, shape):
    """Several rows per CTA, ragged chunk counts, a row count below the CTA count."""
    M, K = shape
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if kind == oracle.NORM_LAYER else None
    x = _acts(M, K, dtype)
    am_o = oracle.calibrate_absmax(x, kind, g, b)
    am_g = sq.calibrate_absmax(to_gpu(x), kind, to_gpu(g),
                               None if b is None else to_gpu(b)).cpu().numpy()
    ties = norm_near_tie_rows(x, kind, 1e-5)
    if not ties.any():
        assert np.array_equal(am_g.view(np.uint32), am_o.view(np.uint32))
    else:
        assert np.all(np.abs(am_g - am_o) <= 2 * np.spacing(am_o))


@pytest.mark.parametrize("NK", [(5000, 4112), (20000, 64), (3, 2064)], ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_weight_column_max_through_scales(NK, dtype):
    """alpha = 0 makes s_j = 1 / max(w_j, eps): the column maxima of a tall,
    ragged weight come back exactly through s."""
    N, K = NK
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[RNG.integers(0, N, 40), RNG.integers(0, K, 40)] = 3.5  # isolated column peaks
    W[:, 7] = 0.0
    if dtype == "bf16":
        W = S.to_bf16_bits(W)
    act_max = np.ones(K, np.float32)
    s_o, s64 = oracle.smooth_scales(act_max, [W], 0.0, 1e-5)
    s_g, _, _ = sq.compute_smooth_scales(to_gpu(act_max), [to_gpu(W)], 0.0, 1e-5)
    s_g = s_g.cpu().numpy()
    diff = s_g.view(np.uint32) != s_o.view(np.uint32)
    assert not np.any(diff & ~scale_near_tie_channels(s64))


@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.8, 1.0])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_smooth_scales_and_fold(alpha, dtype):
    K = 4096
    act_max = np.abs(RNG.standard_normal(K)).astype(np.float32) * 3
    act_max[[5, 77, 300]] = [60.0, 0.0, 1e-7]
    Ws = [(RNG.standard_normal((n, K)) * 0.02).astype(np.float32) for n in (1024, 512, 512)]
    Ws[1][:, 9] = 0.0
    Ws[0][:, 9] = 0.0
    Ws[2][:, 9] = 0.0
    if dtype == "bf16":
        Ws = [S.to_bf16_bits(w) for w in Ws]
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32)
    s_o, s64 = oracle.smooth_scales(act_max, Ws, alpha, 1e-5)
    gf_o, bf_o = oracle.fold_norm(s_o, g, b)
    s_g, gf_g, bf_g = sq.compute_smooth_scales(to_gpu(act_max), [to_gpu(w) for w in Ws], alpha,
                                               1e-5, to_gpu(g), to_gpu(b))
    s_g, gf_g, bf_g = s_g.cpu().numpy(), gf_g.cpu().numpy(), bf_g.cpu().numpy()
    diff = s_g.view(np.uint32) != s_o.view(np.uint32)
    ties = scale_near_tie_channels(s64)
    assert not np.any(diff & ~ties), np.nonzero(diff & ~ties)[0][:10]
    assert np.all(np.abs(s_g[diff] - s_o[diff]) <= np.spacing(s_o[diff]))
    same = ~diff
    assert np.array_equal(gf_g[same].view(np.uint32), gf_o[same].view(np.uint32))
    assert np.array_equal(bf_g[same].view(np.uint32), bf_o[same].view(np.uint32))
    # no norm in front: gamma = 1, gamma' = 1/s
    _, gf1, bf1 = sq.compute_smooth_scales(to_gpu(act_max), [to_gpu(Ws[0])], alpha, 1e-5)
    s1, _ = oracle.smooth_scales(act_max, [Ws[0]], alpha, 1e-5)
    gfo1, _ = oracle.fold_norm(s1)
    assert bf1 is None
    assert np.array_equal(gf1.cpu().numpy().view(np.uint32), gfo1.view(np.uint32))


@pytest.mark.parametrize("NK", [(1, 16), (7, 48), (300, 4096), (129, 4112), (64, 28672)])
@pytest.mark.parametrize("smoothed", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_weight_quant_matches_oracle(NK, smoothed, dtype):
    N, K = NK
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    if N > 3:
        W[2] = 0.0
    if dtype == "bf16":
        W = S.to_bf16_bits(W)
    s = RNG.uniform(0.05, 20.0, K).astype(np.float32) if smoothed else None
    Wq_o, ws_o = oracle.quantize_weights(W, s)
    Wq_g, ws_g = sq.smooth_quantize_weights(to_gpu(W), None if s is None else to_gpu(s))
    assert np.array_equal(Wq_g.cpu().numpy(), Wq_o)
    assert np.array_equal(ws_g.cpu().numpy().view(np.uint32), ws_o.view(np.uint32))


# ---------------------------------------------------------------------------
# K3 / K4: the INT8 GEMM and its epilogue
# ---------------------------------------------------------------------------

# the automatic pair-tile width differs by shape: most small shapes take
# 256 x 192 tiles (fewer rounds over the SM pairs), (2048, 9472, 128) 256 x 256
GEMM_SHAPES = [(16, 64, 64), (3, 5, 16), (1, 300, 48), (129, 257, 4112), (256, 512, 1024),
               (200, 1000, 128), (300, 777, 160), (1024, 768, 2048), (2048, 1536, 512),
               (600, 2304, 4096), (1024, 3000, 272), (2048, 9472, 128), (200, 15000, 64)]


def _codes(M, K, extreme=False):
    if extreme:
        return np.full((M, K), -127, np.int8)
    return RNG.integers(-127, 128, (M, K)).astype(np.int8)


# path hints: 1 = prefill on CTA pairs (2-SM MMA), 2 = decode tiles, 3 = prefill on one SM
@pytest.mark.parametrize("shape", GEMM_SHAPES, ids=lambda s: "%dx%dx%d" % s)
@pytest.mark.parametrize("path", [1, 2, 3])
def test_gemm_int32_exact(shape, path):
    M, N, K = shape
    if path == 2 and M > 256:
        pytest.skip("decode tiles take at most 256 tokens")
    A, B = _codes(M, K), _codes(N, K)
    acc_o = oracle.gemm_i64(A, B)
    out = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "i32", path_hint=path)
    assert np.array_equal(out.cpu().numpy().astype(np.int64), acc_o)


def test_gemm_int32_extremes_and_max_k():
    # |acc| = 127*127*K at the largest K whose products fit INT32
    K = sq.MAX_K // 16 * 16
    A, B = _codes(3, K, extreme=True), _codes(130, K, extreme=True)
    B[1] = 127
    acc_o = oracle.gemm_i64(A, B)
    assert acc_o.max() == 127 * 127 * K and acc_o.min() == -127 * 127 * K
    for path in (1, 2, 3):
        out = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "i32", path_hint=path)
        assert np.array_equal(out.cpu().numpy().astype(np.int64), acc_o)


@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_split_k_invariance(M):
    N, K = 640, 4096
    A, B = _codes(M, K), _codes(N, K)
    acc_o = oracle.gemm_i64(A, B)
    for split in (1, 2, 4, 8):
        out = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "i32", path_hint=2,
                                   split_k=split)
        assert np.array_equal(out.cpu().numpy().astype(np.int64), acc_o), split


@pytest.mark.parametrize("shape", [(16, 64, 64), (129, 257, 4112), (7, 1000, 512), (512, 384, 256),
                                   (200, 15000, 64)],
                         ids=lambda s: "%dx%dx%d" % s)
@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("path", [1, 2, 3])
def test_gemm_bf16_epilogue(shape, relu, path):
    M, N, K = shape
    if path == 2 and M > 256:
        pytest.skip("decode tiles take at most 256 tokens")
    A, B = _codes(M, K), _codes(N, K)
    xs = (RNG.random(M) * 0.05 + 1e-3).astype(np.float32)
    ws = (RNG.random(N) * 0.002 + 1e-5).astype(np.float32)
    acc = oracle.gemm_i64(A, B)
    o32, out_o = oracle.epilogue(acc, xs, ws, relu)
    ldo = N + 24 if (N + 24) % 8 == 0 else (N + 24 + 7) // 8 * 8
    buf = torch.full((M, ldo), 1.5, dtype=torch.bfloat16, device="cuda")
    view = buf[:, :N]
    sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws),
                         "bf16_relu" if relu else "bf16", out=view, path_hint=path)
    assert torch.all(buf[:, N:] == 1.5)  # the padding columns are untouched
    out_g = bf16_bits(view.contiguous())
    assert bf16_ulp_diff(out_g, out_o).max() <= 1
    assert np.array_equal(out_g, out_o)


# ---------------------------------------------------------------------------
# fc1 -> ReLU -> fc2: row maxima reduced in the GEMM epilogue, then the
# per-token quantisation with those maxima given
# ---------------------------------------------------------------------------

def _bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("shape", [(16, 64, 64), (129, 257, 4112), (512, 384, 256),
                                   (300, 2304, 512), (1024, 3000, 272)],
                         ids=lambda s: "%dx%dx%d" % s)
@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("path", [0, 3])
def test_gemm_rowmax_epilogue(shape, relu, path):
    M, N, K = shape
    A, B = _codes(M, K), _codes(N, K)
    xs = (RNG.random(M) * 0.05 + 1e-3).astype(np.float32)
    ws = (RNG.random(N) * 0.002 + 1e-5).astype(np.float32)
    xs[M // 2] = 0.0  # an all-zero output row: its max is 0
    o32, out_o = oracle.epilogue(oracle.gemm_i64(A, B), xs, ws, relu)
    am_o = np.abs(_bf16_to_f32(out_o)).max(axis=1)
    am = torch.full((M,), 3e38, dtype=torch.float32, device="cuda")  # the call zeroes it
    out_g, am_g = sq.w8a8_gemm_dequant_rowmax(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws),
                                              "bf16_relu" if relu else "bf16", row_absmax=am,
                                              path_hint=path)
    assert np.array_equal(bf16_bits(out_g), out_o)
    assert np.array_equal(am_g.cpu().numpy().view(np.uint32), am_o.view(np.uint32))
    # the plain call's output is the same
    ref = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws),
                               "bf16_relu" if relu else "bf16", path_hint=path or 1)
    assert torch.equal(ref, out_g)


@pytest.mark.parametrize("split", [0, 2])
def test_decode_split_tiles_relu_of_negative_zero(split):
    """The stream-K tile finish and the split-K reduction apply the same ReLU as
    the main epilogue: a zero token scale gives +0, never -0."""
    M, N, K = 5, 4096, 8192
    A, B = _codes(M, K), _codes(N, K)
    xs = (RNG.random(M) * 0.05 + 1e-3).astype(np.float32)
    ws = (RNG.random(N) * 0.002 + 1e-5).astype(np.float32)
    xs[2] = 0.0
    _, out_o = oracle.epilogue(oracle.gemm_i64(A, B), xs, ws, True)
    out = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws), "bf16_relu",
                               path_hint=2, split_k=split)
    assert np.array_equal(bf16_bits(out), out_o)


@pytest.mark.parametrize("shape", [(1, 10240, 8192), (8, 8192, 8192), (32, 1000, 4112),
                                   (128, 3000, 2048), (3, 28672, 8192)],
                         ids=lambda s: "%dx%dx%d" % s)
def test_decode_streamk_on_a_dirty_workspace_twice(shape):
    """Nothing of the stream-K plan's workspace has to start at any value: a
    workspace full of garbage, then reused by a second call with other
    inputs, gives the oracle's bits both times."""
    M, N, K = shape
    need = sq.gemm_workspace_size(M, N, K, 0)
    plan = sq.gemm_plan(M, N, K, 0, 0)
    assert plan.stream_k == 1 and plan.launches == (2 if need else 1)
    ws_buf = torch.full((max(need, 1),), 0x7f, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        A, B = _codes(M, K), _codes(N, K)
        xs = (RNG.random(M) * 0.05 + 1e-3).astype(np.float32)
        ws = (RNG.random(N) * 0.002 + 1e-5).astype(np.float32)
        acc = oracle.gemm_i64(A, B)
        _, out_o = oracle.epilogue(acc, xs, ws)
        out = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws), "bf16",
                                   workspace=ws_buf if need else None)
        raw = sq.w8a8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "i32",
                                   workspace=ws_buf if need else None)
        assert sq.get_device_error() == 0
        assert np.array_equal(bf16_bits(out), out_o)
        assert np.array_equal(raw.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("cuts", [(0, 4096, 8192), (0, 1024, 5120, 8192), (0, 16, 8192)],
                         ids=["2-even", "3-uneven", "2-thin"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_row_split_slices_equal_the_unsplit_layer(cuts, dtype):
    """The row split of ksplit through the C ABI, its slices run one after
    another on this GPU and reduced by torch (max of the row maxima, sum of
    the INT32 partials): weight codes and scales, token scales, the
    accumulator and the bf16 output equal the oracle's unsplit layer."""
    from w8a8_int8_quantized_norm_b200 import ksplit
    M, N, K = 37, 1000, cuts[-1]
    x = _acts(M, K, dtype)
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    if dtype == "bf16":
        W = S.to_bf16_bits(W)
    Wq_o, ws_o = oracle.quantize_weights(W, None)
    _, xs_o, acc_o, _, out_o = oracle.linear(x, oracle.NORM_NONE, None, None, 1e-5, Wq_o, ws_o)
    spans = list(zip(cuts, cuts[1:]))
    xg = [to_gpu(np.ascontiguousarray(x[:, a:b])) for a, b in spans]
    Wg = [to_gpu(np.ascontiguousarray(W[:, a:b])) for a, b in spans]
    am_w = torch.stack([ksplit.LibOps.row_absmax(w) for w in Wg]).amax(0)
    qw = [ksplit.LibOps.quant_given(w, am_w) for w in Wg]
    am = torch.stack([ksplit.shard_row_max(v) for v in xg]).amax(0)
    parts = [ksplit.shard_partial(v, am, q[0]) for v, q in zip(xg, qw)]
    acc = parts[0][0].clone()
    for p_, _ in parts[1:]:
        acc += p_
    out = ksplit.finish(acc, parts[0][1], qw[0][1])
    assert sq.get_device_error() == 0
    for (a, b), (wq, ws) in zip(spans, qw):
        assert np.array_equal(ws.cpu().numpy().view(np.uint32), ws_o.view(np.uint32))
        assert np.array_equal(wq.cpu().numpy(), Wq_o[:, a:b])
    for _, xs in parts:
        assert np.array_equal(xs.cpu().numpy().view(np.uint32), xs_o.view(np.uint32))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_o)
    assert np.array_equal(bf16_bits(out), out_o)
    assert np.array_equal(am.cpu().numpy(), np.abs(x.view(np.float32) if dtype == "f32" else
                                                   _bf16_to_f32(x)).max(axis=1))


def _bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("case", [(37, 4096, 1000, "bf16", 6.0, False),
                                  (5, 64, 48, "f32", 6.0, True),
                                  (64, 512, 300, "bf16", 1.0, False),
                                  (9, 256, 128, "bf16", 1e9, False),
                                  (2048, 4096, 12288, "bf16", 6.0, False)],
                         ids=["37x4096x1000", "5x64x48-f32-relu", "many-outliers",
                              "no-outliers", "opt-qkv-sampled"])
def test_llmint8_comparator_matches_oracle(case):
    """LLM.int8()'s decomposition through the C ABI against the oracle: the
    column maxima, outlier mask and list, codes, token scales, the INT32
    accumulator and the bf16 output, bit for bit (the full-size case on
    sampled rows; its outlier set comes from all tokens on both sides)."""
    from w8a8_int8_quantized_norm_b200 import llmint8
    M, K, N, dtype, tau, relu = case
    x = _acts(M, K, dtype, outliers=8)
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    if dtype == "bf16":
        W = S.to_bf16_bits(W)
    Wq_o, ws_o = oracle.quantize_weights(W, None)
    lin = llmint8.LLMInt8Linear(to_gpu(W), tau).prepare()
    out = lin.forward(to_gpu(x), "bf16_relu" if relu else "bf16")
    assert sq.get_device_error() == 0
    assert np.array_equal(lin.Wq.cpu().numpy(), Wq_o)
    col = oracle.calibrate_absmax(x, oracle.NORM_NONE)
    mask, idx = oracle.llmint8_outliers(col, tau)
    assert np.array_equal(lin.col.cpu().numpy().view(np.uint32), col.view(np.uint32))
    assert np.array_equal(lin.mask.cpu().numpy(), mask)
    n = int(lin.count.item())
    assert n == idx.size and np.array_equal(lin.idx[:n].cpu().numpy(), idx)
    rows = np.arange(M) if M <= 64 else np.sort(RNG.choice(M, 48, replace=False))
    xr = np.ascontiguousarray(x[rows])
    Xq_o, xs_o = oracle.norm_quant(xr, oracle.NORM_NONE, mask, None)
    acc_o = oracle.gemm_i64(Xq_o, Wq_o)
    o32, _ = oracle.epilogue(acc_o, xs_o, ws_o, False)
    _, out_o = oracle.llmint8_combine(o32, xr, W, idx, relu)
    st = lin.stages
    assert np.array_equal(st["Xq"].cpu().numpy()[rows], Xq_o)
    assert np.array_equal(st["x_scale"].cpu().numpy()[rows].view(np.uint32), xs_o.view(np.uint32))
    assert np.array_equal(st["acc"].cpu().numpy()[rows].astype(np.int64), acc_o)
    assert np.array_equal(bf16_bits(out)[rows], out_o)


def test_gemm_rowmax_rejects_other_epilogues_and_decode_tiles():
    A, B = to_gpu(_codes(8, 64)), to_gpu(_codes(32, 64))
    xs, ws = torch.ones(8, device="cuda"), torch.ones(32, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.w8a8_gemm_dequant_rowmax(A, B, xs, ws, "i32",
                                    out=torch.empty((8, 32), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == 1  # SQ_ERR_INVALID_ARG
    with pytest.raises(sq.SQError) as e:
        sq.w8a8_gemm_dequant_rowmax(A, B, xs, ws, "bf16", path_hint=2)
    assert e.value.status == 1  # SQ_ERR_INVALID_ARG


@pytest.mark.parametrize("shape", [(1, 16), (17, 4096), (300, 4112), (64, 9216), (40, 36864),
                                   (5, 28672)], ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quant_given_absmax_equals_per_token(shape, dtype):
    M, K = shape
    if dtype == "f32" and K > 25600:
        pytest.skip("fp32 rows above 25600 elements are unsupported")
    x = _acts(M, K, dtype)
    if M > 2:
        x[1] = 0  # a zero row: step 0, codes 0
    y, _, _ = oracle.norm(x, oracle.NORM_NONE)
    am = np.abs(y).max(axis=1).astype(np.float32)
    Xq_o, xs_o = oracle.norm_quant(x, oracle.NORM_NONE)
    Xq_g, xs_g = sq.quant_per_token_given_absmax(to_gpu(x), to_gpu(am))
    assert np.array_equal(xs_g.cpu().numpy().view(np.uint32), xs_o.view(np.uint32))
    assert np.array_equal(Xq_g.cpu().numpy(), Xq_o)


def test_quant_given_absmax_below_the_row_max_saturates():
    M, K = 33, 4096
    x = _acts(M, K, "bf16")
    y, _, _ = oracle.norm(x, oracle.NORM_NONE)
    am = (np.abs(y).max(axis=1) * np.float32(0.3)).astype(np.float32)
    Xq_g, xs_g = sq.quant_per_token_given_absmax(to_gpu(x), to_gpu(am))
    for m in range(M):
        step = oracle.step_of(am[m])
        assert xs_g[m].item() == step
        Xq_o = oracle.quantize_with_step(y[m:m + 1], step)
        assert np.count_nonzero(np.abs(Xq_o) == 127) > 0
        assert np.array_equal(Xq_g[m:m + 1].cpu().numpy(), Xq_o), m


# SiLU(gate) * up quantised per token (the down projection's input)
SILU_SHAPES = [(1, 16), (3, 64), (17, 4096), (300, 4112), (64, 28672), (5, 28928), (2000, 1024)]


def _gate_up(M, I, seed=0):
    r = np.random.default_rng(seed)
    g = (r.standard_normal((M, I)) * 2.5).astype(np.float32)
    u = r.standard_normal((M, I)).astype(np.float32)
    if I >= 16:
        g[:, :8] = np.float32([0.0, -0.0, 90.0, -90.0, 1e-20, 40.0, -40.0, 87.5])
        u[:, 8] *= 60.0  # an outlier channel of up
    if M > 2:
        g[1] = 0.0  # a row whose h is all zero: step 0, codes 0
    return S.to_bf16_bits(np.concatenate([g, u], axis=1))


@pytest.mark.parametrize("shape", SILU_SHAPES, ids=lambda s: "%dx%d" % s)
def test_silu_mul_quant_matches_oracle(shape):
    M, I = shape
    gu = _gate_up(M, I)
    Xq_o, xs_o, hb_o = oracle.silu_mul_quant(gu)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    Xq_g, xs_g = sq.silu_mul_quant_per_token(to_gpu(gu), h_out=h)
    assert np.array_equal(bf16_bits(h), hb_o)
    assert np.array_equal(xs_g.cpu().numpy().view(np.uint32), xs_o.view(np.uint32))
    assert np.array_equal(Xq_g.cpu().numpy(), Xq_o)
    Xq2, xs2 = sq.silu_mul_quant_per_token(to_gpu(gu))  # without storing h
    assert torch.equal(Xq2, Xq_g) and torch.equal(xs2, xs_g)


@pytest.mark.parametrize("shape", [(1, 16), (17, 4096), (64, 28672), (2000, 1024)],
                         ids=lambda s: "%dx%d" % s)
def test_silu_mul_quant_fp8_matches_oracle(shape):
    M, I = shape
    gu = _gate_up(M, I, seed=4)
    _, hb_o = oracle.silu_mul(gu)
    Xq_o, xs_o = oracle.norm_quant_fp8(hb_o, oracle.NORM_NONE)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    Xq_g, xs_g = sq.silu_mul_quant_per_token(to_gpu(gu), h_out=h, fp8=True)
    assert Xq_g.dtype == torch.uint8
    assert np.array_equal(bf16_bits(h), hb_o)
    assert np.array_equal(xs_g.cpu().numpy().view(np.uint32), xs_o.view(np.uint32))
    assert np.array_equal(Xq_g.cpu().numpy(), Xq_o)


def test_silu_mul_quant_strided_rows():
    M, I = 37, 2048
    gu = _gate_up(M, I, seed=3)
    buf = torch.zeros((M, 2 * I + 64), dtype=torch.bfloat16, device="cuda")
    buf[:, :2 * I] = to_gpu(gu)
    hbuf = torch.full((M, I + 24), 2.0, dtype=torch.bfloat16, device="cuda")
    Xq_g, xs_g = sq.silu_mul_quant_per_token(buf[:, :2 * I], h_out=hbuf[:, :I])
    Xq_o, xs_o, hb_o = oracle.silu_mul_quant(gu)
    assert np.array_equal(Xq_g.cpu().numpy(), Xq_o)
    assert np.array_equal(bf16_bits(hbuf[:, :I].contiguous()), hb_o)
    assert torch.all(hbuf[:, I:] == 2.0)


def test_silu_mul_quant_rejects_what_it_cannot_run():
    gu = torch.zeros((2, 2 * 28944), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sq.SQError) as e:  # two half-rows beyond one CTA's shared memory
        sq.silu_mul_quant_per_token(gu)
    assert e.value.status == 2
    with pytest.raises(sq.SQError) as e:  # bf16 rows only
        sq.silu_mul_quant_per_token(torch.zeros((2, 64), dtype=torch.float32, device="cuda"))
    assert e.value.status == 2


# ---------------------------------------------------------------------------
# whole workloads
# ---------------------------------------------------------------------------

def _gpu_inputs(inp):
    dev = lambda a: None if a is None else to_gpu(a)
    return ({k: dev(v) for k, v in inp.x.items()}, {k: dev(v) for k, v in inp.x_cal.items()},
            {k: dev(v) for k, v in inp.W.items()}, {k: dev(v) for k, v in inp.gamma.items()},
            {k: dev(v) for k, v in inp.beta.items()})


_FAMILY = {}


def _family_state(w, seed=0):
    """Weights, calibration and both sides' offline preparation, shared by
    every workload drawn from the same weights (the decode sweep reuses the
    prefill block's)."""
    fam = S._family(w)
    if fam not in _FAMILY:
        _FAMILY.clear()
        base = S.WORKLOADS[fam]
        inp = S.make_inputs(base, seed=seed, rows=1)
        _, xc, W, g, b = _gpu_inputs(inp)
        prep_g = {"xc": xc, "W": W, "g": g, "b": b}
        torch.cuda.synchronize()
        _FAMILY[fam] = (inp, prepare(base, inp), prep_g)
    return _FAMILY[fam]


def _check_workload(w, rows=None, seed=0):
    inp_w, prep_o, prep_g = _family_state(w, seed)
    inp = S.make_inputs(w, seed=seed, weights=False)
    inp.W = inp_w.W
    x = {k: to_gpu(v) for k, v in inp.x.items()}
    blk = pipeline.Block(w, w.M, "cuda")
    blk.prepare(prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"])
    out_g = blk.forward(x)
    torch.cuda.synchronize()
    # offline results: bit-exact on the full tensors
    for site in w.sites:
        so = prep_o["sites"][site.name]
        if site.smoothed:
            ties = scale_near_tie_channels(so["s64"])
            s_g = blk.s[site.name].cpu().numpy()
            diff = s_g.view(np.uint32) != so["s"].view(np.uint32)
            assert not np.any(diff & ~ties)
            if diff.any():
                pytest.skip("certified smoothing-factor near-tie: downstream not comparable")
            assert np.array_equal(blk.act_max[site.name].cpu().numpy().view(np.uint32),
                                  so["act_max"].view(np.uint32))
            assert np.array_equal(blk.gamma_f[site.name].cpu().numpy().view(np.uint32),
                                  so["gamma_f"].view(np.uint32))
            if so["beta_f"] is not None:
                assert np.array_equal(blk.beta_f[site.name].cpu().numpy().view(np.uint32),
                                      so["beta_f"].view(np.uint32))
    for lin in w.linears:
        lo = prep_o["linears"][lin.name]
        assert np.array_equal(blk.Wq[lin.name].cpu().numpy(), lo["Wq"]), lin.name
        assert np.array_equal(blk.w_scale[lin.name].cpu().numpy().view(np.uint32),
                              lo["w_scale"].view(np.uint32))
    # runtime path on the chosen rows
    rows = np.arange(w.M) if rows is None else np.asarray(rows)
    res = forward_rows(w, prep_o, inp, rows)
    idx = torch.from_numpy(rows).cuda()
    for site in w.sites:
        r = res["sites"][site.name]
        Xq_g = blk.xq[site.name][idx].cpu().numpy()
        xs_g = blk.xs[site.name][idx].cpu().numpy()
        compare_rows_quant(Xq_g, xs_g, r["Xq"], r["xs"], norm_near_tie_rows(r["x"], site.norm, w.eps))
    for lin in w.linears:
        o = res["linears"][lin.name]
        out_rows = bf16_bits(out_g[lin.name][idx].contiguous())
        d = bf16_ulp_diff(out_rows, o["out"])
        assert d.max() <= 1, (lin.name, int(d.max()))
        assert np.array_equal(out_rows, o["out"]), lin.name
    return blk


def test_workload_small_smoothed_linear():
    _check_workload(S.SMALL)


def test_workload_opt_prefill_qkv():
    _check_workload(S.OPT_QKV)


def _sample_rows(M, n=16, seed=7):
    r = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, M - 1], r.choice(M, size=min(n, M), replace=False)]))
    return rows


def test_workload_opt66b_mlp_sampled():
    _check_workload(S.OPT66B_MLP, rows=_sample_rows(S.OPT66B_MLP.M))


def test_workload_llama_block_prefill_sampled():
    _check_workload(S.LLAMA_BLOCK, rows=_sample_rows(S.LLAMA_BLOCK.M, n=8))


@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_workload_llama_block_decode(M):
    _check_workload(S.WORKLOADS["llama-block-8192-decode-m%d" % M])


@pytest.mark.parametrize("wname,granularity,fmt", [
    ("opt-prefill-rmsnorm-qkv-2048x4096x12288", "per_token", "int8"),
    ("llama-block-8192-decode-m1", "per_token", "int8"),
    ("llama-block-8192-decode-m8", "per_tensor_static", "int8"),
    ("llama-block-8192-decode-m8", "per_token", "fp8"),
    ("opt66b-mlp-layernorm-fc1-relu-fc2-4096x9216x36864", "per_token", "int8")])
def test_graph_replay_matches_eager_step(wname, granularity, fmt):
    """The benchmark replays the whole step as one CUDA graph, with
    independent work on a second stream: every buffer the step writes must
    come out bit-identical to the one-stream eager calls' results, both from
    the graph and from an eager overlapped step."""
    w = S.WORKLOADS[wname]
    inp_w, _, prep_g = _family_state(w)
    inp = S.make_inputs(w, seed=0, weights=False)
    x = {k: to_gpu(v) for k, v in inp.x.items()}
    blk = pipeline.Block(w, w.M, "cuda", granularity, fmt)
    blk.prepare(prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"])
    blk.forward(x)
    torch.cuda.synchronize()

    def snapshot():
        bufs = [blk.out, blk.xq, blk.xs, blk.Wq, blk.w_scale, blk.act_max, blk.s, blk.gamma_f]
        return {(i, k): v.clone() for i, d in enumerate(bufs) for k, v in d.items()
                if v is not None}

    eager = snapshot()
    for d in (blk.out, blk.xq, blk.Wq):
        for v in d.values():
            v.zero_()
    blk.step(prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"], x)
    torch.cuda.synchronize()
    for key, v in snapshot().items():
        assert torch.equal(v, eager[key]), ("step", key)
    graph = blk.capture(prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"], x)
    for d in (blk.out, blk.xq, blk.Wq):
        for v in d.values():
            v.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for key, v in snapshot().items():
        assert torch.equal(v, eager[key]), key
    del graph
    # the benchmark's offline graph (calibration on the second stream beside
    # the column maxima) prepares the same weights, factors and folds
    for d in (blk.Wq, blk.w_scale, blk.s, blk.gamma_f):
        for v in d.values():
            if v is not None:
                v.zero_()
    graph = pipeline.capture_prepare(blk, prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"])
    for d in (blk.Wq, blk.w_scale):
        for v in d.values():
            v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for key, v in snapshot().items():
        if key[0] in (3, 4, 5, 6, 7):  # Wq, w_scale, act_max, s, gamma_f
            assert torch.equal(v, eager[key]), ("prepare graph", key)
    del graph


# ---------------------------------------------------------------------------
# per-tensor variants (O2 dynamic, O3 static; per-tensor weights)
# ---------------------------------------------------------------------------

PT_KINDS = [("none_mult", oracle.NORM_NONE), ("rms", oracle.NORM_RMS),
            ("layer", oracle.NORM_LAYER)]


@pytest.mark.parametrize("shape", [(1, 64), (17, 4096), (300, 4112), (2048, 4096), (40, 28672)],
                         ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("kind", PT_KINDS, ids=lambda k: k[0])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_per_tensor_dynamic_matches_oracle(shape, kind, dtype):
    M, K = shape
    _, norm = kind
    x = _acts(M, K, dtype)
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if norm == oracle.NORM_LAYER else None
    gg, bb = to_gpu(g), (None if b is None else to_gpu(b))
    xg = to_gpu(x)
    if dtype == "f32" and K > 25600:  # fp32 rows this wide do not fit the row ring
        with pytest.raises(sq.SQError) as e:
            sq.norm_smooth_absmax(xg, norm, gg, bb)
        assert e.value.status == 2  # SQ_ERR_UNSUPPORTED, nothing launched
        return
    y_o, _, _ = oracle.norm(x, norm, g, b, 1e-5)
    ties = norm_near_tie_rows(x, norm, 1e-5)
    am_o = oracle.absmax_all(y_o)
    am_g = sq.norm_smooth_absmax(xg, norm, gg, bb)
    am_gv = np.float32(am_g.item())
    if not ties.any():
        assert am_gv.view(np.uint32) == am_o.view(np.uint32)
    else:
        assert abs(am_gv - am_o) <= 2 * np.spacing(am_o)
    # a second call keeps the running max
    sq.norm_smooth_absmax(xg[: max(1, M // 2)], norm, gg, bb, absmax=am_g)
    assert np.float32(am_g.item()) == am_gv
    # O2: one step from the tensor's own max (the GPU's, equal to the oracle's
    # unless a certified near-tie moved it)
    Xq_g, xs_g = sq.norm_smooth_quant_per_tensor(xg, norm, am_g, gg, bb)
    step = oracle.step_of(am_gv)
    Xq_o = oracle.quantize_with_step(y_o, step)
    xs_o = np.full(M, step, np.float32)
    compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, xs_o, ties)


@pytest.mark.parametrize("kind", PT_KINDS, ids=lambda k: k[0])
def test_per_tensor_static_saturates_like_the_oracle(kind):
    """O3: the step comes from a calibrated max below this tensor's own, so
    the largest values clamp at +-127."""
    _, norm = kind
    M, K = 257, 4096
    x = _acts(M, K, "bf16")
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) if norm == oracle.NORM_LAYER else None
    y_o, _, _ = oracle.norm(x, norm, g, b, 1e-5)
    am_static = np.float32(0.37 * oracle.absmax_all(y_o))
    Xq_g, xs_g = sq.norm_smooth_quant_per_tensor(
        to_gpu(x), norm, to_gpu(np.array([am_static], np.float32)), to_gpu(g),
        None if b is None else to_gpu(b))
    step = oracle.step_of(am_static)
    Xq_o = oracle.quantize_with_step(y_o, step)
    assert np.count_nonzero(np.abs(Xq_o) == 127) > 0
    compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, np.full(M, step, np.float32),
                       norm_near_tie_rows(x, norm, 1e-5))
    # a zero static max gives step 0 and all-zero codes
    Xq0, xs0 = sq.norm_smooth_quant_per_tensor(to_gpu(x), norm, torch.zeros(1, device="cuda"),
                                               to_gpu(g), None if b is None else to_gpu(b))
    assert not Xq0.any() and not xs0.any()


@pytest.mark.parametrize("NK", [(1, 16), (300, 4096), (129, 4112), (64, 28672)],
                         ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_per_tensor_weights_match_oracle(NK, dtype):
    N, K = NK
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    if N > 3:
        W[2] = 0.0
    if dtype == "bf16":
        W = S.to_bf16_bits(W)
    s = RNG.uniform(0.25, 4.0, K).astype(np.float32)
    if dtype == "f32" and K > 25600:  # fp32 rows this wide do not fit the row ring
        with pytest.raises(sq.SQError) as e:
            sq.smooth_quantize_weights_per_tensor(to_gpu(W), to_gpu(s))
        assert e.value.status == 2  # SQ_ERR_UNSUPPORTED, nothing launched
        return
    q_o, step_o = oracle.quantize_weights_per_tensor(W, s)
    am = torch.full((1,), 123.0, device="cuda")  # overwritten by the call
    Wq_g, ws_g = sq.smooth_quantize_weights_per_tensor(to_gpu(W), to_gpu(s), w_absmax=am)
    assert np.array_equal(Wq_g.cpu().numpy(), q_o)
    assert np.all(ws_g.cpu().numpy().view(np.uint32) == np.float32(step_o).view(np.uint32))
    assert oracle.step_of(am.item()) == step_o  # the call leaves max |W-hat| there


@pytest.mark.parametrize("granularity", ["per_tensor_dynamic", "per_tensor_static"])
@pytest.mark.parametrize("wname", ["smoothed-linear-16x64x64",
                                   "opt-prefill-rmsnorm-qkv-2048x4096x12288"])
def test_workload_per_tensor_granularity(wname, granularity):
    """The whole block with one activation scale per tensor and one weight
    scale per matrix, against the oracle's block on the full token batch."""
    w = S.WORKLOADS[wname]
    inp = S.make_inputs(w, seed=0)
    prep_o = prepare(w, inp, granularity)
    x, xc, W, g, b = _gpu_inputs(inp)
    blk = pipeline.Block(w, w.M, "cuda", granularity)
    blk.prepare(xc, W, g, b)
    out_g = blk.forward(x)
    torch.cuda.synchronize()
    for lin in w.linears:
        lo = prep_o["linears"][lin.name]
        ties = scale_near_tie_channels(prep_o["sites"][lin.site]["s64"]) \
            if prep_o["sites"][lin.site]["s64"] is not None else None
        if ties is not None and ties.any():
            pytest.skip("certified smoothing-factor near-tie")
        assert np.array_equal(blk.Wq[lin.name].cpu().numpy(), lo["Wq"]), lin.name
        assert np.array_equal(blk.w_scale[lin.name].cpu().numpy().view(np.uint32),
                              lo["w_scale"].view(np.uint32))
    # activation codes on every token (the per-tensor max needs them all); the
    # GEMM and epilogue on sampled tokens (these workloads read only inputs)
    rows = _sample_rows(w.M)
    for site in w.sites:
        st = prep_o["sites"][site.name]
        x_o = inp.x[site.name]
        if norm_near_tie_rows(x_o, site.norm, w.eps).any():
            pytest.skip("certified norm near-tie: the tensor-wide max is not comparable")
        Xq_o, step = oracle.norm_quant_per_tensor(x_o, site.norm, st["gamma_f"], st["beta_f"],
                                                  w.eps, absmax=st["static_absmax"])
        assert np.array_equal(blk.xq[site.name].cpu().numpy(), Xq_o), site.name
        assert np.all(blk.xs[site.name].cpu().numpy().view(np.uint32) ==
                      np.float32(step).view(np.uint32))
        for lin in w.linears_of(site.name):
            lo = prep_o["linears"][lin.name]
            acc = oracle.gemm_i64(Xq_o[rows], lo["Wq"])
            _, out_o = oracle.epilogue(acc, np.full(len(rows), step, np.float32), lo["w_scale"],
                                       lin.relu)
            idx = torch.from_numpy(rows).cuda()
            assert np.array_equal(bf16_bits(out_g[lin.name][idx].contiguous()), out_o), lin.name


# ---------------------------------------------------------------------------
# FP8 (e4m3) W8A8
# ---------------------------------------------------------------------------

F8_SHAPES = [(1, 16), (3, 48), (17, 64), (129, 4112), (64, 8192), (5, 28672), (1000, 4096)]


@pytest.mark.parametrize("shape", F8_SHAPES, ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("kind", KINDS, ids=lambda k: k[0])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fp8_norm_quant_matches_oracle(shape, kind, dtype):
    M, K = shape
    if dtype == "f32" and K > 25600:
        pytest.skip("fp32 rows above 25600 elements are unsupported")
    _, norm, with_params = kind
    x = _acts(M, K, dtype)
    if M > 2:
        x[1] = 0  # zero row: step 0, codes 0
    g = RNG.uniform(0.5, 1.5, K).astype(np.float32) if with_params else None
    b = (RNG.standard_normal(K) * 0.1).astype(np.float32) \
        if (with_params and norm == oracle.NORM_LAYER) else None
    Xq_o, xs_o = oracle.norm_quant_fp8(x, norm, g, b, 1e-5)
    Xq_g, xs_g = sq.norm_smooth_quant_per_token_fp8(
        to_gpu(x), norm, None if g is None else to_gpu(g), None if b is None else to_gpu(b), 1e-5)
    compare_rows_quant(Xq_g.cpu().numpy(), xs_g.cpu().numpy(), Xq_o, xs_o,
                       norm_near_tie_rows(x, norm, 1e-5))


@pytest.mark.parametrize("NK", [(1, 16), (300, 4096), (129, 4112), (64, 28672)],
                         ids=lambda s: "%dx%d" % s)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fp8_weights_match_oracle(NK, dtype):
    N, K = NK
    if dtype == "f32" and K > 25600:
        pytest.skip("fp32 rows above 25600 elements are unsupported")
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    W = S.to_bf16_bits(W) if dtype == "bf16" else W
    s = RNG.uniform(0.25, 4.0, K).astype(np.float32)
    Wq_o, ws_o = oracle.quantize_weights_fp8(W, s)
    Wq_g, ws_g = sq.smooth_quantize_weights_fp8(to_gpu(W), to_gpu(s))
    assert np.array_equal(Wq_g.cpu().numpy(), Wq_o)
    assert np.array_equal(ws_g.cpu().numpy().view(np.uint32), ws_o.view(np.uint32))


_F8_CODES = np.concatenate([np.arange(0, 0x7f), np.arange(0x80, 0xff)]).astype(np.uint8)
def fp8_acc_bound(K):
    """Relative bound (times sum |a b|) on |fp32 accumulator - exact sum| of an
    e4m3 GEMM over K: each 32-deep MMA step sums its (exact) products in an
    order and with roundings of the tensor cores' own -- at most 31 additions,
    each rounding by at most 2^-23 of a partial sum bounded by the step's
    sum |a b| -- and adds the result into the fp32 accumulator with one more
    rounding of at most 2^-23 of sum |a b|.  (The hardware exceeds a model
    with exact step sums, ceil(K/32) 2^-23, by up to 1.4x at K = 64.)  A
    stream-K decode tile adds its contributors' fp32 partial sums with one
    more rounding each; they are at most ceil(K/128), one per 128-deep
    block."""
    return (31 + max(1, (K + 31) // 32) + max(1, (K + 127) // 128)) * 2.0 ** -23


F8_GEMM_SHAPES = [(16, 64, 64), (3, 5, 16), (129, 257, 4112), (256, 512, 1024), (300, 777, 160),
                  (1024, 768, 2048), (2048, 1536, 512), (200, 15000, 64)]


@pytest.mark.parametrize("shape", F8_GEMM_SHAPES, ids=lambda s: "%dx%dx%d" % s)
@pytest.mark.parametrize("path", [1, 2, 3])
def test_fp8_gemm_accumulator_and_epilogue(shape, path):
    """The fp32 accumulator is the exact sum of the decoded products to within
    fp8_acc_bound: the tensor cores' order and rounding inside a 32-deep MMA
    step are theirs.  Given that accumulator, the bf16 epilogue is bit-exact."""
    M, N, K = shape
    if path == 2 and M > 256:
        pytest.skip("decode tiles take at most 256 tokens")
    A = RNG.choice(_F8_CODES, (M, K)).astype(np.uint8)
    B = RNG.choice(_F8_CODES, (N, K)).astype(np.uint8)
    exact = oracle.gemm_fp8(A, B)
    da = oracle.e4m3_decode(A).astype(np.float64)
    db = oracle.e4m3_decode(B).astype(np.float64)
    absum = np.abs(da) @ np.abs(db).T
    xs = (RNG.random(M) * 0.05 + 1e-3).astype(np.float32)
    ws = (RNG.random(N) * 0.002 + 1e-5).astype(np.float32)
    # decode tiles: stream-K (the default, fp32 partials added in CTA order)
    # and whole-K tiles; the prefill paths have whole-K tiles only
    for whole_k in ((False, True) if path == 2 else (False,)):
        acc = sq.fp8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "f32", path_hint=path,
                                  whole_k=whole_k)
        acc_g = acc.cpu().numpy()
        assert np.all(np.abs(acc_g.astype(np.float64) - exact) <= fp8_acc_bound(K) * absum)
        # the partial sums are added in a fixed order: the same bits on every run
        again = sq.fp8_gemm_dequant(to_gpu(A), to_gpu(B), None, None, "f32", path_hint=path,
                                    whole_k=whole_k)
        assert np.array_equal(again.cpu().numpy().view(np.uint32), acc_g.view(np.uint32))
        for relu in (False, True):
            out = sq.fp8_gemm_dequant(to_gpu(A), to_gpu(B), to_gpu(xs), to_gpu(ws),
                                      "bf16_relu" if relu else "bf16", path_hint=path,
                                      whole_k=whole_k)
            _, out_o = oracle.epilogue_f32(acc_g, xs, ws, relu)
            assert np.array_equal(bf16_bits(out), out_o)


def test_fp8_gemm_rejects_int8_only_epilogues():
    A = torch.zeros((8, 64), dtype=torch.uint8, device="cuda")
    B = torch.zeros((32, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.fp8_gemm_dequant(A, B, None, None, "i32",
                            out=torch.empty((8, 32), dtype=torch.int32, device="cuda"))
    assert e.value.status == 1
    with pytest.raises(sq.SQError) as e:  # the INT8 GEMM has no fp32 accumulator
        sq.w8a8_gemm_dequant(A.view(torch.int8), B.view(torch.int8), None, None, "f32",
                             out=torch.empty((8, 32), dtype=torch.float32, device="cuda"))
    assert e.value.status == 1


def test_fp8_decode_workspace_too_small_is_refused():
    A = torch.zeros((1, 4096), dtype=torch.uint8, device="cuda")
    B = torch.zeros((4096, 4096), dtype=torch.uint8, device="cuda")
    need = sq.gemm_workspace_size(1, 4096, 4096, 0)
    assert need > 16
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.fp8_gemm_dequant(A, B, None, None, "f32", path_hint=2, workspace=small)
    assert e.value.status == 7
    # a workspace of the planned size, and none at all (whole-K tiles), both run
    full = torch.empty(need, dtype=torch.uint8, device="cuda")
    for ws, whole in ((full, False), (None, True)):
        out = sq.fp8_gemm_dequant(A, B, None, None, "f32", path_hint=2, workspace=ws,
                                  whole_k=whole)
        assert torch.count_nonzero(out).item() == 0


def _check_workload_fp8(w, rows=None, seed=0):
    """The whole block with FP8 codes.  Offline results and every site's codes
    are bit-exact (a site fed by a GEMM is checked stage-wise, from the GPU's
    own bf16 output of that GEMM); each GEMM output is within the
    accumulation bound of the exact product of the codes, plus bf16 rounding."""
    inp_w, prep_o, prep_g = _family_state(w, seed)
    inp = S.make_inputs(w, seed=seed, weights=False)
    inp.W = inp_w.W
    x = {k: to_gpu(v) for k, v in inp.x.items()}
    blk = pipeline.Block(w, w.M, "cuda", fmt="fp8")
    blk.prepare(prep_g["xc"], prep_g["W"], prep_g["g"], prep_g["b"])
    out_g = blk.forward(x)
    torch.cuda.synchronize()
    wq = {}
    for lin in w.linears:
        so = prep_o["sites"][lin.site]
        if so["s64"] is not None and scale_near_tie_channels(so["s64"]).any():
            pytest.skip("certified smoothing-factor near-tie")
        Wq_o, ws_o = oracle.quantize_weights_fp8(inp.W[lin.name], so["s"])
        assert np.array_equal(blk.Wq[lin.name].cpu().numpy(), Wq_o), lin.name
        assert np.array_equal(blk.w_scale[lin.name].cpu().numpy().view(np.uint32),
                              ws_o.view(np.uint32))
        wq[lin.name] = (Wq_o, ws_o)
    rows = np.arange(w.M) if rows is None else np.asarray(rows)
    idx = torch.from_numpy(rows).cuda()
    for site in w.sites:
        so = prep_o["sites"][site.name]
        src = next((l.source for l in w.linears if l.site == site.name and l.source), None)
        if src:
            xs_in = bf16_bits(out_g[src][idx].contiguous())
            if site.act == "silu_mul":
                _, xs_in = oracle.silu_mul(xs_in)
        else:
            xs_in = np.ascontiguousarray(inp.x[site.name][rows])
        Xq_o, xsc_o = oracle.norm_quant_fp8(xs_in, site.norm, so["gamma_f"], so["beta_f"], w.eps)
        Xq_g = blk.xq[site.name][idx].cpu().numpy()
        xsc_g = blk.xs[site.name][idx].cpu().numpy()
        compare_rows_quant(Xq_g, xsc_g, Xq_o, xsc_o, norm_near_tie_rows(xs_in, site.norm, w.eps))
        for lin in w.linears_of(site.name):
            Wq_o, ws_o = wq[lin.name]
            exact = oracle.gemm_fp8(Xq_g, Wq_o)      # the GPU's codes (equal but for ties)
            absum = np.abs(oracle.e4m3_decode(Xq_g).astype(np.float64)) @ \
                np.abs(oracle.e4m3_decode(Wq_o).astype(np.float64)).T
            scale = xsc_g.astype(np.float64)[:, None] * ws_o.astype(np.float64)[None, :]
            o_exact = exact * scale
            if lin.relu:
                o_exact = np.maximum(o_exact, 0.0)
            o = bf16_bits(out_g[lin.name][idx].contiguous())
            o = (o.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            tol = fp8_acc_bound(site.K) * absum * scale + 2.0 ** -8 * np.abs(o_exact) + 1e-30
            assert np.all(np.abs(o - o_exact) <= tol), lin.name
    return blk


def test_workload_fp8_small_smoothed_linear():
    _check_workload_fp8(S.SMALL)


def test_workload_fp8_opt_prefill_qkv():
    _check_workload_fp8(S.OPT_QKV, rows=_sample_rows(S.OPT_QKV.M))


@pytest.mark.parametrize("M", [8, 128])
def test_workload_fp8_llama_block_decode(M):
    _check_workload_fp8(S.WORKLOADS["llama-block-8192-decode-m%d" % M])
