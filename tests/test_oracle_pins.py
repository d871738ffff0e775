"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests retypes the oracle's own formulas: each compares the
oracle with a worked example printed on the pages (``tests/golden``), a closed
form, an invariant, or an independent library routine (``math.fsum``, torch's
fp64 norms, numpy integer matmul, torch's bf16 cast).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_norm_b200 import synthetic as S

RNG = np.random.default_rng(1234)


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(np.maximum(x, np.float32(np.finfo(np.float32).tiny)))


# --------------------------------------------------------------------------
# exact summation (the norm statistics)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", range(6))
def test_exact_sum_matches_fsum(case):
    n = [1, 7, 100, 4096, 9216, 28672][case]
    x = RNG.standard_normal(n) * np.exp2(RNG.integers(-60, 60, n))
    assert oracle.exact_sum(x) == math.fsum(x)


def test_exact_sum_adversarial():
    cases = [
        [1e308, 1e308, -1e308, -1e308, 1.0],
        [1.0, 1e-300, -1.0],
        [2.0 ** 53, 1.0, -(2.0 ** 53)],
        [2.0 ** 53, 1.0, 1e-30],            # sticky bit breaks the tie upward
        [2.0 ** 53, 1.0],                   # exact tie, rounds to even
        [2.0 ** 53 + 2, 1.0],               # exact tie, rounds up to even
        [5e-324, 5e-324, 5e-324],
        [-3.5, 1.25, -0.0, 0.0],
        [0.1] * 10,
        list(-np.arange(1000, dtype=np.float64) ** 2),
    ]
    for c in cases:
        # exact rational sum, rounded once by CPython's correctly rounded int division
        exact = float(sum((Fraction(v) for v in c), Fraction(0)))
        assert oracle.exact_sum(np.array(c)) == exact, c


# --------------------------------------------------------------------------
# bf16 rounding of the epilogue output
# --------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    x = np.concatenate([
        RNG.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 3.0e38, -3.0e38,
                  1e-40, -1e-40, np.inf, -np.inf], np.float32),
        # exact ties between two bf16 neighbours
        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ])
    ours = oracle.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# norms (step 4) against torch's fp64 implementations
# --------------------------------------------------------------------------

def _torch_norm64(x32, kind, gamma, beta, eps):
    t = torch.from_numpy(x32.astype(np.float64))
    K = t.shape[1]
    g = torch.from_numpy(gamma.astype(np.float64)) if gamma is not None else None
    b = torch.from_numpy(beta.astype(np.float64)) if beta is not None else None
    if kind == oracle.NORM_RMS:
        return torch.nn.functional.rms_norm(t, (K,), g, eps).numpy()
    return torch.nn.functional.layer_norm(t, (K,), g, b, eps).numpy()


@pytest.mark.parametrize("kind", [oracle.NORM_RMS, oracle.NORM_LAYER])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_norm_matches_torch_fp64(kind, dtype):
    M, K = 37, 1000
    x = RNG.standard_normal((M, K)).astype(np.float32)
    x[:, [3, 500]] *= 60.0
    x[5] += 7.0  # a row with a large mean (cancellation in the variance)
    gamma = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    beta = (RNG.standard_normal(K) * 0.1).astype(np.float32) if kind == oracle.NORM_LAYER else None
    if dtype == "bf16":
        xin = S.to_bf16_bits(x)
        x32 = torch.from_numpy(xin.view(np.int16)).view(torch.bfloat16).float().numpy()
    else:
        xin, x32 = x, x
    y, mu, r = oracle.norm(xin, kind, gamma, beta, 1e-5)
    ref = _torch_norm64(x32, kind, gamma, beta, 1e-5)
    # the oracle rounds r (and mu) to fp32 and then does 2-4 fp32 operations
    err = np.abs(y.astype(np.float64) - ref)
    bound = 6 * _ulp32(ref).astype(np.float64) + 4 * np.finfo(np.float32).eps * np.abs(ref) \
        + (1e-6 if kind == oracle.NORM_LAYER else 0.0)
    assert np.all(err <= bound), float((err / bound).max())


def test_norm_closed_forms():
    K = 64
    c = np.float32(3.0)
    x = np.full((1, K), c, np.float32)
    y, _, r = oracle.norm(x, oracle.NORM_RMS, None, None, 0.0)
    assert r[0] == np.float32(1.0 / 3.0) and np.all(y == np.float32(c * np.float32(1.0 / 3.0)))
    # LayerNorm of a constant row is beta exactly (x - mu == 0)
    beta = RNG.standard_normal(K).astype(np.float32)
    y, mu, _ = oracle.norm(x, oracle.NORM_LAYER, None, beta, 1e-5)
    assert mu[0] == c and np.array_equal(y[0], beta)
    # all-zero RMS row: y = 0; r = 1/sqrt(eps)
    z = np.zeros((1, K), np.float32)
    y, _, r = oracle.norm(z, oracle.NORM_RMS, None, None, 1e-5)
    assert np.all(y == 0) and r[0] == np.float32(1.0 / math.sqrt(np.float64(np.float32(1e-5))))
    # NONE with a multiplier is an element-wise product
    g = RNG.uniform(0.5, 2, K).astype(np.float32)
    xx = RNG.standard_normal((3, K)).astype(np.float32)
    y, _, _ = oracle.norm(xx, oracle.NORM_NONE, g, None, 1e-5)
    assert np.array_equal(y, (xx * g[None, :]).astype(np.float32))


# --------------------------------------------------------------------------
# per-token quantisation (steps 5/6)
# --------------------------------------------------------------------------

def test_worked_example_token_row(golden_dir):
    g = _golden(golden_dir, "token_row_outliers.json")
    K = g["row_width"]
    lo, hi = g["ordinary_range"]
    row = RNG.uniform(lo, hi, K).astype(np.float32)
    row[[0, 1]] = [lo, hi]  # the range ends are present
    for ch, v in g["outliers"].items():
        row[int(ch)] = v
    q, step = oracle.quantize_rows(row[None, :])
    p, tol = g["printed"], g["printed_precision"]
    assert abs(step[0] - p["step_with_outliers"]) <= tol["step_with_outliers"]
    assert step[0] == np.float32(np.float32(60.0) / np.float32(127.0))
    ordinary = np.ones(K, bool)
    ordinary[[int(c) for c in g["outliers"]]] = False
    levels = np.unique(q[0, ordinary])
    assert levels.min() == -4 and levels.max() == 4
    assert len(levels) == p["ordinary_levels_with_outliers"]
    assert q[0, 2817] == -127 and q[0, 1512] == 95  # 45 / (60/127) = 95.25
    # without the outliers: step = 2/127, about 30 times finer
    row2 = row.copy()
    row2[~ordinary] = 0
    q2, step2 = oracle.quantize_rows(row2[None, :])
    assert abs(step2[0] - p["step_without_outliers"]) <= tol["step_without_outliers"]
    assert step2[0] == np.float32(np.float32(2.0) / np.float32(127.0))
    assert abs(step[0] / step2[0] - p["finer_factor"]) <= tol["finer_factor"]
    assert q2[0].min() == -127 and q2[0].max() == 127


def test_quantize_ties_round_half_even():
    # absmax 127 makes the step exactly 1.0, so y/step are the values themselves
    y = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 3.4999998]], np.float32)
    q, step = oracle.quantize_rows(y)
    assert step[0] == 1.0
    assert q[0].tolist() == [127, 0, 2, 2, 0, -2, -2, 126, -126, 3]


def test_quantize_clamp_and_zero_rows():
    # a subnormal absmax: step = fl32(2^-140 / 127) = 2^-147 and the quotient
    # 2^-140 / 2^-147 = 128 must clamp to 127 (and -128 to -127)
    a = np.float32(2.0 ** -140)
    y = np.array([[a, -a, 0.0], [0.0, 0.0, 0.0]], np.float32)
    q, step = oracle.quantize_rows(y)
    assert step[0] == np.float32(2.0 ** -147)
    assert q[0].tolist() == [127, -127, 0]
    assert step[1] == 0.0 and q[1].tolist() == [0, 0, 0]
    # the symmetric range never produces -128
    yy = RNG.standard_normal((200, 333)).astype(np.float32)
    qq, _ = oracle.quantize_rows(yy)
    assert qq.min() >= -127 and qq.max() <= 127
    assert np.all(np.abs(qq).max(axis=1) == 127)


def test_try_it_steps(golden_dir):
    g = _golden(golden_dir, "try_it_steps.json")
    for key, big in (("x_step", g["largest_abs_x"]), ("w_step", g["largest_abs_w"])):
        t = np.array([[big, -0.25 * big, 0.0]], np.float32)
        _, step = oracle.quantize_rows(t)
        assert abs(step[0] - g["printed"][key]) <= g["printed_precision"][key], key


# --------------------------------------------------------------------------
# per-tensor variants (O2 dynamic, O3 static)
# --------------------------------------------------------------------------

def test_per_tensor_one_row_is_the_per_token_quantiser():
    rng = np.random.default_rng(5)
    for K in (1, 7, 4096):
        y = (rng.standard_normal((1, K)) * rng.uniform(0.01, 100)).astype(np.float32)
        q_t, st_t = oracle.quantize_tensor(y)
        q_r, st_r = oracle.quantize_rows(y)
        assert st_t == st_r[0] and np.array_equal(q_t, q_r)


def test_per_tensor_step_is_the_largest_row_step_and_order_free():
    rng = np.random.default_rng(6)
    y = rng.standard_normal((37, 300)).astype(np.float32)
    y[11, 250] = -41.0
    q, step = oracle.quantize_tensor(y)
    _, row_steps = oracle.quantize_rows(y)
    assert step == row_steps.max() == np.float32(np.float32(41.0) / np.float32(127.0))
    assert q[11, 250] == -127 and np.abs(q).max() == 127
    perm_r, perm_c = rng.permutation(37), rng.permutation(300)
    q2, step2 = oracle.quantize_tensor(y[perm_r][:, perm_c])
    assert step2 == step and np.array_equal(q2, q[perm_r][:, perm_c])
    # every element with the one step, against numpy's float32 arithmetic
    ref = np.clip(np.rint((y / step).astype(np.float32)), -127, 127).astype(np.int8)
    assert np.array_equal(q, ref)


def test_try_it_per_tensor(golden_dir):
    """The demo quantises each whole tensor with one step: a 64 x 64 block of
    ordinary values whose largest magnitude is the printed max gives the
    printed step, and ordinary values use only a few levels."""
    g = _golden(golden_dir, "try_it_steps.json")
    rng = np.random.default_rng(7)
    for key, big in (("x_step", g["largest_abs_x"]), ("w_step", g["largest_abs_w"])):
        t = np.clip(rng.standard_normal((64, 64)), -2.5, 2.5).astype(np.float32) * np.float32(
            big / 84.3 if key == "w_step" else 1.0)
        t[17, 3] = np.float32(big)
        q, step = oracle.quantize_tensor(t)
        assert abs(step - g["printed"][key]) <= g["printed_precision"][key], key
        if key == "x_step":  # about +-4 of the 127 levels for the ordinary channels
            mask = np.ones_like(t, bool)
            mask[17, 3] = False
            assert np.abs(q[mask]).max() <= 4


def test_static_step_saturates_beyond_the_calibrated_range():
    # a static max of 127 gives step 1 exactly; values outside [-127, 127] clamp
    assert oracle.step_of(127.0) == np.float32(1.0)
    y = np.array([[254.0, -381.0, 127.0, -127.0, 63.5, 62.5, -0.5, 126.49]], np.float32)
    q = oracle.quantize_with_step(y, oracle.step_of(127.0))
    assert q.tolist() == [[127, -127, 127, -127, 64, 62, 0, 126]]
    assert not oracle.quantize_with_step(y, 0.0).any()
    # O3 on a norm: the static max comes from the calibration tokens through
    # the folded norm; a runtime row twice as large saturates
    rng = np.random.default_rng(8)
    xc = rng.standard_normal((16, 64)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, 64).astype(np.float32)
    yc, _, _ = oracle.norm(xc, oracle.NORM_NONE, g)
    am = oracle.absmax_all(yc)
    q_run, step = oracle.norm_quant_per_tensor(2 * xc, oracle.NORM_NONE, g, absmax=am)
    assert step == oracle.step_of(am)
    assert np.count_nonzero(np.abs(q_run) == 127) > 1


def test_per_tensor_weights():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((48, 96)) * 0.02).astype(np.float32)
    s = rng.uniform(0.5, 4.0, 96).astype(np.float32)
    q, step = oracle.quantize_weights_per_tensor(W, s)
    _, row_steps = oracle.quantize_weights(W, s)
    assert step == row_steps.max()
    assert np.array_equal(q, oracle.quantize_with_step(oracle.smooth_weights(W, s), step))


# --------------------------------------------------------------------------
# smoothing factors, fold and weight smoothing (steps 1-3)
# --------------------------------------------------------------------------

def _two_channel_weights():
    # nn.Linear layout [N_out=3, K_in=2]; column maxima are (0.2, 0.5) while
    # the row maxima are different, so a max over the wrong axis is caught
    return np.array([[0.2, -0.05], [-0.1, 0.5], [0.15, 0.3]], np.float32)


def test_worked_example_two_channels(golden_dir):
    g = _golden(golden_dir, "two_channel_alpha.json")
    act_max = np.array(g["act_max"], np.float32)
    W = _two_channel_weights()
    assert np.allclose(np.abs(W).max(axis=0), g["w_max"])
    token = act_max[None, :].copy()  # a token that reaches both channel maxima
    p, tol = g["printed"], g["printed_precision"]

    q0, st0 = oracle.quantize_rows(token)
    assert abs(st0[0] - p["unsmoothed"]["step"]) <= tol["step"]
    assert q0[0, 1] == p["unsmoothed"]["ch2_levels"]

    res = {}
    for alpha in (0.5, 0.8):
        s, _ = oracle.smooth_scales(act_max, [W], alpha)
        gf, _ = oracle.fold_norm(s)                      # gamma = 1: gamma' = 1/s
        y, _, _ = oracle.norm(token, oracle.NORM_NONE, gf, None)
        q, st = oracle.quantize_rows(y)
        What = oracle.smooth_weights(W, s)
        res[alpha] = (s, y, q, st, np.abs(What).max(axis=0))

    s, y, q, st, wmax = res[0.5]
    pa = p["alpha_0.5"]
    assert abs(float(np.abs(y).max()) - pa["step_numerator"]) <= tol["step_numerator"]
    assert abs(st[0] - pa["step"]) <= tol["step"]
    assert q[0, 1] == pa["ch2_levels"]
    s, y, q, st, wmax = res[0.8]
    pb = p["alpha_0.8"]
    assert q[0, 1] == pb["ch2_levels"]
    assert abs(wmax.max() / wmax.min() - pb["weight_spread"]) <= tol["weight_spread"]


def test_geometric_mean_at_half_alpha():
    """At alpha = 0.5 the smoothed activation and weight channel maxima are both
    sqrt(max|X_j| * max|W_j|) (the page 'LLM.int8() and SmoothQuant', going deeper)."""
    w = S.SMALL
    inp = S.make_inputs(w)
    xc = inp.x_cal["x"]
    W = inp.W["fc"]
    act_max = oracle.calibrate_absmax(xc, oracle.NORM_NONE)
    s, _ = oracle.smooth_scales(act_max, [W], 0.5)
    gf, _ = oracle.fold_norm(s)
    y, _, _ = oracle.norm(xc, oracle.NORM_NONE, gf, None)
    x_hat_max = np.abs(y).max(axis=0).astype(np.float64)
    w_hat_max = np.abs(oracle.smooth_weights(W, s)).max(axis=0).astype(np.float64)
    gm = np.sqrt(act_max.astype(np.float64) * np.abs(W).max(axis=0).astype(np.float64))
    assert np.all(np.abs(x_hat_max - gm) <= 4e-7 * gm)
    assert np.all(np.abs(w_hat_max - gm) <= 4e-7 * gm)


def test_equivalence_fp64():
    """Y = (X diag(s)^-1)(diag(s) W) to 1e-12 relative in fp64, with the oracle's s."""
    w = S.SMALL
    inp = S.make_inputs(w)
    X = inp.x["x"].astype(np.float64)
    W = inp.W["fc"]
    act_max = oracle.calibrate_absmax(inp.x_cal["x"], oracle.NORM_NONE)
    for alpha in (0.5, 0.8):
        s, _ = oracle.smooth_scales(act_max, [W], alpha)
        s = s.astype(np.float64)
        Y = X @ W.astype(np.float64).T
        Ys = (X / s[None, :]) @ (W.astype(np.float64) * s[None, :]).T
        assert np.max(np.abs(Ys - Y)) <= 1e-12 * np.max(np.abs(Y))


@pytest.mark.parametrize("kind", [oracle.NORM_RMS, oracle.NORM_LAYER])
def test_fold_keeps_the_layer_output(kind):
    """The folded norm times the smoothed weights reproduces the unsmoothed
    product within fp32 rounding; folding in the wrong direction does not."""
    M, K, N = 24, 256, 48
    x = RNG.standard_normal((M, K)).astype(np.float32)
    x[:, [7, 100]] *= 50
    gamma = RNG.uniform(0.5, 1.5, K).astype(np.float32)
    beta = (RNG.standard_normal(K) * 0.1).astype(np.float32) if kind == oracle.NORM_LAYER else None
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    act_max = oracle.calibrate_absmax(x, kind, gamma, beta)
    s, _ = oracle.smooth_scales(act_max, [W], 0.5)
    gf, bf = oracle.fold_norm(s, gamma, beta)
    y, _, _ = oracle.norm(x, kind, gamma, beta)
    yf, _, _ = oracle.norm(x, kind, gf, bf)
    What = oracle.smooth_weights(W, s)
    Y = y.astype(np.float64) @ W.astype(np.float64).T
    Yf = yf.astype(np.float64) @ What.astype(np.float64).T
    scale = np.abs(y).astype(np.float64) @ np.abs(W).astype(np.float64).T
    assert np.all(np.abs(Yf - Y) <= 1e-6 * scale + 1e-30)
    # the check discriminates: a fold in the wrong direction (gamma * s, so
    # the norm would emit y * s while the weights also carry s) fails it
    s64 = s.astype(np.float64)
    wrong = (y.astype(np.float64) * s64[None, :]) @ What.astype(np.float64).T
    assert np.max(np.abs(wrong - Y)) > 1e-2 * np.max(np.abs(Y))


def test_shared_scale_is_max_over_all_linears():
    """Linears reading one norm share s from the element-wise max of their
    weights: equal to treating them as one stacked weight."""
    K = 96
    act_max = np.abs(RNG.standard_normal(K)).astype(np.float32) * 10
    Ws = [(RNG.standard_normal((n, K)) * 0.02).astype(np.float32) for n in (16, 40, 8)]
    Ws[2][3, 11] = 0.9  # one large weight in the third matrix decides channel 11
    s_list, _ = oracle.smooth_scales(act_max, Ws, 0.8)
    s_cat, _ = oracle.smooth_scales(act_max, [np.concatenate(Ws, axis=0)], 0.8)
    s_first, _ = oracle.smooth_scales(act_max, [Ws[0]], 0.8)
    assert np.array_equal(s_list, s_cat)
    assert s_list[11] != s_first[11]


def test_smoothing_clamps():
    K = 4
    act_max = np.array([0.0, 1e-9, 5.0, 5.0], np.float32)
    W = np.array([[0.0, 0.3, 0.0, 1e-9]], np.float32)
    s, s64 = oracle.smooth_scales(act_max, [W], 0.5)
    eps = float(np.float32(1e-5))
    assert np.all(s >= np.float32(1e-5))
    # channel 0: both maxima clamp to eps -> s = eps^0.5 / eps^0.5 = 1
    assert abs(s64[0] - 1.0) < 1e-15
    # channel 2: w clamps to eps -> s = sqrt(5) / sqrt(eps)
    assert abs(s64[2] - math.sqrt(5.0) / math.sqrt(eps)) < 1e-12 * s64[2]


def test_calibration_running_max():
    inp = S.make_inputs(S.OPT_QKV, rows=8, weights=False)
    xc = inp.x_cal["attn_norm"]
    g = inp.gamma["attn_norm"]
    full = oracle.calibrate_absmax(xc, oracle.NORM_RMS, g)
    run = oracle.calibrate_absmax(xc[:200], oracle.NORM_RMS, g)
    run = oracle.calibrate_absmax(xc[200:], oracle.NORM_RMS, g, act_max=run)
    assert np.array_equal(full, run)
    x32 = torch.from_numpy(xc.view(np.int16)).view(torch.bfloat16).float().numpy()
    ref = np.abs(_torch_norm64(x32, oracle.NORM_RMS, g, None, 1e-5)).max(axis=0)
    assert np.all(np.abs(full - ref) <= 4 * _ulp32(ref))
    ch, _ = S.outlier_channels(S.OPT_QKV, "attn_norm")
    others = np.setdiff1d(np.arange(xc.shape[1]), ch)
    assert full[ch].min() > 3 * full[others].max()  # the outlier channels stand out


# --------------------------------------------------------------------------
# the integer GEMM and the epilogue (steps 7/8)
# --------------------------------------------------------------------------

def test_gemm_brute_force():
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (4, 6, 33)]:
        A = RNG.integers(-127, 128, (M, K)).astype(np.int8)
        B = RNG.integers(-127, 128, (N, K)).astype(np.int8)
        acc = oracle.gemm_i64(A, B)
        for m in range(M):
            for n in range(N):
                t = 0
                for k in range(K):
                    t += int(A[m, k]) * int(B[n, k])
                assert acc[m, n] == t


def test_gemm_matches_numpy_and_extremes():
    M, N, K = 17, 29, 4112
    A = RNG.integers(-127, 128, (M, K)).astype(np.int8)
    B = RNG.integers(-127, 128, (N, K)).astype(np.int8)
    assert np.array_equal(oracle.gemm_i64(A, B), A.astype(np.int64) @ B.astype(np.int64).T)
    A[:] = -127
    B[:] = -127
    assert np.all(oracle.gemm_i64(A, B) == 127 * 127 * K)


def test_epilogue_matches_float32_and_torch_bf16():
    M, N = 9, 31
    acc = RNG.integers(-(2 ** 31) + 1, 2 ** 31 - 1, (M, N)).astype(np.int64)
    acc[0, :5] = [0, 1, -1, 2 ** 24 + 1, -(2 ** 24) - 3]
    xs = (RNG.random(M) * 0.05).astype(np.float32)
    ws = (RNG.random(N) * 0.002).astype(np.float32)
    for relu in (False, True):
        o32, out = oracle.epilogue(acc, xs, ws, relu)
        ref = (acc.astype(np.float32) * xs[:, None]).astype(np.float32) * ws[None, :]
        ref = ref.astype(np.float32)
        if relu:
            ref = np.maximum(ref, np.float32(0))
        assert np.array_equal(o32, ref)
        tb = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(out, tb)


def test_epilogue_relu_of_negative_zero_is_positive_zero():
    """max(o32, 0) orders -0 below +0 (IEEE 754-2019 maximum): a negative
    accumulator times a zero token scale gives -0, which the ReLU maps to +0;
    without the ReLU the -0 stays."""
    acc = np.array([[-5, 0, 7]], np.int64)
    xs = np.zeros(1, np.float32)
    ws = np.ones(3, np.float32)
    o32, out = oracle.epilogue(acc, xs, ws, False)
    assert out[0, 0] == 0x8000 and out[0, 1] == 0 and out[0, 2] == 0
    o32, out = oracle.epilogue(acc, xs, ws, True)
    assert np.array_equal(out, np.zeros((1, 3), np.uint16))
    assert not np.signbit(o32).any()


# ---------------------------------------------------------------------------
# SiLU(gate) * up: the down projection's input
# ---------------------------------------------------------------------------

def test_exp_cw_within_a_few_ulps_of_float64_exp():
    t = np.concatenate([np.linspace(-87, 87, 400001, dtype=np.float32),
                        np.float32([0.0, -0.0, 1e-30, -1e-30, 0.5, -0.5, 1.0, -1.0, 86.99, -86.99]),
                        (np.arange(-125, 126) * np.log(2)).astype(np.float32)])
    e = oracle.exp_cw(t)
    ref = np.exp(t.astype(np.float64))
    rel = np.abs(e.astype(np.float64) / ref - 1.0)
    assert rel.max() < 4 * 2.0 ** -23, rel.max()
    assert oracle.exp_cw(np.float32([0.0]))[0] == np.float32(1.0)
    # the argument is clamped to [-87, 87]
    big = oracle.exp_cw(np.float32([87.0, 100.0, 1e30, -87.0, -100.0, -1e30]))
    assert big[0] == big[1] == big[2] and big[3] == big[4] == big[5]
    assert np.isfinite(big).all() and (big > 0).all()


def _gu(M, I, g_scale=3.0, seed=5):
    r = np.random.default_rng(seed)
    g = (r.standard_normal((M, I)) * g_scale).astype(np.float32)
    u = r.standard_normal((M, I)).astype(np.float32)
    return S.to_bf16_bits(np.concatenate([g, u], axis=1))


def test_silu_mul_against_the_float64_formula():
    M, I = 7, 4096
    gu = _gu(M, I)
    gf = (gu.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    g, u = gf[:, :I], gf[:, I:]
    exact = g * u / (1.0 + np.exp(-g))
    h32, hb = oracle.silu_mul(gu)
    nz = exact != 0
    rel = np.abs(h32[nz] / exact[nz] - 1.0)
    assert rel.max() < 8 * 2.0 ** -23, rel.max()
    # bf16 h within one bf16 ulp of the exact value (RNE of a nearly exact fp32)
    hv = (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.abs(exact[nz]))) - 7)
    assert np.all(np.abs(hv[nz] - exact[nz]) <= ulp)
    assert np.array_equal(hb, oracle.f32_to_bf16_bits(h32))
    # gate is the first half: swapping the halves changes the result
    swapped = np.concatenate([gu[:, I:], gu[:, :I]], axis=1)
    assert not np.array_equal(oracle.silu_mul(swapped)[1], hb)


def test_silu_mul_special_values():
    g = np.float32([0.0, 0.0, 80.0, 200.0, -80.0, -200.0, 1.0, -1.0])
    u = np.float32([1.0, -3.0, 1.5, 1.0, 1.0, 7.0, 0.0, 2.0])
    gu = S.to_bf16_bits(np.concatenate([g, u])[None, :])
    h32, hb = oracle.silu_mul(gu)
    h32 = h32[0]
    assert h32[0] == 0 and h32[1] == 0           # silu(0) = 0
    assert h32[2] == np.float32(120.0)           # sigma(80) rounds to 1
    assert h32[3] == np.float32(200.0)           # beyond the clamp: sigma = 1
    assert 0 < -h32[4] < 1e-30 and 0 < -h32[5] < 1e-30   # sigma(-80) ~ e^-80
    assert h32[6] == 0                           # up = 0
    ref = -1.0 / (1.0 + np.exp(1.0)) * 2.0       # silu(-1) * 2
    assert abs(h32[7] / ref - 1) < 4 * 2.0 ** -23


def test_silu_mul_quant_is_the_per_token_quant_of_bf16_h():
    M, I = 5, 320
    gu = _gu(M, I, seed=9)
    Xq, xs, hb = oracle.silu_mul_quant(gu)
    h = (hb.astype(np.uint32) << 16).view(np.float32)
    am = np.abs(h).max(axis=1)
    step = (am / np.float32(127)).astype(np.float32)   # numpy float32 division is IEEE
    assert np.array_equal(xs, step)
    q = np.clip(np.rint((h / step[:, None]).astype(np.float32)), -127, 127).astype(np.int8)
    assert np.array_equal(Xq, q)


# ---------------------------------------------------------------------------
# FP8 (e4m3) W8A8
# ---------------------------------------------------------------------------

def _e4m3_by_definition(c):
    """The value of an e4m3 ("fn") code from the format: bias 7, 3 mantissa bits."""
    sign = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_decode_follows_the_format_and_torch():
    d = oracle.e4m3_decode(np.arange(256))
    ref = np.array([_e4m3_by_definition(c) for c in range(256)])
    finite = ~np.isnan(ref)
    assert np.array_equal(d[finite].astype(np.float64), ref[finite])
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(d[finite], t[finite])
    assert d[0x7e] == 448 and d[0x01] == 2.0 ** -9 and d[0x08] == 2.0 ** -6


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    vals = np.sort(np.unique(np.abs(oracle.e4m3_decode(np.arange(0x7f)))))
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)  # exact in fp32
    codes = oracle.e4m3_encode(mids)
    lo = oracle.e4m3_encode(vals[:-1])
    hi = oracle.e4m3_encode(vals[1:])
    # a tie goes to the neighbour whose code (mantissa) is even
    expect = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(codes, expect)
    # just off the midpoints: nearest
    assert np.array_equal(oracle.e4m3_encode(np.nextafter(mids, np.float32(0))), lo)
    assert np.array_equal(oracle.e4m3_encode(np.nextafter(mids, np.float32(1e9))), hi)
    # saturation at 448 (464 is the tie with the non-finite 480: even -> 448)
    big = np.float32([448, 455, 464, 465, 1e6, 3e38, -448, -470, -3e38])
    assert list(oracle.e4m3_encode(big)) == [0x7e] * 6 + [0xfe] * 3
    assert list(oracle.e4m3_encode(np.float32([0.0, -0.0]))) == [0x00, 0x80]
    # random values inside the range: torch's cast (nearest even) agrees
    x = (np.random.default_rng(3).standard_normal(100000) * 40).astype(np.float32)
    x = np.concatenate([x[np.abs(x) < 448], np.float32(np.random.default_rng(4).uniform(
        -2.0 ** -5, 2.0 ** -5, 20000))])
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), t)


def test_fp8_row_quantisation():
    r = np.random.default_rng(11)
    y = (r.standard_normal((6, 4096)) * 3).astype(np.float32)
    y[0, 17] = 60.0                 # the row max: code 448 exactly
    y[1] = 0.0                      # zero row
    y[2] = 1e-37 * np.sign(y[2])    # step would be subnormal: zero row
    y[3, :] = np.abs(y[3, :])       # one sign
    q, step = oracle.quantize_rows_fp8(y)
    am = np.abs(y).max(axis=1)
    st = (am / np.float32(448)).astype(np.float32)
    st[st < np.finfo(np.float32).tiny] = 0
    assert np.array_equal(step, st)
    assert step[0] == np.float32(60) / np.float32(448) and q[0, 17] == 0x7e
    assert not q[1].any() and not q[2].any() and step[1] == step[2] == 0
    # every other row: the decoded code times the step is y to within half an
    # e4m3 spacing (relative 2^-4 for normals, 2^-10 * step absolute below)
    for m in (0, 3, 4, 5):
        dq = oracle.e4m3_decode(q[m]).astype(np.float64) * step[m]
        err = np.abs(dq - y[m])
        assert np.all(err <= np.abs(y[m]) * 2.0 ** -4 + 2.0 ** -10 * step[m] * 1.0001)
        assert np.abs(oracle.e4m3_decode(q[m])).max() == 448
    # the code is the cast of fl32(y * fl32(1 / step)) (numpy float32, torch cast)
    inv = (np.float32(1) / step[4]).astype(np.float32)
    t = torch.from_numpy((y[4] * inv).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q[4], t.view(torch.uint8).numpy())


def test_fp8_gemm_is_the_exact_sum():
    r = np.random.default_rng(12)
    codes = np.concatenate([np.arange(0, 0x7f), np.arange(0x80, 0xff)]).astype(np.uint8)
    A = r.choice(codes, (5, 40)).astype(np.uint8)
    B = r.choice(codes, (7, 40)).astype(np.uint8)
    acc = oracle.gemm_fp8(A, B)
    da = [[Fraction(_e4m3_by_definition(int(c))) for c in row] for row in A]
    db = [[Fraction(_e4m3_by_definition(int(c))) for c in row] for row in B]
    for m in range(5):
        for n in range(7):
            assert Fraction(acc[m, n]) == sum(x * w for x, w in zip(da[m], db[n]))
    # extremes: 448 * 448 * K exactly
    K = 4096
    full = oracle.gemm_fp8(np.full((1, K), 0x7e, np.uint8), np.full((2, K), 0xfe, np.uint8))
    assert np.all(full == -448.0 * 448.0 * K)


def test_fp8_epilogue_matches_float32_arithmetic():
    r = np.random.default_rng(13)
    acc = (r.standard_normal((9, 31)) * 1e4).astype(np.float32)
    xs = (r.random(9) * 0.05).astype(np.float32)
    ws = (r.random(31) * 0.002).astype(np.float32)
    for relu in (False, True):
        o32, out = oracle.epilogue_f32(acc, xs, ws, relu)
        ref = ((acc * xs[:, None]).astype(np.float32) * ws[None, :]).astype(np.float32)
        if relu:
            ref = np.where(ref > 0, ref, np.float32(0))
        assert np.array_equal(o32, ref)
        tb = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(out, tb)


# ---------------------------------------------------------------------------
# Comparator: LLM.int8()'s mixed-precision decomposition
# ---------------------------------------------------------------------------

def test_llmint8_worked_token_row(golden_dir):
    """[LLMint8] "one token through a layer": LLM.int8() sends channels 1512
    and 2817 (45 and -60, above tau = 6) through 16-bit; the remaining
    channels get the step 2/127, about 30 times finer than 60/127."""
    g = _golden(golden_dir, "token_row_outliers.json")
    K = g["row_width"]
    lo, hi = g["ordinary_range"]
    row = RNG.uniform(lo, hi, K).astype(np.float32)
    row[[0, 1]] = [lo, hi]
    for ch, v in g["outliers"].items():
        row[int(ch)] = v
    x = row[None, :]
    col = oracle.calibrate_absmax(x, oracle.NORM_NONE)
    mask, idx = oracle.llmint8_outliers(col, 6.0)
    assert list(idx) == sorted(int(c) for c in g["outliers"])
    assert mask[idx].tolist() == [0.0, 0.0] and mask.sum() == K - 2
    Xq, xs = oracle.norm_quant(x, oracle.NORM_NONE, mask, None)
    p, tol = g["printed"], g["printed_precision"]
    assert xs[0] == np.float32(np.float32(2.0) / np.float32(127.0))
    assert abs(xs[0] - p["step_without_outliers"]) <= tol["step_without_outliers"]
    assert Xq[0, idx].tolist() == [0, 0]
    assert Xq[0].min() == -127 and Xq[0].max() == 127


def test_llmint8_threshold_is_inclusive():
    col = np.array([6.0, np.nextafter(np.float32(6.0), np.float32(0.0)), 7.5, 0.0, 60.0],
                   np.float32)
    mask, idx = oracle.llmint8_outliers(col, 6.0)
    assert idx.tolist() == [0, 2, 4]
    assert mask.tolist() == [0.0, 1.0, 0.0, 1.0, 0.0]


def _small_layer(rng, M, N, K, scale=1.0):
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x, W


def test_llmint8_without_outliers_is_the_plain_w8a8_layer():
    rng = np.random.default_rng(11)
    x, W = _small_layer(rng, 9, 24, 64, scale=1.0)  # |x| < 6 everywhere
    assert np.abs(x).max() < 6.0
    Wq, ws = oracle.quantize_weights(W, None)
    r = oracle.llmint8_linear(x, Wq, ws, W)
    assert r["idx"].size == 0 and (r["mask"] == 1.0).all()
    _, _, acc, o32, out = oracle.linear(x, oracle.NORM_NONE, None, None, 1e-5, Wq, ws)
    assert np.array_equal(r["acc"], acc)
    assert np.array_equal(r["y"].view(np.uint32), o32.view(np.uint32))
    assert np.array_equal(r["out"], out)


def test_llmint8_sixteen_bit_lane_is_an_exact_dot_product():
    """Integer-valued inputs: every product and partial sum is exact, so the
    16-bit lane is the integer dot product over the outlier channels, and
    with every channel an outlier (tau = 0: every max is >= 0) the INT8 lane is
    empty (zero codes, zero steps) and y is that dot product."""
    rng = np.random.default_rng(12)
    M, N, K = 5, 7, 48
    x = rng.integers(-40, 41, (M, K)).astype(np.float32)
    W = rng.integers(-9, 10, (N, K)).astype(np.float32)
    Wq, ws = oracle.quantize_weights(W, None)
    r = oracle.llmint8_linear(x, Wq, ws, W, tau=0.0)
    assert r["idx"].tolist() == list(range(K))
    assert (r["Xq"] == 0).all() and (r["x_scale"] == 0).all() and (r["o32"] == 0).all()
    exact = x.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(r["y"], exact.astype(np.float32))
    # a chosen outlier set: the lane sums only those channels
    col = np.zeros(K, np.float32)
    chosen = [3, 17, 40]
    col[chosen] = 10.0
    _, idx = oracle.llmint8_outliers(col, 6.0)
    y, _ = oracle.llmint8_combine(np.zeros((M, N), np.float32), x, W, idx)
    assert np.array_equal(y, (x[:, chosen].astype(np.int64) @
                              W[:, chosen].astype(np.int64).T).astype(np.float32))


def test_llmint8_sixteen_bit_lane_in_fp64_order():
    """Real-valued bf16 inputs: the lane equals a sequential fp64 sum of the
    exact products in ascending channel order, rounded once to fp32."""
    rng = np.random.default_rng(13)
    M, N, K = 3, 4, 64
    x = S.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * 9)
    W = S.to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    wf = (W.astype(np.uint32) << 16).view(np.float32)
    idx = np.array([1, 5, 6, 30, 63], np.int32)
    y, out = oracle.llmint8_combine(np.zeros((M, N), np.float32), x, W, idx)
    for m in range(M):
        for n in range(N):
            s = 0.0
            for j in idx:
                s = s + float(xf[m, j]) * float(wf[n, j])
            assert y[m, n] == np.float32(s)


def test_llmint8_is_finer_than_plain_int8_on_outlier_channels():
    """The pages' claim in numbers: with a few outlier channels, the plain
    per-token INT8 layer's output error is several times LLM.int8()'s."""
    rng = np.random.default_rng(14)
    M, N, K = 32, 64, 256
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, [7, 200]] *= np.float32(50.0)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, ws = oracle.quantize_weights(W, None)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    _, _, _, o32, _ = oracle.linear(x, oracle.NORM_NONE, None, None, 1e-5, Wq, ws)
    r = oracle.llmint8_linear(x, Wq, ws, W)
    assert r["idx"].tolist() == [7, 200]
    e_plain = np.linalg.norm(o32 - ref) / np.linalg.norm(ref)
    e_int8 = np.linalg.norm(r["y"] - ref) / np.linalg.norm(ref)
    assert e_int8 * 5 < e_plain


def test_llmint8_layer_is_the_exact_product_on_integer_data():
    """A closed form of the whole decomposition: integer inputs whose ordinary
    channels lie in [-127, 127] with a +-127 in every token row and every
    weight row (token and weight steps fl32(127 / 127) = 1, so codes equal the
    values), outlier channels at 200 or more (tau = 200 sends exactly them to
    the 16-bit lane).  Both lanes are then exact integer sums below 2^24 and
    the bf16 output is the rounding of the exact product x W^T.  A lane
    counted twice, an outlier left in the INT8 lane (its step would no longer
    be 1) or a dropped lane fails."""
    import torch
    rng = np.random.default_rng(15)
    M, N, K = 6, 10, 40
    out_ch = [4, 21, 33]
    x = rng.integers(-127, 128, (M, K)).astype(np.float32)
    x[:, [0, 1]] = 0.0
    x[:, 0] = np.where(np.arange(M) % 2 == 0, 127.0, -127.0)
    x[:, out_ch] = rng.integers(200, 400, (M, len(out_ch))) * rng.choice([-1, 1], (M, len(out_ch)))
    W = rng.integers(-127, 128, (N, K)).astype(np.float32)
    W[:, 1] = 127.0
    Wq, ws = oracle.quantize_weights(W, None)
    assert (ws == 1.0).all() and np.array_equal(Wq.astype(np.float32), W)
    r = oracle.llmint8_linear(x, Wq, ws, W, tau=200.0)
    assert r["idx"].tolist() == out_ch
    assert (r["x_scale"] == 1.0).all()
    exact = x.astype(np.int64) @ W.astype(np.int64).T
    assert np.abs(exact).max() < 2 ** 24
    assert np.array_equal(r["y"], exact.astype(np.float32))
    want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(r["out"], want.view(torch.int16).numpy().view(np.uint16))
