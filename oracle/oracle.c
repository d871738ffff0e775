/*
 * oracle.c -- plain, slow, obviously-correct CPU restatement of the
 * SmoothQuant W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity oracle for the CUDA
 * library: only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark load it.  It shares no code, header, table or helper with the
 * CUDA path, and the CUDA path never calls it.
 *
 * Every function states the passage of the source pages it follows.  Page
 * titles used in the citations:
 *   [SQ-depth]  "SmoothQuant, in depth: where the scales fold, how calibration
 *               feeds them, and a W8A8 pipeline you can ship"
 *   [LLMint8]   "LLM.int8() and SmoothQuant"
 *   [SQ-expl]   "SmoothQuant explained"
 *   [SQ-map]    "SmoothQuant: Accurate and Efficient PTQ" (interactive explainer)
 *   [SQ-rec]    "SmoothQuant (W8A8 via offline outlier migration)" (research record)
 *
 * Arithmetic conventions (the pages fix none of them; these are the readings
 * this project adopts):
 *   - fl32(.) / fl64(.) are single IEEE operations rounded to nearest-even;
 *     the file is compiled with -ffp-contract=off and without fast-math, so
 *     every C operator below is exactly one such rounding.
 *   - Row statistics of a norm are computed from the EXACT sums of x and x^2
 *     (an exact fixed-point accumulator, then one rounding to fp64).
 *   - Quantisation is symmetric absmax INT8: step = fl32(absmax / 127),
 *     q = clamp(rne(fl32(y / step)), -127, 127); an all-zero row has step 0
 *     and q = 0.
 *   - The integer GEMM is exact in int64.
 *
 * Parity status of each function is stated in its comment.  The pins live in
 * tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype / norm codes of this oracle (its own numbering, documented in
 * oracle/__init__.py; they are not taken from any other header). */
#define OR_F32 0
#define OR_BF16 1

#define OR_NORM_NONE 0
#define OR_NORM_RMS 1
#define OR_NORM_LAYER 2

/* ------------------------------------------------------------------------ */
/* Element access                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static float bf16_bits_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static float load_elem(const void* base, int dtype, int64_t idx) {
  if (dtype == OR_BF16) return bf16_bits_to_f32(((const uint16_t*)base)[idx]);
  return ((const float*)base)[idx];
}

/* Round a binary32 to bfloat16, round-to-nearest-even on the 16 dropped
 * bits; NaN stays NaN.  Written from the definition of RNE truncation. */
uint16_t oracle_f32_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
    return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
  }
  uint32_t lsb = (u >> 16) & 1u;
  uint32_t rounded = u + 0x7fffu + lsb;
  return (uint16_t)(rounded >> 16);
}

/* ------------------------------------------------------------------------ */
/* Exact summation of binary64 terms                                         */
/* ------------------------------------------------------------------------ */
/*
 * A fixed-point big integer that holds any sum of binary64 values exactly
 * (a long accumulator in the sense of Kulisch).  Bit 0 of the accumulator has
 * weight 2^EXACC_EMIN; limbs hold 32 bits of payload each in int64 storage so
 * that up to 2^30 terms can be added before carries must be propagated.
 */
#define EXACC_EMIN (-1152)
#define EXACC_LIMBS 72 /* 72*32 = 2304 bits: weights 2^-1152 .. 2^1151 */

typedef struct {
  int64_t limb[EXACC_LIMBS];
} exacc_t;

static void exacc_clear(exacc_t* a) { memset(a, 0, sizeof *a); }

static void exacc_add(exacc_t* a, double d) {
  if (d == 0.0) return;
  int e;
  double fr = frexp(d, &e);              /* d = fr * 2^e, 0.5 <= |fr| < 1 */
  int64_t m = (int64_t)ldexp(fr, 53);    /* exact: 53-bit integer mantissa */
  e -= 53;                               /* d = m * 2^e */
  int neg = m < 0;
  uint64_t mag = (uint64_t)(neg ? -m : m);
  int pos = e - EXACC_EMIN;              /* bit position of m's lsb */
  int li = pos / 32, off = pos % 32;
  unsigned __int128 v = ((unsigned __int128)mag) << off; /* < 2^85 */
  for (int k = 0; k < 3 && li + k < EXACC_LIMBS; ++k) {
    int64_t chunk = (int64_t)(uint64_t)(v & 0xffffffffu);
    a->limb[li + k] += neg ? -chunk : chunk;
    v >>= 32;
  }
}

static void exacc_carry(exacc_t* a) {
  /* afterwards limbs 0..L-2 lie in [0, 2^32); the top limb carries the sign */
  for (int i = 0; i < EXACC_LIMBS - 1; ++i) {
    int64_t c = a->limb[i] >> 32; /* arithmetic shift = floor division */
    a->limb[i] -= c * 4294967296LL;
    a->limb[i + 1] += c;
  }
}

/* Correctly rounded (nearest-even) binary64 value of the exact sum. */
static double exacc_round(const exacc_t* a_in) {
  exacc_t a = *a_in;
  exacc_carry(&a);
  int neg = a.limb[EXACC_LIMBS - 1] < 0;
  if (neg) { /* magnitude of a negative sum: negate every limb, re-carry */
    for (int i = 0; i < EXACC_LIMBS; ++i) a.limb[i] = -a.limb[i];
    exacc_carry(&a);
  }
  int h = EXACC_LIMBS - 1;
  while (h >= 0 && a.limb[h] == 0) --h;
  if (h < 0) return 0.0;
  /* the top three limbs (the highest one non-zero) and a sticky bit for the
   * rest; h >= 2 for every sum of binary64 terms (see EXACC_EMIN) */
  int base = h - 2;
  unsigned __int128 v = 0;
  for (int i = h; i >= base; --i) v = (v << 32) | (uint64_t)a.limb[i];
  int sticky = 0;
  for (int i = base - 1; i >= 0; --i)
    if (a.limb[i]) { sticky = 1; break; }
  int nbits = 0;
  for (unsigned __int128 t = v; t; t >>= 1) ++nbits;
  int shift = nbits - 53; /* in [12, 43]: bits 64..95 hold the top limb */
  unsigned __int128 keep = v >> shift;
  unsigned __int128 rem = v & ((((unsigned __int128)1) << shift) - 1);
  unsigned __int128 half = ((unsigned __int128)1) << (shift - 1);
  int round_up = rem > half || (rem == half && (sticky || (keep & 1)));
  keep += round_up; /* may reach 2^53, still exact in binary64 */
  double r = ldexp((double)(uint64_t)keep, EXACC_EMIN + 32 * base + shift);
  return neg ? -r : r;
}

/* Exposed for the pins: correctly rounded sum of n binary64 terms. */
double oracle_exact_sum(const double* x, int64_t n) {
  exacc_t a;
  exacc_clear(&a);
  for (int64_t i = 0; i < n; ++i) exacc_add(&a, x[i]);
  return exacc_round(&a);
}

/* ------------------------------------------------------------------------ */
/* Step 4: the norm that feeds the smoothed Linear                           */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "Where the scales go in a decoder block": the input of the
 * smoothed projections is the output of a LayerNorm or RMSNorm whose final
 * element-wise multiply by gamma (and add of beta) carries the folded 1/s.
 * The pages name the norms but not their formulas; the standard definitions
 * are used:
 *   RMSNorm:   y_k = x_k / sqrt(mean(x^2) + eps) * gamma_k
 *   LayerNorm: y_k = (x_k - mean(x)) / sqrt(var(x) + eps) * gamma_k + beta_k
 *              (biased variance)
 * and NONE:   y_k = x_k, or x_k * gamma_k when a per-channel multiplier is
 *              given (a Linear with no norm in front whose 1/s is applied as
 *              a multiplier).
 * Precision: S1 = sum x, S2 = sum x^2 exact, rounded once to fp64;
 *   RMS:  v = fl64(fl64(S2/K) + eps); r = fl32(fl64(1/fl64(sqrt(v))))
 *         y = fl32(fl32(x*r) * gamma)
 *   LN:   mu64 = fl64(S1/K); var = max(0, fl64(fl64(S2/K) - fl64(mu64*mu64)))
 *         r = fl32(fl64(1/fl64(sqrt(fl64(var+eps))))); mu = fl32(mu64)
 *         y = fl32(fl32(fl32(fl32(x-mu)*r)*gamma) + beta)
 * gamma == NULL means gamma = 1; beta == NULL means beta = 0 (LN only).
 * The per-row (mu, r) are written to mu_out / r_out when non-NULL.
 * Parity: pinned against torch's fp64 rms_norm / layer_norm (a library
 * routine) to within fp32 rounding, and by closed forms (constant rows).
 */
int oracle_norm(const void* x, int dtype, int64_t M, int64_t K, int64_t ldx,
                int norm, const float* gamma, const float* beta, float eps,
                float* y, float* mu_out, float* r_out) {
  if (K <= 0 || M < 0) return -1;
  for (int64_t m = 0; m < M; ++m) {
    const int64_t row = m * ldx;
    float mu = 0.0f, r = 1.0f;
    if (norm == OR_NORM_RMS || norm == OR_NORM_LAYER) {
      exacc_t s1, s2;
      exacc_clear(&s1);
      exacc_clear(&s2);
      for (int64_t k = 0; k < K; ++k) {
        double xv = (double)load_elem(x, dtype, row + k);
        exacc_add(&s1, xv);
        exacc_add(&s2, xv * xv); /* exact: a binary32 squared fits binary64 */
      }
      double S1 = exacc_round(&s1), S2 = exacc_round(&s2);
      double ms = S2 / (double)K;
      double v;
      if (norm == OR_NORM_RMS) {
        v = ms + (double)eps;
      } else {
        double mu64 = S1 / (double)K;
        double var = ms - mu64 * mu64;
        if (var < 0.0) var = 0.0;
        v = var + (double)eps;
        mu = (float)mu64;
      }
      double rs = 1.0 / sqrt(v);
      r = (float)rs;
    }
    if (mu_out) mu_out[m] = mu;
    if (r_out) r_out[m] = r;
    for (int64_t k = 0; k < K; ++k) {
      float xv = load_elem(x, dtype, row + k);
      float g = gamma ? gamma[k] : 1.0f;
      float out;
      if (norm == OR_NORM_RMS) {
        float t = xv * r;
        out = t * g;
      } else if (norm == OR_NORM_LAYER) {
        float c = xv - mu;
        float t = c * r;
        float u = t * g;
        out = beta ? u + beta[k] : u;
      } else {
        out = gamma ? xv * g : xv;
      }
      y[m * K + k] = out;
    }
  }
  return 0;
}

/* Exact row sums, each rounded once to fp64: S1 = sum x, S2 = sum x^2 and
 * SA = sum |x|.  Used by the tests to bound how far a differently ordered
 * fp64 reduction can move the norm statistics (near-tie certification). */
void oracle_row_sums(const void* x, int dtype, int64_t M, int64_t K, int64_t ldx,
                     double* S1, double* S2, double* SA) {
  for (int64_t m = 0; m < M; ++m) {
    exacc_t a1, a2, aa;
    exacc_clear(&a1);
    exacc_clear(&a2);
    exacc_clear(&aa);
    for (int64_t k = 0; k < K; ++k) {
      double xv = (double)load_elem(x, dtype, m * ldx + k);
      exacc_add(&a1, xv);
      exacc_add(&a2, xv * xv);
      exacc_add(&aa, fabs(xv));
    }
    S1[m] = exacc_round(&a1);
    S2[m] = exacc_round(&a2);
    SA[m] = exacc_round(&aa);
  }
}

/* ------------------------------------------------------------------------ */
/* Steps 5 and 6: symmetric absmax INT8 quantisation of rows                  */
/* ------------------------------------------------------------------------ */
/*
 * [LLMint8] "Try it": INT8 step = max / 127; [LLMint8] "example - one token
 * through a layer": one INT8 scale for the whole row, step 60/127.
 * [SQ-depth] "Granularity": per-token dynamic activation scales and
 * per-output-channel weight scales, both applied in the GEMM epilogue.
 * Each row of y gets step = fl32(max_k |y_k| / 127) and
 * q_k = clamp(rne(fl32(y_k / step)), -127, 127).  A row whose absmax is 0,
 * or whose step underflows to 0, has step 0 and q = 0.
 * Parity: pinned by the worked 4096-wide example (step 60/127, about nine
 * levels for ordinary values), hand-built ties and the clamp boundary.
 */
static int8_t quantize_one(float v, float step) {
  if (step == 0.0f) return 0;
  float t = v / step;         /* fl32 division */
  float q = nearbyintf(t);    /* default mode: round half to even */
  if (q > 127.0f) q = 127.0f;
  if (q < -127.0f) q = -127.0f;
  return (int8_t)q;
}

void oracle_quantize_rows(const float* y, int64_t M, int64_t K, int8_t* q,
                          float* step_out) {
  for (int64_t m = 0; m < M; ++m) {
    const float* row = y + m * K;
    float am = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(row[k]);
      if (a > am) am = a;
    }
    float step = am / 127.0f;
    step_out[m] = step;
    for (int64_t k = 0; k < K; ++k) q[m * K + k] = quantize_one(row[k], step);
  }
}

/* ------------------------------------------------------------------------ */
/* Per-tensor variants (O2 dynamic, O3 static)                               */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "Granularity: O1, O2, O3 and what kernels run today": the paper's
 * three levels all use per-tensor weight scales; O2 shares one dynamic
 * activation scale across the whole tensor, O3 uses a static activation
 * scale fixed offline (the page warns that O3's static scales break on inputs
 * outside the calibration distribution: values beyond it saturate).
 * [LLMint8] "Try it": plain INT8 with one scale per tensor, step = max / 127.
 * oracle_absmax_all: the running max over every element of |y| (in/out, the
 * caller starts it at zero).  oracle_quantize_with_step: every element with
 * the same step, q = clamp(rne(fl32(y / step)), -127, 127), step 0 -> q 0.
 * O2 is step = fl32(absmax_all / 127) on the tensor itself; O3 the same on
 * the calibration batch passed through the runtime (folded) norm, then
 * applied to every later tensor.
 * Parity: pinned by the one-row case (identical to the per-row quantiser),
 * the "Try it" steps, and the clamp of values beyond a static range.
 */
void oracle_absmax_all(const float* y, int64_t M, int64_t K, float* absmax) {
  float am = *absmax;
  for (int64_t i = 0; i < M * K; ++i) {
    float a = fabsf(y[i]);
    if (a > am) am = a;
  }
  *absmax = am;
}

float oracle_step_of(float absmax) { return absmax / 127.0f; }

void oracle_quantize_with_step(const float* y, int64_t M, int64_t K, float step, int8_t* q) {
  for (int64_t i = 0; i < M * K; ++i) q[i] = quantize_one(y[i], step);
}

/* ------------------------------------------------------------------------ */
/* Step 1: calibration -- running per-channel absmax of the norm output      */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "The calibration data flow": for every smoothed layer, record
 * the running maximum over all calibration tokens of |x_j| at the Linear's
 * input, combining batches with an element-wise maximum.  The Linear's input
 * is the (unsmoothed) norm output, computed by oracle_norm.
 * act_max is in/out: the caller starts it at zero.
 * Parity: pinned by the running-max property (two calls equal one call on
 * the concatenation) and by numpy's column max of |y|.
 */
int oracle_calibrate_absmax(const void* x, int dtype, int64_t M, int64_t K,
                            int64_t ldx, int norm, const float* gamma,
                            const float* beta, float eps, float* act_max) {
  float* y = (float*)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1) * (size_t)K);
  if (!y) return -2;
  int rc = oracle_norm(x, dtype, M, K, ldx, norm, gamma, beta, eps, y, NULL, NULL);
  if (rc == 0) {
    for (int64_t m = 0; m < M; ++m)
      for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(y[m * K + k]);
        if (a > act_max[k]) act_max[k] = a;
      }
  }
  free(y);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* Step 2: smoothing factors                                                 */
/* ------------------------------------------------------------------------ */
/*
 * [LLMint8] "going deeper": s_j = max_t|X_tj|^alpha / max_k|W_jk|^(1-alpha),
 * with X-hat = X diag(s)^-1 and W-hat = diag(s) W.
 * [SQ-depth] "Where the scales go in a decoder block": the projections that
 * read one norm share one s, computed from the element-wise maximum of their
 * weight matrices.  [SQ-depth] "The calibration data flow" (the printed
 * smoothing routine): both maxima are clamped below at eps before the powers
 * and s itself is clamped below at eps.
 * Weights are nn.Linear-shaped [N, K] (K = input channel), so max|W_j| is
 * the maximum over the output dimension n of column j.
 * Computation: w_j = max_L max_n |W^L[n, j]| (exact); in fp64:
 *   s_j = pow(max(a_j, eps), alpha) / pow(max(w_j, eps), 1 - alpha),
 *   s_j = max(s_j, eps); stored as fl32(s_j).
 * s64_out (nullable) receives the fp64 value before the final rounding.
 * Parity: pinned by the pages' two-channel worked example (alpha 0.5 and
 * 0.8) and by the alpha = 0.5 geometric-mean property.
 */
int oracle_smooth_scales(const float* act_max, const void* const* W,
                         const int64_t* N, int num_w, int dtype, int64_t K,
                         double alpha, float eps, float* s, double* s64_out) {
  if (num_w < 1 || K <= 0) return -1;
  for (int64_t j = 0; j < K; ++j) {
    float w = 0.0f;
    for (int l = 0; l < num_w; ++l)
      for (int64_t n = 0; n < N[l]; ++n) {
        float a = fabsf(load_elem(W[l], dtype, n * K + j));
        if (a > w) w = a;
      }
    double a_c = (double)act_max[j] > (double)eps ? (double)act_max[j] : (double)eps;
    double w_c = (double)w > (double)eps ? (double)w : (double)eps;
    double sj = pow(a_c, alpha) / pow(w_c, 1.0 - alpha);
    if (sj < (double)eps) sj = (double)eps;
    if (s64_out) s64_out[j] = sj;
    s[j] = (float)sj;
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 3: fold 1/s into the norm, s into the weights                        */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "Where the scales go in a decoder block": dividing gamma (and
 * beta, for LayerNorm) by s makes the norm emit X/s with no extra kernel.
 * [LLMint8] "Fix 2": divide activation channel j by s_j and multiply row j of
 * W (in the d x o orientation; column j of an nn.Linear weight) by s_j.
 * gamma' = fl32(gamma / s) (gamma == NULL means gamma = 1),
 * beta'  = fl32(beta / s).
 * Parity: pinned by the equivalence Y = (X diag(s)^-1)(diag(s) W).
 */
void oracle_fold_norm(const float* s, const float* gamma, const float* beta,
                      int64_t K, float* gamma_f, float* beta_f) {
  for (int64_t j = 0; j < K; ++j) {
    float g = gamma ? gamma[j] : 1.0f;
    gamma_f[j] = g / s[j];
    if (beta && beta_f) beta_f[j] = beta[j] / s[j];
  }
}

/* W-hat[n, j] = fl32(W[n, j] * s_j); s == NULL means s = 1 (an unsmoothed
 * Linear, [SQ-depth] "Where the scales go": o_proj / down_proj). */
void oracle_smooth_weights(const void* W, int dtype, int64_t N, int64_t K,
                           int64_t ldw, const float* s, float* What) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j) {
      float w = load_elem(W, dtype, n * ldw + j);
      What[n * K + j] = s ? w * s[j] : w;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 7: the integer GEMM                                                  */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "The problem SmoothQuant solves": both operands are 8-bit
 * integers and the products are accumulated exactly; [SQ-rec] "notes": int8
 * weights times int8 activations with int32 accumulate.
 * acc[m, n] = sum_k Xq[m, k] * Wq[n, k], in int64 (exact for any K).
 * Parity: pinned by a pure-Python triple loop on tiny shapes and by numpy's
 * int64 matmul.
 */
void oracle_gemm_i64(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N,
                     int64_t K, int64_t* acc) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t t = 0;
      for (int64_t k = 0; k < K; ++k)
        t += (int64_t)Xq[m * K + k] * (int64_t)Wq[n * K + k];
      acc[m * N + n] = t;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 8: dequantising epilogue                                             */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "Granularity": out = acc x scale_token[i] x scale_channel[j],
 * then converted to FP16/BF16.  Evaluation order and precision:
 *   o32 = fl32(fl32(fl32(acc) * xs[m]) * ws[n]); optional ReLU max(o32, 0);
 *   out = bf16_rne(o32).
 * The ReLU's max orders -0 below +0 (IEEE 754-2019 maximum): a negative
 * product that underflowed to -0 (a zero scale) becomes +0, like every other
 * non-positive value.
 * o32_out and out_bf16 are each nullable.
 * Parity: pinned against numpy float32 arithmetic and torch's bf16 cast.
 */
void oracle_epilogue(const int64_t* acc, const float* xs, const float* ws,
                     int64_t M, int64_t N, int relu, float* o32_out,
                     uint16_t* out_bf16) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      float a = (float)acc[m * N + n];
      float t = a * xs[m];
      float o = t * ws[n];
      if (relu && !(o > 0.0f)) o = 0.0f;
      if (o32_out) o32_out[m * N + n] = o;
      if (out_bf16) out_bf16[m * N + n] = oracle_f32_to_bf16_bits(o);
    }
}

/* ------------------------------------------------------------------------ */
/* The down projection's input: SiLU(gate) * up                              */
/* ------------------------------------------------------------------------ */
/*
 * [SQ-depth] "Where the scales go in a decoder block": the down_proj input is
 * SiLU(gate) times up; it has no norm in front, is not smoothed and is
 * quantised with per-token scales.  The pages give neither the SiLU formula's
 * precision nor the layout of the merged gate/up projection.  Readings:
 *   - gate_up's output row holds gate in columns [0, I) and up in [I, 2I);
 *   - silu(g) = g * sigma(g), sigma(g) = 1 / (1 + e^-g), in fp32;
 *   - h = fl32(fl32(g * fl32(1 / fl32(1 + e))) * u), e = exp_cw(-g) below,
 *     and h is stored in the model dtype (bf16, round to nearest even) before
 *     it is quantised, as an unfused model would write it.
 *
 * exp_cw: e^t in fp32 by Cody and Waite's argument reduction (W. J. Cody and
 * W. Waite, "Software Manual for the Elementary Functions", 1980) followed by
 * the degree-7 Taylor polynomial of e^r, so that the result is a fixed
 * sequence of IEEE operations that any implementation can repeat bit for bit:
 *   t is first clamped to [-87, 87] (beyond that sigma is 0 or 1 to far below
 *   an fp32 ulp of silu, and 2^n below stays a normal number);
 *   n = rint(fl32(t * L2E)), L2E = fl32(1 / ln 2);
 *   r = fma(-n, LN2_HI, t), then r = fma(-n, LN2_LO, r), where LN2_HI is ln 2
 *       cut to 16 significant bits (n * LN2_HI is exact for |n| < 2^8) and
 *       LN2_LO = fl32(ln 2 - LN2_HI);
 *   p = 1/7!, then p = fma(p, r, 1/k!) for k = 6 .. 0 (coefficients fl32);
 *   e^t = fl32(p * 2^n), 2^n exact.
 * |r| <= about ln2 / 2, so the truncation term is below 1e-8 relative; the
 * rounding of the Horner steps adds a few fp32 ulps.
 * Parity: pinned against float64 exp (relative error bound), and SiLU * up
 * against the float64 formula (within one bf16 ulp of the exact value).
 */
#define CW_L2E 1.44269504088896340736f
#define CW_LN2_HI 0.693145751953125f      /* 45426 / 65536 */
#define CW_LN2_LO 1.428606765330187e-06f  /* ln 2 - LN2_HI, rounded to fp32 */

static float exp_cw(float t) {
  if (t > 87.0f) t = 87.0f;
  if (t < -87.0f) t = -87.0f;
  const float n = rintf(t * CW_L2E);
  float r = fmaf(-n, CW_LN2_HI, t);
  r = fmaf(-n, CW_LN2_LO, r);
  float p = 1.0f / 5040.0f;
  p = fmaf(p, r, 1.0f / 720.0f);
  p = fmaf(p, r, 1.0f / 120.0f);
  p = fmaf(p, r, 1.0f / 24.0f);
  p = fmaf(p, r, 1.0f / 6.0f);
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  const uint32_t bits = (uint32_t)((int32_t)n + 127) << 23; /* 2^n, n in [-126, 126] */
  float two_n;
  memcpy(&two_n, &bits, sizeof two_n);
  return p * two_n;
}

void oracle_exp_cw(const float* t, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = exp_cw(t[i]);
}

/* One element of the down projection's input, before the bf16 store. */
static float silu_mul_one(float g, float u) {
  const float e = exp_cw(-g);
  const float sigma = 1.0f / (1.0f + e);
  const float silu = g * sigma;
  return silu * u;
}

/* gu: [M, 2I] (row stride ld) bf16 or fp32; h32 [M, I] fp32 and h_bf16
 * [M, I] bf16 bits, each nullable. */
void oracle_silu_mul(const void* gu, int dtype, int64_t M, int64_t I, int64_t ld, float* h32,
                     uint16_t* h_bf16) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < I; ++j) {
      const float g = load_elem(gu, dtype, m * ld + j);
      const float u = load_elem(gu, dtype, m * ld + I + j);
      const float h = silu_mul_one(g, u);
      if (h32) h32[m * I + j] = h;
      if (h_bf16) h_bf16[m * I + j] = oracle_f32_to_bf16_bits(h);
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 (e4m3) W8A8                                                           */
/* ------------------------------------------------------------------------ */
/*
 * [LLMint8] "example . what you get": on GPUs with FP8 support, FP8 W8A8 has
 * largely taken over INT8's role, with the same smoothing applied before the
 * activations are quantised; [SQ-map] "What it did NOT solve": FP8 hardware
 * later overtook INT8 serving.  The pages give no FP8 arithmetic.  Readings:
 *   - format: e4m3 without infinities (OCP FP8 E4M3, "fn"): sign, 4 exponent
 *     bits with bias 7, 3 mantissa bits; largest finite 448, smallest
 *     subnormal 2^-9; 0x7f / 0xff are NaN and never produced here;
 *   - encoding: round to nearest even; magnitudes beyond 448 saturate to 448;
 *   - per-token (and per-output-channel) scaling as for INT8 with the grid's
 *     largest value 448 in place of 127: step = fl32(absmax / 448);
 *   - the code multiplies by the correctly rounded reciprocal of the step,
 *     code = e4m3(fl32(y * fl32(1 / step))): the stored step is what the
 *     epilogue multiplies by; (the pages quantise by division for INT8 only);
 *   - a row whose step is zero or subnormal (absmax below 448 * 2^-126) is
 *     all zero codes with step 0;
 *   - the GEMM accumulates the products of the decoded codes; its exact value
 *     is computed here in fp64 (every product is a multiple of 2^-18 below
 *     2^18, so sums of up to 2^17 of them are exact);
 *   - epilogue as for INT8 from the fp32 accumulator:
 *     out = bf16(fl32(fl32(acc * xs[m]) * ws[n])).
 */
#define E4M3_MAX 448.0f

float oracle_e4m3_to_f32(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  float v;
  if (e == 0) v = ldexpf((float)m, -9);                /* subnormal: m * 2^-9 */
  else v = ldexpf((float)(8 + m), e - 10);             /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* Round |x| (finite) to the e4m3 grid, nearest, ties to even; saturate. */
uint8_t oracle_f32_to_e4m3(float x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 464.0) return sign | 0x7e;  /* at or past the midpoint above 448 */
  /* the grid spacing at a: 2^-9 below 2^-6, else 2^(floor(log2 a) - 3) */
  int e2 = -6;
  if (a >= ldexp(1.0, -6)) e2 = ilogb(a);
  const double q = ldexp(1.0, e2 - 3);
  double n = a / q;                       /* exact: a power-of-two scaling */
  double r = nearbyint(n);                /* current rounding mode: to nearest even */
  /* the integer multiple r of q: 8..16 in the normal binade, 0..8 below */
  double val = r * q;
  if (val >= 464.0) return sign | 0x7e;
  if (val == 0.0) return sign;
  int ev = ilogb(val);
  if (ev < -6) return sign | (uint8_t)(val / ldexp(1.0, -9)); /* subnormal code */
  const int m = (int)(val / ldexp(1.0, ev - 3)) - 8;
  return sign | (uint8_t)(((ev + 7) << 3) | m);
}

/* Per-row FP8 quantisation of y [M, K]: q [M, K] e4m3 codes, step [M]. */
void oracle_quantize_rows_fp8(const float* y, int64_t M, int64_t K, uint8_t* q, float* step) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    float am = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      const float a = fabsf(y[m * K + k]);
      if (a > am) am = a;
    }
    float st = am / E4M3_MAX;
    if (!(st >= 1.17549435e-38f)) st = 0.0f; /* zero or subnormal step: zero row */
    step[m] = st;
    const float inv = st > 0.0f ? 1.0f / st : 0.0f;
    for (int64_t k = 0; k < K; ++k)
      q[m * K + k] = st > 0.0f ? oracle_f32_to_e4m3(y[m * K + k] * inv) : 0;
  }
}

/* Exact acc[m, n] = sum_k dec(Xq[m, k]) * dec(Wq[n, k]) in fp64 (K <= 2^17). */
void oracle_gemm_fp8(const uint8_t* Xq, const uint8_t* Wq, int64_t M, int64_t N, int64_t K,
                     double* acc) {
  float lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = oracle_e4m3_to_f32((uint8_t)c);
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k)
        s += (double)lut[Xq[m * K + k]] * (double)lut[Wq[n * K + k]];
      acc[m * N + n] = s;
    }
}

/* Epilogue from an fp32 accumulator: o32 = fl32(fl32(acc * xs) * ws), ReLU
 * as in oracle_epilogue, out = bf16(o32). */
void oracle_epilogue_f32(const float* acc, const float* xs, const float* ws, int64_t M,
                         int64_t N, int relu, float* o32_out, uint16_t* out_bf16) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      float t = acc[m * N + n] * xs[m];
      float o = t * ws[n];
      if (relu && !(o > 0.0f)) o = 0.0f;
      if (o32_out) o32_out[m * N + n] = o;
      if (out_bf16) out_bf16[m * N + n] = oracle_f32_to_bf16_bits(o);
    }
}

/* Thread count the OpenMP loops will use (for the CPU-baseline report). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Comparator: LLM.int8()'s mixed-precision decomposition                    */
/* ------------------------------------------------------------------------ */
/*
 * [LLMint8] "Fix 1: give the outliers their own lane (LLM.int8())" and
 * "going deeper -- LLM.int8() decomposition": the outlier channels are
 * O = { j : max_t |X[t, j]| >= tau } (tau = 6 in the paper); the layer is
 * X[:, O] W[O, :] in 16-bit plus the vector-wise INT8 product of the other
 * channels (one absmax scale per token row of X, one per output channel of
 * W), and the two results are added.
 *
 * oracle_llmint8_outliers: from col_absmax[j] = max_t |X[t, j]| (the
 * calibration max with no norm), mask[j] = 0 for j in O and 1 otherwise (the
 * INT8 lane quantises x * mask: the channels of O give code 0 and do not
 * count towards a token's step), idx = the channels of O in ascending order.
 * Returns |O|.
 * Parity: pinned by the pages' one-token example (channels 1512 and 2817
 * taken out, the step of the rest 2/127), the tau boundary (>=) and an empty
 * set.
 */
int64_t oracle_llmint8_outliers(const float* col_absmax, int64_t K, float tau, float* mask,
                                int32_t* idx) {
  int64_t n = 0;
  for (int64_t j = 0; j < K; ++j) {
    const int out = col_absmax[j] >= tau;
    mask[j] = out ? 0.0f : 1.0f;
    if (out) idx[n++] = (int32_t)j;
  }
  return n;
}

/*
 * oracle_llmint8_combine: y[m, n] = fl32(o32[m, n] + y16[m, n]), ReLU when
 * asked (as in oracle_epilogue), out = bf16_rne(y), where o32 is the INT8
 * lane's dequantised value (oracle_epilogue's o32 without ReLU) and
 *   y16[m, n] = fl32(s),  s = sum over j in O, ascending, of x[m, j] * w[n, j]
 * accumulated in fp64 (s starts at +0; each step s = fl64(s + x w)).  The
 * product of two bf16 (or two fp32) values is exact in fp64, so s is a fixed
 * sequence of roundings.  Readings (the pages give no precision): the 16-bit
 * lane multiplies the unquantised inputs in their stored type with a wide
 * accumulator; W is quantised once per output channel over all its input
 * channels (the stored INT8 weights, whose outlier columns the INT8 lane
 * never meets because their activation codes are 0); "add the two results"
 * is one fp32 addition.
 * y_out and out_bf16 are each nullable.
 * Parity: pinned by exact integer dot products on small inputs, by the empty
 * outlier set (equal to the plain W8A8 layer) and by the all-outlier set
 * (equal to a sequential fp64 dot product).
 */
void oracle_llmint8_combine(const float* o32, int64_t M, int64_t N, const void* x, int xdtype,
                            int64_t ldx, const void* W, int wdtype, int64_t ldw,
                            const int32_t* idx, int64_t nout, int relu, float* y_out,
                            uint16_t* out_bf16) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t i = 0; i < nout; ++i) {
        const int64_t j = idx[i];
        const double xv = (double)load_elem(x, xdtype, m * ldx + j);
        const double wv = (double)load_elem(W, wdtype, n * ldw + j);
        s = s + xv * wv;
      }
      float y = o32[m * N + n] + (float)s;
      if (relu && !(y > 0.0f)) y = 0.0f;
      if (y_out) y_out[m * N + n] = y;
      if (out_bf16) out_bf16[m * N + n] = oracle_f32_to_bf16_bits(y);
    }
}
