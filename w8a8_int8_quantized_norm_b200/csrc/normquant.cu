// normquant.cu -- the fused norm + per-token INT8 quantisation on sm_100a,
// as a persistent, memory-pipelined kernel.
//
// Source pages (by title and section): "SmoothQuant, in depth" -- "Where the
// scales go in a decoder block" (the norm's gamma / beta carry 1/s, so the
// norm emits X/s), "Granularity" (per-token dynamic activation scales and
// per-output-channel weight scales); "LLM.int8() and SmoothQuant" -- "Try it"
// (INT8 step = max / 127).
//
// Design (HBM-bound: 2 bytes read + 1 byte written per bf16 element):
//   * persistent CTAs, several per SM; each owns rows first, first + G, ...;
//   * every row is fetched whole with one cp.async.bulk into a ring of NBUF
//     shared-memory row buffers, so NBUF - 1 rows per CTA are in flight while
//     the CTA computes on the current one;
//   * the norm kind is a template parameter (no per-element branches); row
//     sums are fp64 (x^2 of a bf16 / fp32 value is exact in fp64), reduced in
//     a fixed order so results repeat bit for bit;
//   * the quantiser avoids a division per element.  With a row's own step
//     (max / 127) the codes come from two fused multiply-adds that bracket
//     y / step (codes8_bracket); with a given step, from r = fl32(1/step),
//     whose product t = fl32(y r) is within 3 * 2^-24 relative of y/step, so
//     rne(fl32(y/step)) = rne(t) unless y/step lies within 1e-4 of a
//     half-integer (codes8).  Either way a chunk of 8 values that the fast
//     test cannot decide is redone with the exact division.  Rounding to the
//     nearest integer (ties to even) is the float add of 1.5 * 2^23, whose low
//     8 mantissa bits are then the two's-complement INT8 code.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_launch.h"

namespace sq {
namespace {

constexpr int kChunk = 8;       // elements per thread chunk
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr long long kWaitBudgetCycles = 4000000000LL;

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <bool kBF16>
__device__ __forceinline__ void smem_chunk(const uint8_t* row, int ch, float2 (&v)[4]) {
  if constexpr (kBF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + ch * 16);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  } else {
    const float4 a = *reinterpret_cast<const float4*>(row + ch * 32);
    const float4 b = *reinterpret_cast<const float4*>(row + ch * 32 + 16);
    v[0] = make_float2(a.x, a.y);
    v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y);
    v[3] = make_float2(b.z, b.w);
  }
}

// ---- SiLU(gate) * up ---------------------------------------------------
// e^t as a fixed sequence of IEEE fp32 operations: Cody and Waite's argument
// reduction (W. J. Cody, W. Waite, "Software Manual for the Elementary
// Functions", 1980) with ln 2 split into a 16-significant-bit head (n * head
// is exact for |n| < 256) and an fp32 tail, then the degree-7 Taylor
// polynomial of e^r by Horner's rule in fused multiply-adds, then the exact
// scaling by 2^n.  t is clamped to [-87, 87]: 2^n stays normal and sigma is
// already 0 or 1 to far below an ulp of the product beyond that.
// Max relative error against the exact exponential: under one fp32 ulp.
constexpr float kLog2e = 1.44269504088896340736f;       // fl32(1 / ln 2)
constexpr float kLn2Head = 0.693145751953125f;          // floor(ln 2 * 2^16) / 2^16
constexpr float kLn2Tail = 1.4286067653301870e-06f;     // fl32(ln 2 - head)

__device__ __forceinline__ float2 exp_cw2(float2 t) {
  t.x = fminf(fmaxf(t.x, -87.0f), 87.0f);
  t.y = fminf(fmaxf(t.y, -87.0f), 87.0f);
  // n = rint(fl32(t * log2 e)): adding 1.5 * 2^23 rounds |x| < 2^22 to an
  // integer (nearest, ties to even) and subtracting it back is exact; the
  // integer itself sits in the low bits of the sum
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float2 sum = __fadd2_rn(__fmul2_rn(t, make_float2(kLog2e, kLog2e)),
                                make_float2(kMagic, kMagic));
  const float2 nn = __fadd2_rn(make_float2(kMagic, kMagic), make_float2(-sum.x, -sum.y));  // -n
  float2 r = __ffma2_rn(nn, make_float2(kLn2Head, kLn2Head), t);
  r = __ffma2_rn(nn, make_float2(kLn2Tail, kLn2Tail), r);
  // Taylor coefficients 1/k!, each rounded to fp32
  constexpr float c7 = 1.0f / 5040.0f, c6 = 1.0f / 720.0f, c5 = 1.0f / 120.0f,
                  c4 = 1.0f / 24.0f, c3 = 1.0f / 6.0f;
  float2 p = make_float2(c7, c7);
  p = __ffma2_rn(p, r, make_float2(c6, c6));
  p = __ffma2_rn(p, r, make_float2(c5, c5));
  p = __ffma2_rn(p, r, make_float2(c4, c4));
  p = __ffma2_rn(p, r, make_float2(c3, c3));
  p = __ffma2_rn(p, r, make_float2(0.5f, 0.5f));
  p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
  p = __ffma2_rn(p, r, make_float2(1.0f, 1.0f));
  // 2^n from the integer in the sum's low bits: bits(sum) = 0x4b400000 + n
  const float2 two_n =
      make_float2(__int_as_float((__float_as_int(sum.x) - (0x4b400000 - 127)) << 23),
                  __int_as_float((__float_as_int(sum.y) - (0x4b400000 - 127)) << 23));
  return __fmul2_rn(p, two_n);
}

// Eight outputs h = bf16(fl32(fl32(g * fl32(1 / fl32(1 + e^-g))) * u)) of a
// chunk, as packed bf16 pairs.
__device__ __forceinline__ void silu_mul8(const float2 (&g)[4], const float2 (&u)[4],
                                          uint32_t (&hb)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 e = exp_cw2(make_float2(-g[i].x, -g[i].y));
    const float2 d = __fadd2_rn(make_float2(1.0f, 1.0f), e);
    const float2 sig = make_float2(__frcp_rn(d.x), __frcp_rn(d.y));
    const float2 h = __fmul2_rn(__fmul2_rn(g[i], sig), u[i]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(h.x, h.y);
    hb[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
}

// FP8 (e4m3) codes of 8 values, packed little-endian: e4m3(fl32(v * inv)),
// nearest even, saturating at +-448 (cvt.rn.satfinite), where inv is the
// correctly rounded reciprocal of the row's step.
__device__ __forceinline__ uint2 codes8_f8(const float2 (&v)[4], float inv) {
  const float2 inv2 = make_float2(inv, inv);
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(__fmul2_rn(v[2 * h], inv2), __NV_SATFINITE,
                                                 __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(__fmul2_rn(v[2 * h + 1], inv2), __NV_SATFINITE,
                                                 __NV_E4M3);
    w[h] = (lo & 0xffffu) | (hi << 16);
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void param8(const float* p, int ch, float2 (&v)[4]) {
  const float4* q = reinterpret_cast<const float4*>(p + ch * kChunk);
  const float4 a = __ldg(q), b = __ldg(q + 1);
  v[0] = make_float2(a.x, a.y);
  v[1] = make_float2(a.z, a.w);
  v[2] = make_float2(b.x, b.y);
  v[3] = make_float2(b.z, b.w);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// INT8 codes of 8 values, packed little-endian into two words:
// clamp(rne(fl32(v / step)), -127, 127).  Fast path: one fused multiply-add
// rounds the exact product P = v * rstep (rstep = fl32(1 / step)) to an
// integer, ties to even, as the low mantissa bits of P + 1.5 * 2^23; P is
// within 3 * 2^-24 relative of v / step and, when step is the row's own
// max / 127, |P| < 127.5, so the code equals the exact one -- no clamp
// needed -- unless v / step lies within 1e-4 of a half-integer.  The residual
// P - n (one more fused multiply-add) flags that case; a chunk holding such a
// value, or a step without a finite reciprocal, is recomputed from the exact
// quotient.  kClamp: the step may be smaller than max |v| / 127 (a fixed,
// per-tensor step), so the rounded integer is clamped to [-127, 127] in the
// magic domain (the only boundary, 127.5, is a half-integer: the residual
// test sends it to the exact path, which clamps too).
template <bool kClamp = false>
__device__ __forceinline__ uint2 codes8(const float2 (&v)[4], float rstep, float step,
                                        bool exact_only) {
  uint32_t m[8];
  float dmax = 0.0f;
  const float2 rs = make_float2(rstep, rstep);
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // paired fp32 instructions: each component rounds exactly like the scalar op
    float2 mf = __ffma2_rn(v[i], rs, mg);
    const float2 n = __fadd2_rn(mf, make_float2(-kMagic, -kMagic));
    const float2 d = __ffma2_rn(v[i], rs, make_float2(-n.x, -n.y));
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
    if constexpr (kClamp) {
      mf.x = fminf(fmaxf(mf.x, kMagic - 127.0f), kMagic + 127.0f);
      mf.y = fminf(fmaxf(mf.y, kMagic - 127.0f), kMagic + 127.0f);
    }
    m[2 * i] = __float_as_uint(mf.x);
    m[2 * i + 1] = __float_as_uint(mf.y);
  }
  if (exact_only || dmax > 0.4999f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float vv[2] = {v[i].x, v[i].y};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float e = (step == 0.0f) ? 0.0f : __fdiv_rn(vv[j], step);
        e = fminf(fmaxf(e, -127.0f), 127.0f);
        m[2 * i + j] = __float_as_uint(__fadd_rn(e, kMagic));
      }
    }
  }
  // the low byte of each magic sum is the two's-complement code
  const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

// INT8 codes of 8 values, packed little-endian, by bracketing: with
// rhi >= (1 + 2^-24) / step and rlo <= (1 - 2^-24) / step (both finite,
// step normal), the exact quotient q = v / step and its fp32 rounding lie
// between v rlo and v rhi; round-half-even to an integer is monotone, so
// when the two fused multiply-adds rne(v rhi) and rne(v rlo) (as the low
// bits of the product + 1.5 * 2^23, one rounding each) agree, that integer
// is rne(fl32(q)) -- no clamp needed when |v| <= 127 step.  They disagree
// only when an integer + 1/2 lies within about 2^-21 |q| of q (at most
// 2^-13 of the values); a chunk holding one, or a step without a finite
// reciprocal, is recomputed from the exact quotient.
__device__ __forceinline__ uint2 codes8_bracket(const float2 (&v)[4], float rhi, float rlo,
                                                float step, bool exact_only) {
  uint32_t m[8];
  uint32_t diff = 0u;
  const float2 rh = make_float2(rhi, rhi), rl = make_float2(rlo, rlo);
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = __ffma2_rn(v[i], rh, mg);
    const float2 b = __ffma2_rn(v[i], rl, mg);
    diff |= __float_as_uint(a.x) ^ __float_as_uint(b.x);
    diff |= __float_as_uint(a.y) ^ __float_as_uint(b.y);
    m[2 * i] = __float_as_uint(a.x);
    m[2 * i + 1] = __float_as_uint(a.y);
  }
  if (exact_only || diff != 0u) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float vv[2] = {v[i].x, v[i].y};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float e = (step == 0.0f) ? 0.0f : __fdiv_rn(vv[j], step);
        e = fminf(fmaxf(e, -127.0f), 127.0f);
        m[2 * i + j] = __float_as_uint(__fadd_rn(e, kMagic));
      }
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

// The bracketing codes of 8 values without the fallback: returns the packed
// codes of v rhi and ORs into `diff` a non-zero word when some value's two
// roundings disagree (the caller then recomputes with exact8).
__device__ __forceinline__ uint2 bracket8(const float2 (&v)[4], float2 rh, float2 rl,
                                          uint32_t& diff) {
  uint32_t m[8];
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = __ffma2_rn(v[i], rh, mg);
    const float2 b = __ffma2_rn(v[i], rl, mg);
    diff |= __float_as_uint(a.x) ^ __float_as_uint(b.x);
    diff |= __float_as_uint(a.y) ^ __float_as_uint(b.y);
    m[2 * i] = __float_as_uint(a.x);
    m[2 * i + 1] = __float_as_uint(a.y);
  }
  const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

// clamp(rne(fl32(v / step)), -127, 127) of 8 values by the exact division
// (step 0: zero codes).
__device__ __forceinline__ uint2 exact8(const float2 (&v)[4], float step) {
  uint32_t m[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float vv[2] = {v[i].x, v[i].y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float e = (step == 0.0f) ? 0.0f : __fdiv_rn(vv[j], step);
      e = fminf(fmaxf(e, -127.0f), 127.0f);
      m[2 * i + j] = __float_as_uint(__fadd_rn(e, kMagic));
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

// The bracketing multipliers of a row's step (normal): rs = fl32(1 / step)
// is within 2^-24 of 1 / step, and fl32(rs (1 +- 2^-21)) stay more than
// 2^-22 away from rs on their side, so rhi >= (1 + 2^-24) / step and
// rlo <= (1 - 2^-24) / step.
__device__ __forceinline__ void bracket_of(float step, float& rhi, float& rlo) {
  const float rs = __frcp_rn(step);
  rhi = __fmul_rn(rs, 1.0f + 0x1p-21f);
  rlo = __fmul_rn(rs, 1.0f - 0x1p-21f);
}

// fl32(a / 127) for every non-negative finite binary32 a, in three
// instructions: q0 = fl32(a c) with c = fl32(1/127) is within an ulp of the
// quotient, the remainder a - 127 q0 is exact in one fused multiply-add, and a
// second one corrects q0.  The sequence was compared with the IEEE quotient
// for all 2^31 - 2^23 such inputs (subnormals included) and agrees on every
// one; infinities take the division.
__device__ __forceinline__ float div127(float a) {
  constexpr float c = 1.0f / 127.0f;
  if (!(a <= FLT_MAX)) return __fdiv_rn(a, 127.0f);
  const float q0 = __fmul_rn(a, c);
  const float r = __fmaf_rn(-q0, 127.0f, a);
  return __fmaf_rn(r, c, q0);
}

// Bounded wait for a row copy: buffer `b`, phase parity `parity`.
__device__ __forceinline__ bool row_landed(uint32_t bar_base, int b, uint32_t parity) {
  const uint32_t bar = bar_base + 8u * static_cast<uint32_t>(b);
  if (mbar_try_wait(bar, parity)) return true;
  const long long c0 = clock64();
  for (uint32_t k = 0;; ++k) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((k & 63u) == 63u && clock64() - c0 > kWaitBudgetCycles) return false;
  }
}

// The buffer `pb` of row number `i` has been read: load the row nbuf further
// on into it (if there is one).  Returns the new count of issued copies.
__device__ __forceinline__ int refill_row(uint32_t smem_base, uint32_t bar_base,
                                          uint32_t buf_stride, uint32_t row_bytes, int nbuf, int i,
                                          int pb, int64_t row, int64_t G, int64_t M,
                                          const uint8_t* xb, int64_t row_pitch, int issued) {
  const int64_t nrow = row + static_cast<int64_t>(nbuf) * G;
  if (nrow >= M) return issued;
  mbar_arrive_expect_tx(bar_base + 8u * pb, row_bytes);
  bulk_load(smem_base + pb * buf_stride, xb + nrow * row_pitch, row_bytes, bar_base + 8u * pb);
  return i + nbuf + 1;
}

// NORMK: 0 = no norm (optional per-channel multiplier), 1 = RMSNorm, 2 = LayerNorm.
// What a launch of the row pipeline produces.
enum RowMode : int {
  kModeRowQuant = 0,    // per-row (per-token) step and codes
  kModeColMax = 1,      // calibration: running per-column max of |y|
  kModeTensorMax = 2,   // one running max of |y| over the whole tensor
  kModeFixedQuant = 3,  // codes with one given step (per-tensor: O2 / O3)
  kModeGivenQuant = 4,  // per-row codes, each row's max |y| given in act_max[row]
  kModeSiluMul = 5,     // per-row codes of h = SiLU(gate) * up (rows hold [gate | up])
  kModeRowQuantF8 = 6,  // per-row step and FP8 (e4m3) codes
  kModeSiluMulF8 = 7,   // SiLU * up rows with FP8 codes
  kModeRowAbsmax = 8,   // each row's max |y| into act_max[row], no codes
};

// Bytes of one input row: SiLU * up rows hold both halves.
template <int kMode>
constexpr int kInRowFactor = (kMode == kModeSiluMul || kMode == kModeSiluMulF8) ? 2 : 1;

template <int CH, int kMode>
struct PipeBounds {
  // SiLU * up rows (at most 28928 outputs: 3616 chunks) run 4 chunks a thread
  // on up to 1024 threads: the row holds one CTA per SM (two 113 KB input
  // buffers), so its warps are the only latency hiding there is
  static constexpr bool kGLU = kMode == kModeSiluMul || kMode == kModeSiluMulF8;
  static constexpr int kMaxThreads = kGLU ? 1024 : (CH <= 4 ? 512 : 640);
  // 4-chunk CTAs keep to 64 registers a thread so four 256-thread CTAs fit
  // an SM; calibration also keeps a running column max per element
  static constexpr int kMinBlocks =
      (CH <= 4 && kMode != kModeColMax && !kGLU) ? 2 : 1;
};

// One row per iteration, three CTA barriers per row (two when calibrating):
//   A  the warps' partial sums are in shared memory (norm kinds only); the
//      row buffer has been read into registers, so it is refilled here;
//   B  warp 0 has turned the sums into r (and mu);
//   C  the warps' partial absmax is merged, and thread 0 has seen the next
//      row land (a bounded wait; a timeout aborts the CTA).
// Modes without a per-row absmax (calibration column max, fixed-step codes)
// fold C into B.  Calibration keeps a per-thread running max of |y| over the
// rows it sees, merged into act_max[K] at the end; the tensor-max mode keeps
// the CTA's running max of the row maxima and merges it into act_max[0]; the
// fixed-step mode reads its step's max |y| from act_max[0] once; the given-max
// mode reads row i's from act_max[i] (a producer already reduced it).
//
// kFull: every thread owns all CH of its chunks (T * CH == K / 8): no bounds checks.
template <bool kBF16, int NORMK, int CH, bool kGamma, bool kBeta, bool kFull, int kMode>
__global__ void __launch_bounds__(PipeBounds<CH, kMode>::kMaxThreads,
                                  PipeBounds<CH, kMode>::kMinBlocks)
    norm_rows_pipe_kernel(const void* __restrict__ x, int64_t ldx, int64_t M, int K,
                          const float* __restrict__ gamma, const float* __restrict__ beta,
                          float eps, int8_t* __restrict__ q, float* __restrict__ scale,
                          float* __restrict__ act_max, int nbuf, int* error_word,
                          __nv_bfloat16* __restrict__ h_out, int64_t ldh) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kEsz = kBF16 ? 2 : 4;
  constexpr bool kGLU = kMode == kModeSiluMul || kMode == kModeSiluMulF8;
  static_assert(!kGLU || (kBF16 && NORMK == 0 && !kGamma && !kBeta), "SiLU * up: bf16, no norm");
  const uint32_t row_bytes = static_cast<uint32_t>(K) * kEsz * kInRowFactor<kMode>;
  const uint32_t buf_stride = (row_bytes + 127u) & ~127u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + nbuf * buf_stride);
  double* dscr = reinterpret_cast<double*>(bars + nbuf);      // [64]: sum x^2, sum x per warp
  float* fscr = reinterpret_cast<float*>(dscr + 64);           // [2]: r, mu of the row
  // [3]: row absmax bits, rotating: row i merges into slot i mod 3 before
  // barrier C and reads it after; thread 0 clears the slot of row i + 2 after
  // C, which every thread passes again (C of row i + 1) before touching it
  unsigned int* smax = reinterpret_cast<unsigned int*>(fscr + 2);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);

  const int t = threadIdx.x, T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nchunks = K / kChunk;
  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;
  const uint8_t* xb = static_cast<const uint8_t*>(x);
  const int64_t row_pitch = ldx * kEsz;
  // launched as a programmatic dependent: let the next kernel be scheduled,
  // and touch no global memory before the previous grid has completed
  if (t == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (t == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(bar_base + 8u * b, 1);
    smax[0] = 0u;
    smax[1] = 0u;
    smax[2] = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  // thread 0: row copies issued so far, in the CTA's row order (the first
  // nbuf at once, then one refill per iteration, each into the buffer of the
  // row it replaces)
  int issued = 0;
  if (t == 0) {
    for (int b = 0; b < nbuf; ++b) {
      const int64_t row = first + b * G;
      if (row < M) {
        mbar_arrive_expect_tx(bar_base + 8u * b, row_bytes);
        bulk_load(smem_base + b * buf_stride, xb + row * row_pitch, row_bytes, bar_base + 8u * b);
        issued = b + 1;
      }
    }
  }
  bool aborted = false;
  {
    const bool ok = (t != 0 || first >= M) ? true : row_landed(bar_base, 0, 0u);
    if (__syncthreads_or(!ok)) aborted = true;
  }
  constexpr bool kCalib = kMode == kModeColMax;
  constexpr bool kF8 = kMode == kModeRowQuantF8 || kMode == kModeSiluMulF8;
  constexpr bool kRowMax = kMode == kModeRowQuant || kMode == kModeTensorMax || kGLU || kF8 ||
                           kMode == kModeRowAbsmax;
  float cta_max = 0.0f;  // tensor-max mode, thread 0
  // fixed-step mode: the one step, from the given max |y|
  float fstep = 0.0f, frstep = 0.0f;
  bool fexact = false;
  if constexpr (kMode == kModeFixedQuant) {
    fstep = div127(__ldg(act_max));
    fexact = fstep < FLT_MIN;
    frstep = fexact ? 0.0f : __frcp_rn(fstep);
  }
  // given-max mode: row i's max is loaded one row ahead (its global-load
  // latency hides behind the previous row's work)
  float gmax_next = 0.0f;
  if constexpr (kMode == kModeGivenQuant) {
    if (first < M) gmax_next = __ldg(act_max + first);
  }
  float2 cm[kCalib ? CH : 1][4];  // calibration: running max of |y| per owned element
  if constexpr (kCalib) {
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) cm[c][i] = make_float2(0.0f, 0.0f);
  }

  int it = 0;
  int buf = 0;            // it mod nbuf
  int slot = 0;           // it mod 3
  int nbuf_next = nbuf > 1 ? 1 : 0;  // (it + 1) mod nbuf
  uint32_t par_next = nbuf > 1 ? 0u : 1u;  // phase parity of row it + 1's copy
  for (int64_t row = first; row < M && !aborted;
       row += G, ++it, buf = nbuf_next, slot = (slot == 2 ? 0 : slot + 1),
               par_next ^= (nbuf_next + 1 == nbuf) ? 1u : 0u,
               nbuf_next = (nbuf_next + 1 == nbuf) ? 0 : nbuf_next + 1) {
    const uint8_t* rowp = smem + buf * buf_stride;
    float gmax = 0.0f;
    if constexpr (kMode == kModeGivenQuant) {
      gmax = gmax_next;
      if (row + G < M) gmax_next = __ldg(act_max + row + G);
    }

    // ---- this thread's chunks of the row, from shared memory
    // (SiLU * up keeps h as packed bf16 pairs instead: half the registers)
    float2 v[kGLU ? 1 : CH][4];
    uint32_t hbv[kGLU ? CH : 1][4];
    uint32_t amb = 0;  // SiLU * up: max |h| as bf16 bits (magnitudes order like ints)
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (kFull || ch < nchunks) {
        if constexpr (kGLU) {
          float2 g[4], u[4];
          smem_chunk<true>(rowp, ch, g);
          smem_chunk<true>(rowp + static_cast<uint32_t>(K) * 2u, ch, u);
          silu_mul8(g, u, hbv[c]);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            amb = max(amb, max(hbv[c][i] & 0x7fffu, (hbv[c][i] >> 16) & 0x7fffu));
          if (h_out)
            *reinterpret_cast<uint4*>(h_out + row * ldh + ch * kChunk) =
                make_uint4(hbv[c][0], hbv[c][1], hbv[c][2], hbv[c][3]);
        } else {
          smem_chunk<kBF16>(rowp, ch, v[c]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if constexpr (kGLU) hbv[c][i] = 0u;
          else v[c][i] = make_float2(0.0f, 0.0f);
        }
      }
    }
    // ---- row statistics in fp64 (two accumulators per sum for ILP)
    if constexpr (NORMK != 0) {
      double s1a = 0.0, s1b = 0.0, s2a = 0.0, s2b = 0.0;
#pragma unroll
      for (int c = 0; c < CH; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double d0 = static_cast<double>(v[c][i].x);
          const double d1 = static_cast<double>(v[c][i].y);
          if constexpr (NORMK == 2) {
            s1a = __dadd_rn(s1a, d0);
            s1b = __dadd_rn(s1b, d1);
          }
          s2a = __fma_rn(d0, d0, s2a);
          s2b = __fma_rn(d1, d1, s2b);
        }
      double s2 = warp_sum(__dadd_rn(s2a, s2b));
      double s1 = 0.0;
      if constexpr (NORMK == 2) s1 = warp_sum(__dadd_rn(s1a, s1b));
      if (lane == 0) {
        dscr[warp] = s2;
        if constexpr (NORMK == 2) dscr[32 + warp] = s1;
      }
      __syncthreads();  // A
      if (t == 0)
        issued = refill_row(smem_base, bar_base, buf_stride, row_bytes, nbuf, it, buf, row, G, M,
                            xb, row_pitch, issued);
      // one warp turns the sums into the row's scalars (the fp64 divide and
      // square root are long instruction sequences: not worth repeating in
      // every warp)
      if (warp == 0) {
        double S2 = dscr[0], S1 = 0.0;
        if constexpr (NORMK == 2) S1 = dscr[32];
        for (int w = 1; w < nwarps; ++w) {
          S2 = __dadd_rn(S2, dscr[w]);
          if constexpr (NORMK == 2) S1 = __dadd_rn(S1, dscr[32 + w]);
        }
        const double ms = __ddiv_rn(S2, static_cast<double>(K));
        double var = ms;
        float mu32 = 0.0f;
        if constexpr (NORMK == 2) {
          const double mu64 = __ddiv_rn(S1, static_cast<double>(K));
          var = __dsub_rn(ms, __dmul_rn(mu64, mu64));
          if (var < 0.0) var = 0.0;
          mu32 = __double2float_rn(mu64);
        }
        const float r32 = __double2float_rn(
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps)))));
        if (lane == 0) {
          fscr[0] = r32;
          fscr[1] = mu32;
        }
      }
    }
    if constexpr (!kRowMax) {
      // B (with C folded in): the row scalars are published and the next row is in
      const bool ok = (t != 0 || row + G >= M) ? true : row_landed(bar_base, nbuf_next, par_next);
      if (__syncthreads_or(!ok)) {
        aborted = true;
        break;
      }
      if (NORMK == 0 && t == 0)
        issued = refill_row(smem_base, bar_base, buf_stride, row_bytes, nbuf, it, buf, row, G, M,
                            xb, row_pitch, issued);
    } else if constexpr (NORMK != 0) {
      __syncthreads();  // B
    }
    float mu = 0.0f, r = 1.0f;
    if constexpr (NORMK != 0) {
      r = fscr[0];
      mu = fscr[1];
    }
    // ---- the norm output (paired fp32 ops, same roundings; a multiply
    // followed by an add uses the scalar intrinsics, which are never
    // contracted into a fused multiply-add)
    float am = kGLU ? __uint_as_float(amb << 16) : 0.0f;
    const float2 r2 = make_float2(r, r), nmu2 = make_float2(-mu, -mu);
#pragma unroll
    for (int c = 0; c < (kGLU ? 0 : CH); ++c) {
      const int ch = t + c * T;
      if (!kFull && ch >= nchunks) continue;
      float2 g[4], bt[4];
      if constexpr (kGamma) param8(gamma, ch, g);
      if constexpr (kBeta) param8(beta, ch, bt);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 y = v[c][i];
        if constexpr (NORMK == 1) y = __fmul2_rn(y, r2);
        if constexpr (NORMK == 2) y = __fmul2_rn(__fadd2_rn(y, nmu2), r2);
        if constexpr (kBeta) {
          if constexpr (kGamma) {
            y.x = __fmul_rn(y.x, g[i].x);
            y.y = __fmul_rn(y.y, g[i].y);
          }
          y.x = __fadd_rn(y.x, bt[i].x);
          y.y = __fadd_rn(y.y, bt[i].y);
        } else if constexpr (kGamma) {
          y = __fmul2_rn(y, g[i]);
        }
        if constexpr (kCalib) {
          cm[c][i].x = fmaxf(cm[c][i].x, fabsf(y.x));
          cm[c][i].y = fmaxf(cm[c][i].y, fabsf(y.y));
        } else {
          v[c][i] = y;
          if constexpr (kRowMax) am = fmaxf(am, fmaxf(fabsf(y.x), fabsf(y.y)));
        }
      }
    }
    if constexpr (kMode == kModeFixedQuant || kMode == kModeGivenQuant) {
      float step = fstep, rstep = frstep;
      bool exact_only = fexact;
      if constexpr (kMode == kModeGivenQuant) {
        step = div127(gmax);
        exact_only = step < FLT_MIN;
        rstep = exact_only ? 0.0f : __frcp_rn(step);
      }
      if (t == 0) scale[row] = step;
      int8_t* qrow = q + row * static_cast<int64_t>(K);
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int ch = t + c * T;
        if (!kFull && ch >= nchunks) continue;
        // clamped: a given max below the row's true max saturates at +-127
        *reinterpret_cast<uint2*>(qrow + ch * kChunk) =
            codes8<true>(v[c], rstep, step, exact_only);
      }
    }
    if constexpr (kRowMax) {
      // non-negative floats order like their bit patterns: integer max reduce
      const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(am));
      if (lane == 0) atomicMax(&smax[slot], wmax);
      const bool ok = (t != 0 || row + G >= M) ? true : row_landed(bar_base, nbuf_next, par_next);
      if (__syncthreads_or(!ok)) {  // C
        aborted = true;
        break;
      }
      if (NORMK == 0 && t == 0)
        issued = refill_row(smem_base, bar_base, buf_stride, row_bytes, nbuf, it, buf, row, G, M,
                            xb, row_pitch, issued);
      am = __uint_as_float(smax[slot]);
      if (t == 0) smax[slot == 0 ? 2 : slot - 1] = 0u;  // the slot of row it + 2

      if constexpr (kMode == kModeTensorMax) {
        if (t == 0) cta_max = fmaxf(cta_max, am);
      } else if constexpr (kMode == kModeRowAbsmax) {
        if (t == 0) act_max[row] = am;
      } else if constexpr (kF8) {
        // ---- per-token FP8 quantisation: step = fl32(max / 448); a zero or
        // subnormal step makes the row all zero codes with step 0
        float step = __fdiv_rn(am, 448.0f);
        if (!(step >= FLT_MIN)) step = 0.0f;
        const float inv = step > 0.0f ? __frcp_rn(step) : 0.0f;
        if (t == 0) scale[row] = step;
        int8_t* qrow = q + row * static_cast<int64_t>(K);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int ch = t + c * T;
          if (!kFull && ch >= nchunks) continue;
          uint2 code = make_uint2(0u, 0u);
          if (step > 0.0f) {
            if constexpr (kGLU) {
              float2 hv[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                hv[i] = make_float2(__uint_as_float(hbv[c][i] << 16),
                                    __uint_as_float(hbv[c][i] & 0xffff0000u));
              code = codes8_f8(hv, inv);
            } else {
              code = codes8_f8(v[c], inv);
            }
          }
          *reinterpret_cast<uint2*>(qrow + ch * kChunk) = code;
        }
      } else {
        // ---- per-token INT8 quantisation (the row's own step: no clamp)
        const float step = div127(am);
        const bool exact_only = step < FLT_MIN;  // zero or subnormal step: no reciprocal
        float rhi = 0.0f, rlo = 0.0f;
        if (!exact_only) bracket_of(step, rhi, rlo);
        if (t == 0) scale[row] = step;
        int8_t* qrow = q + row * static_cast<int64_t>(K);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int ch = t + c * T;
          if (!kFull && ch >= nchunks) continue;
          if constexpr (kGLU) {
            float2 hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              hv[i] = make_float2(__uint_as_float(hbv[c][i] << 16),
                                  __uint_as_float(hbv[c][i] & 0xffff0000u));
            *reinterpret_cast<uint2*>(qrow + ch * kChunk) =
                codes8_bracket(hv, rhi, rlo, step, exact_only);
          } else {
            *reinterpret_cast<uint2*>(qrow + ch * kChunk) =
                codes8_bracket(v[c], rhi, rlo, step, exact_only);
          }
        }
      }
    }
  }
  if (aborted) {
    if (t == 0) {
      record_device_error(error_word, SQ_ERR_PIPELINE_TIMEOUT);
      // let every bulk copy still in flight land before the CTA exits: the
      // latest copy into buffer b is the one of row number s (s = b mod nbuf,
      // s < issued), which completes phase s / nbuf of the buffer's barrier
      for (int b = 0; b < nbuf && b < issued; ++b) {
        const int s_last = b + (issued - 1 - b) / nbuf * nbuf;
        const uint32_t par = static_cast<uint32_t>((s_last / nbuf) & 1);
        const long long c0 = clock64();
        while (!mbar_try_wait(bar_base + 8u * b, par) && clock64() - c0 < kWaitBudgetCycles) {
        }
      }
    }
    return;
  }
  if constexpr (kMode == kModeTensorMax) {
    if (t == 0) {
      unsigned int* dst = reinterpret_cast<unsigned int*>(act_max);
      const unsigned int bits = __float_as_uint(cta_max);
      if (bits > __ldcg(dst)) atomicMax(dst, bits);
    }
  }
  if constexpr (kCalib) {
    // merge into the running maximum.  The CTA's column maxima go to shared
    // memory first (the row ring is idle now: it holds K floats) and are
    // merged in an order rotated by CTA, so concurrent CTAs hit different L2
    // lines instead of queueing on the same ones.  The atomics return nothing
    // (reductions the L2 performs): no thread waits on a global round trip.
    unsigned int* colmax = reinterpret_cast<unsigned int*>(smem);
    __syncthreads();  // every thread is done with the row buffers
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (!kFull && ch >= nchunks) continue;
      uint4* dst = reinterpret_cast<uint4*>(colmax + ch * kChunk);
      dst[0] = make_uint4(__float_as_uint(cm[c][0].x), __float_as_uint(cm[c][0].y),
                          __float_as_uint(cm[c][1].x), __float_as_uint(cm[c][1].y));
      dst[1] = make_uint4(__float_as_uint(cm[c][2].x), __float_as_uint(cm[c][2].y),
                          __float_as_uint(cm[c][3].x), __float_as_uint(cm[c][3].y));
    }
    __syncthreads();
    unsigned int* am_bits = reinterpret_cast<unsigned int*>(act_max);
    const int rot = static_cast<int>((blockIdx.x * 613u) % static_cast<unsigned>(K));
#pragma unroll 4
    for (int i = t; i < K; i += T) {
      int j = i + rot;
      if (j >= K) j -= K;
      const unsigned int a = colmax[j];
      if (a != 0u) atomicMax(am_bits + j, a);
    }
  }
}

// Launch configuration of a row kernel: a programmatic dependent of the
// previous kernel in the stream (the kernel waits for that grid at its top,
// so it may start while that grid finishes).
cudaLaunchConfig_t pdl_config(unsigned grid, int threads, size_t smem, cudaStream_t st) {
  // initialised once (thread-safe), read-only afterwards
  static const cudaLaunchAttribute attr = [] {
    cudaLaunchAttribute a{};
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
  }();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = const_cast<cudaLaunchAttribute*>(&attr);
  cfg.numAttrs = 1;
  return cfg;
}

struct PipeShape {
  int ch, threads, nbuf;
  size_t smem;
};

// row buffers, their barriers, 64 doubles of partial sums, r and mu, 3 absmax slots
size_t pipe_smem(size_t stride, int nbuf) { return nbuf * stride + 8 * nbuf + 64 * 8 + 4 * 8; }

bool pipe_shape(int K, bool bf16, bool calib, PipeShape* ps, int in_factor = 1) {
  const int nchunks = K / kChunk;
  // chunks per thread and threads per CTA within the variant's register budget
  int ch = nchunks <= 4 * PipeBounds<4, kModeRowQuant>::kMaxThreads ? 4
           : (nchunks <= 8 * PipeBounds<8, kModeRowQuant>::kMaxThreads ? 8 : 0);
  (void)calib;  // the calibration variant uses the same shape (4-chunk rows only)
  if (in_factor > 1) ch = 4;  // SiLU * up: four chunks a thread, up to 1024 threads
  if (!ch) return false;
  int threads = (nchunks + ch - 1) / ch;
  threads = (threads + 31) / 32 * 32;
  if (threads < 32) threads = 32;
  if (threads > 1024) return false;
  const size_t row_bytes = static_cast<size_t>(K) * (bf16 ? 2 : 4) * in_factor;
  const size_t stride = (row_bytes + 127) / 128 * 128;
  // about 24 KB of row buffers per CTA: with small rows that leaves room for
  // eight CTAs per SM (more rows in flight, shorter per-CTA row chains)
  int nbuf = static_cast<int>((24u << 10) / stride);
  if (nbuf < 3) nbuf = 3;
  if (nbuf > 8) nbuf = 8;
  while (nbuf > 2 && nbuf * stride > (150u << 10)) --nbuf;
  // two-half rows (SiLU * up) may take two buffers up to the 227 KB a CTA can have
  if (nbuf * stride > (in_factor > 1 ? (226u << 10) : (200u << 10))) return false;
  ps->ch = ch;
  ps->threads = threads;
  ps->nbuf = nbuf;
  ps->smem = pipe_smem(stride, nbuf);
  return true;
}

struct RowArgs {
  const void* x;
  int64_t M;
  int K;
  int64_t ldx;
  const float* gamma;
  const float* beta;
  float eps;
  int8_t* q;
  float* scale;
  float* act_max;
  int* err;
  __nv_bfloat16* h_out = nullptr;
  int64_t ldh = 0;
};

template <bool kBF16, int NORMK, int CH, bool kG, bool kB, bool kF, int kMode>
cudaError_t launch_pipe_k(const RowArgs& a, PipeShape ps, cudaStream_t st) {
  constexpr bool kC = kMode == kModeColMax;
  auto kern = norm_rows_pipe_kernel<kBF16, NORMK, CH, kG, kB, kF, kMode>;
  const void* key = reinterpret_cast<const void*>(kern);
  LaunchCache& lc = launch_cache();
  int per_sm = 0;
  // fewer row buffers when each CTA sees only a few rows: more CTAs fit an SM
  const size_t stride =
      (static_cast<size_t>(a.K) * (kBF16 ? 2 : 4) * kInRowFactor<kMode> + 127) / 128 * 128;
  for (;;) {
    cudaError_t e = lc.ensure_smem(key, ps.smem);
    if (e != cudaSuccess) return e;
    per_sm = lc.blocks_per_sm(key, ps.threads, ps.smem);
    int64_t ctas = static_cast<int64_t>(per_sm) * lc.sms();
    if (kC && ctas > (a.M + 3) / 4) ctas = (a.M + 3) / 4;
    const int64_t rows_per_cta = (a.M + ctas - 1) / ctas;
    if (ps.nbuf <= 2 || rows_per_cta >= ps.nbuf) break;
    ps.nbuf = rows_per_cta < 2 ? 2 : static_cast<int>(rows_per_cta);
    ps.smem = pipe_smem(stride, ps.nbuf);
  }
  int64_t grid = static_cast<int64_t>(per_sm) * lc.sms();
  // calibration merges every CTA's column maxima with atomics: at least four
  // rows per CTA keeps their number (CTAs x K) down
  const int64_t max_grid = kC ? (a.M + 3) / 4 : a.M;
  if (grid > max_grid) grid = max_grid;
  cudaLaunchConfig_t cfg = pdl_config(static_cast<unsigned>(grid), ps.threads, ps.smem, st);
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, a.x, a.ldx, a.M, a.K, a.gamma, a.beta,
                                            a.eps, a.q, a.scale, a.act_max, ps.nbuf, a.err,
                                            a.h_out, a.ldh);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

template <bool kBF16, int NORMK, int CH, bool kG, bool kB, int kMode>
cudaError_t launch_pipe_t(const RowArgs& a, const PipeShape& ps, cudaStream_t st) {
  // bf16 rows whose chunks split evenly over the threads skip the bounds checks
  if constexpr (kBF16) {
    if (ps.threads * ps.ch == a.K / kChunk)
      return launch_pipe_k<kBF16, NORMK, CH, kG, kB, true, kMode>(a, ps, st);
  }
  return launch_pipe_k<kBF16, NORMK, CH, kG, kB, false, kMode>(a, ps, st);
}

template <bool kBF16, int NORMK, int CH, int kMode>
cudaError_t launch_pipe_c(const RowArgs& a, const PipeShape& ps, cudaStream_t st) {
  // beta only matters for LayerNorm
  const bool hb = NORMK == 2 && a.beta != nullptr;
  if (a.gamma) {
    if (hb) return launch_pipe_t<kBF16, NORMK, CH, true, NORMK == 2, kMode>(a, ps, st);
    return launch_pipe_t<kBF16, NORMK, CH, true, false, kMode>(a, ps, st);
  }
  if (hb) return launch_pipe_t<kBF16, NORMK, CH, false, NORMK == 2, kMode>(a, ps, st);
  return launch_pipe_t<kBF16, NORMK, CH, false, false, kMode>(a, ps, st);
}

template <bool kBF16, int NORMK, int kMode>
cudaError_t launch_pipe_n(const RowArgs& a, const PipeShape& ps, cudaStream_t st) {
  if (ps.ch == 4) return launch_pipe_c<kBF16, NORMK, 4, kMode>(a, ps, st);
  if constexpr (kMode == kModeColMax) return cudaErrorInvalidValue;  // 4-chunk shapes only
  else return launch_pipe_c<kBF16, NORMK, 8, kMode>(a, ps, st);
}

template <int kMode>
cudaError_t launch_rows(const RowArgs& a, bool bf16, int norm, cudaStream_t st) {
  PipeShape ps;
  if (!pipe_shape(a.K, bf16, kMode == kModeColMax, &ps)) return cudaErrorInvalidValue;
  if (bf16) {
    if (norm == SQ_NORM_RMS) return launch_pipe_n<true, 1, kMode>(a, ps, st);
    if (norm == SQ_NORM_LAYER) return launch_pipe_n<true, 2, kMode>(a, ps, st);
    return launch_pipe_n<true, 0, kMode>(a, ps, st);
  }
  if (norm == SQ_NORM_RMS) return launch_pipe_n<false, 1, kMode>(a, ps, st);
  if (norm == SQ_NORM_LAYER) return launch_pipe_n<false, 2, kMode>(a, ps, st);
  return launch_pipe_n<false, 0, kMode>(a, ps, st);
}


// ---- norm + per-token quantisation, pipelined across a CTA's rows --------
//
// The per-token modes with a norm (INT8 or FP8 codes) at one CTA barrier per
// row, and without the CTA waiting on a row's scalar chain.  Iteration i of a
// CTA (rows i, i + 1 of its own row sequence):
//   phase 1: the fp64 sums of row i + 1 (read from its buffer) and the
//            normalised values y of row i (its buffer again, with r_i, mu_i)
//            with their partial absmax;
//   barrier X_i (thread 0 has also seen row i + 2 land);
//   phase 2: row i's step and codes; one warp, rotating with the row, turns
//            row i + 1's sums into (r, mu) and publishes them through an
//            mbarrier, which the other warps wait on only when they reach
//            row i + 1's y in the next iteration.
// Row i's buffer is refilled after X_i (both of its reads precede it), so
// nbuf - 2 rows per CTA are in flight while the CTA computes.

struct RowScalars {
  float r, mu;
};

// (r, mu) of a row from its fp64 sums S2 = sum x^2 and S1 = sum x, equal to
// the fp32 roundings of the exact chain
//   ms = fl64(S2 / K), mu64 = fl64(S1 / K),
//   var = max(0, fl64(ms - fl64(mu64 mu64)))   (LayerNorm; RMSNorm: var = ms),
//   r = fl32(fl64(1 / fl64(sqrt(fl64(var + eps))))),  mu = fl32(mu64).
// Fast path: the divisions are products with invK = fl64(1 / K) (exact for a
// power-of-two K) and 1 / sqrt(v) is rsqrt(v) = A, whose own relative error
// d is measured: with t = fl64(v A), e = fl64(1 - t A) (one fused
// multiply-add) gives |d| <= 0.51 (|e| (1 + u) + 1.01 u), u = 2^-53.  Against
// the exact chain, the fast v differs by at most u (6 ms + 11 mu^2 + 2.1 v)
// (the product roundings: 2u on ms and mu against u in the chain, the
// square, the difference and the eps sum), the chain's own sqrt and
// reciprocal add 2.01u, so A is within
//   E = 1.05 (d + 2.01u + (3 ms + 5.5 mu^2) u / v + 1.05u) + 2^-60
// of the chain's fp64 r.  r's fp32 rounding is the chain's whenever the
// distance from A to the nearest fp32 rounding midpoint, in units of A's last
// place (the low 29 bits of its significand against 2^28), exceeds E 2^53 + 1;
// the test below checks 0.6 |e| 2^53 + 0.6 (6 ms + 11 mu^2) / v + 6 >= that
// (both sides times v).  mu's: |fast - chain| <= 3.02u |mu| (at most 6.04
// units of the last place; 8 is checked).  Otherwise (about one row in 10^7,
// or a value outside the normal ranges) the exact chain runs.
template <int NORMK>
__device__ __forceinline__ RowScalars row_scalars(double S2, double S1, double invK, double Kd,
                                                  float eps) {
  const double e64 = static_cast<double>(eps);
  const double ms = __dmul_rn(S2, invK);
  double mu = 0.0, m2 = 0.0, var = ms;
  if constexpr (NORMK == 2) {
    mu = __dmul_rn(S1, invK);
    m2 = __dmul_rn(mu, mu);
    var = __dsub_rn(ms, m2);
    if (var < 0.0) var = 0.0;
  }
  const double v = __dadd_rn(var, e64);
  const double A = rsqrt(v);
  const double e = __fma_rn(-__dmul_rn(v, A), A, 1.0);
  const double tau_v = 0.6 * fabs(e) * 0x1p53 * v + 0.6 * (6.0 * ms + 11.0 * m2) + 6.0 * v;
  const long long ab = __double_as_longlong(A);
  const double dist = fabs(static_cast<double>((ab & 0x1fffffffLL) - 0x10000000LL));
  bool ok = v >= 0x1p-1000 && v <= 0x1p1000 && fabs(e) <= 0x1p-20 && A >= 0x1p-125 &&
            A <= 0x1p125 && dist * v > tau_v;
  RowScalars rs;
  rs.r = __double2float_rn(A);
  rs.mu = 0.0f;
  if constexpr (NORMK == 2) {
    rs.mu = __double2float_rn(mu);
    if (mu != 0.0) {
      const long long dl = (__double_as_longlong(mu) & 0x1fffffffLL) - 0x10000000LL;
      ok = ok && fabs(mu) >= 0x1p-125 && fabs(mu) <= 0x1p125 && (dl > 8 || dl < -8);
    }
  }
  if (!ok) {
    // the exact chain, one IEEE operation per step
    const double msx = __ddiv_rn(S2, Kd);
    double varx = msx;
    if constexpr (NORMK == 2) {
      const double mux = __ddiv_rn(S1, Kd);
      varx = __dsub_rn(msx, __dmul_rn(mux, mux));
      if (varx < 0.0) varx = 0.0;
      rs.mu = __double2float_rn(mux);
    }
    rs.r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(varx, e64))));
  }
  return rs;
}

// This thread's fp64 partial sums (x^2; x for LayerNorm) over its chunks of
// a row in shared memory, two accumulators per sum.
// bf16 pair (low, high half of a word) -> two fp64 values, exactly
__device__ __forceinline__ void bf16x2_to_f64(uint32_t w, double& lo, double& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.f64.bf16 %0, l;\n\tcvt.f64.bf16 %1, h;\n\t}"
      : "=d"(lo), "=d"(hi)
      : "r"(w));
}

template <bool kBF16, int NORMK, int CH, bool kFull>
__device__ __forceinline__ void row_partial_sums(const uint8_t* rowp, int t, int T, int nchunks,
                                                 double& s2, double& s1) {
  // four accumulators per sum (element i of a chunk feeds accumulator i mod 4)
  double a1[4] = {0.0, 0.0, 0.0, 0.0}, a2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = t + c * T;
    if (kFull || ch < nchunks) {
      double d[8];
      if constexpr (kBF16) {
        const uint4 u = *reinterpret_cast<const uint4*>(rowp + ch * 16);
        bf16x2_to_f64(u.x, d[0], d[1]);
        bf16x2_to_f64(u.y, d[2], d[3]);
        bf16x2_to_f64(u.z, d[4], d[5]);
        bf16x2_to_f64(u.w, d[6], d[7]);
      } else {
        float2 v[4];
        smem_chunk<false>(rowp, ch, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d[2 * i] = static_cast<double>(v[i].x);
          d[2 * i + 1] = static_cast<double>(v[i].y);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if constexpr (NORMK == 2) a1[i & 3] = __dadd_rn(a1[i & 3], d[i]);
        a2[i & 3] = __fma_rn(d[i], d[i], a2[i & 3]);
      }
    }
  }
  s2 = __dadd_rn(__dadd_rn(a2[0], a2[1]), __dadd_rn(a2[2], a2[3]));
  s1 = __dadd_rn(__dadd_rn(a1[0], a1[1]), __dadd_rn(a1[2], a1[3]));
}

// Bounded wait for the scalars of a row (parity = the row's number in the
// CTA's sequence, mod 2).
__device__ __forceinline__ bool scalars_ready(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long c0 = clock64();
  for (uint32_t k = 0;; ++k) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((k & 63u) == 63u && clock64() - c0 > kWaitBudgetCycles) return false;
  }
}

// One warp: the row's sums (per-warp partials in a fixed order) -> (r, mu) in
// scal[2 slot .. 2 slot + 1]; lane 0 stores them and arrives on the barrier
// (release; the waiters' try_wait acquires).
template <int NORMK>
__device__ __forceinline__ void publish_scalars(const double* dslot, int nwarps, float* sslot,
                                                uint32_t sbar, double invK, double Kd, float eps,
                                                int lane) {
  double S2 = dslot[0], S1 = dslot[8];
  for (int w = 1; w < nwarps; ++w) {
    S2 = __dadd_rn(S2, dslot[w]);
    if constexpr (NORMK == 2) S1 = __dadd_rn(S1, dslot[8 + w]);
  }
  const RowScalars rs = row_scalars<NORMK>(S2, S1, invK, Kd, eps);
  if (lane == 0) {
    sslot[0] = rs.r;
    sslot[1] = rs.mu;
    mbar_arrive(sbar);
  }
}

// At most 8 warps (256 threads) a CTA, 4 or 8 chunks a thread.  TF > 0: the
// thread count is the compile-time constant TF and TF * CH chunks are the
// whole row (kFull), so every chunk offset is an immediate.
template <int TF, int CH>
struct RowsBounds {
  static constexpr int kThreads = TF > 0 ? TF : 256;
  static constexpr int kMinBlocks = (TF > 0 && TF <= 128) ? 4 : (CH <= 4 ? 3 : 2);
};  // 128 threads: 128 registers; 256 threads, 4 chunks: 85; 8 chunks: 128

template <bool kBF16, int NORMK, int CH, bool kGamma, bool kBeta, bool kFull, bool kF8, int TF>
__global__ void __launch_bounds__(RowsBounds<TF, CH>::kThreads, RowsBounds<TF, CH>::kMinBlocks)
    norm_quant_rows_kernel(const void* __restrict__ x, int64_t ldx, int64_t M, int K, double invK,
                           const float* __restrict__ gamma, const float* __restrict__ beta,
                           float eps, int8_t* __restrict__ q, float* __restrict__ scale, int nbuf,
                           int* error_word) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kEsz = kBF16 ? 2 : 4;
  static_assert(NORMK == 1 || NORMK == 2, "a norm kind");
  const uint32_t row_bytes = static_cast<uint32_t>(K) * kEsz;
  const uint32_t buf_stride = (row_bytes + 127u) & ~127u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + nbuf * buf_stride);  // [nbuf] + scalars
  double* dscr = reinterpret_cast<double*>(bars + nbuf + 1);  // [2 slots][sum x^2, sum x][8]
  float* scal = reinterpret_cast<float*>(dscr + 32);          // [2 slots][r, mu]
  unsigned int* smax = reinterpret_cast<unsigned int*>(scal + 4);  // [3] row absmax bits
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  const uint32_t sbar = bar_base + 8u * static_cast<uint32_t>(nbuf);

  static_assert(TF == 0 || kFull, "a compile-time thread count covers the whole row");
  const int t = threadIdx.x;
  const int T = TF > 0 ? TF : static_cast<int>(blockDim.x);
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nchunks = TF > 0 ? TF * CH : K / kChunk;
  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;
  const uint8_t* xb = static_cast<const uint8_t*>(x);
  const int64_t row_pitch = ldx * kEsz;
  const double Kd = static_cast<double>(K);
  // launched as a programmatic dependent: let the next kernel be scheduled,
  // and touch no global memory before the previous grid has completed
  if (t == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (t == 0) {
    for (int b = 0; b <= nbuf; ++b) mbar_init(bar_base + 8u * b, 1);
    smax[0] = 0u;
    smax[1] = 0u;
    smax[2] = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  int issued = 0;  // thread 0: row copies issued, in the CTA's row order
  if (t == 0) {
    for (int b = 0; b < nbuf; ++b) {
      const int64_t row = first + b * G;
      if (row < M) {
        mbar_arrive_expect_tx(bar_base + 8u * b, row_bytes);
        bulk_load(smem_base + b * buf_stride, xb + row * row_pitch, row_bytes, bar_base + 8u * b);
        issued = b + 1;
      }
    }
  }
  if (first >= M) return;

  // prologue: the sums and scalars of the CTA's first row
  bool aborted = false;
  {
    const bool ok = t != 0 || row_landed(bar_base, 0, 0u);
    if (__syncthreads_or(!ok)) aborted = true;
  }
  if (!aborted) {
    double s2, s1;
    row_partial_sums<kBF16, NORMK, CH, kFull>(smem, t, T, nchunks, s2, s1);
    s2 = warp_sum(s2);
    if constexpr (NORMK == 2) s1 = warp_sum(s1);
    if (lane == 0) {
      dscr[warp] = s2;
      dscr[8 + warp] = s1;
    }
    const bool ok = (t != 0 || first + G >= M) ? true : row_landed(bar_base, 1, 0u);
    if (__syncthreads_or(!ok)) aborted = true;
    else if (warp == 0)
      publish_scalars<NORMK>(dscr, nwarps, scal, sbar, invK, Kd, eps, lane);
  }

  int it = 0;
  int b_cur = 0, b_nxt = 1, b_nn = 2;  // buffers of rows it, it + 1, it + 2
  uint32_t p_nn = 0u;                  // phase parity of row it + 2's copy
  int s_cur = 0;                       // it mod 3
  int pub_warp = 0;                    // it mod nwarps: the warp that published row it
  for (int64_t row = first; row < M && !aborted; row += G, ++it) {
    const bool has_next = row + G < M;
    const int slot = it & 1, nslot = slot ^ 1;
    // ---- phase 1a: row it + 1's sums
    if (has_next) {
      double s2, s1;
      row_partial_sums<kBF16, NORMK, CH, kFull>(smem + b_nxt * buf_stride, t, T, nchunks, s2, s1);
      s2 = warp_sum(s2);
      if constexpr (NORMK == 2) s1 = warp_sum(s1);
      if (lane == 0) {
        dscr[nslot * 16 + warp] = s2;
        dscr[nslot * 16 + 8 + warp] = s1;
      }
    }
    // ---- phase 1b: row it's normalised values and their absmax
    bool ok = scalars_ready(sbar, static_cast<uint32_t>(slot));
    const float r = scal[2 * slot], mu = scal[2 * slot + 1];
    const float2 r2 = make_float2(r, r), nmu2 = make_float2(-mu, -mu);
    const uint8_t* rowp = smem + b_cur * buf_stride;
    float2 y[CH][4];
    float am = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (kFull || ch < nchunks) {
        float2 v[4], g[4], bt[4];
        smem_chunk<kBF16>(rowp, ch, v);
        if constexpr (kGamma) param8(gamma, ch, g);
        if constexpr (kBeta) param8(beta, ch, bt);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 yy = v[i];
          if constexpr (NORMK == 1) yy = __fmul2_rn(yy, r2);
          if constexpr (NORMK == 2) yy = __fmul2_rn(__fadd2_rn(yy, nmu2), r2);
          if constexpr (kBeta) {
            // a multiply followed by an add: the scalar intrinsics, which are
            // never contracted into a fused multiply-add (paired ones were, in
            // a LayerNorm test row, both as intrinsics and as explicit .rn PTX)
            if constexpr (kGamma) {
              yy.x = __fmul_rn(yy.x, g[i].x);
              yy.y = __fmul_rn(yy.y, g[i].y);
            }
            yy.x = __fadd_rn(yy.x, bt[i].x);
            yy.y = __fadd_rn(yy.y, bt[i].y);
          } else if constexpr (kGamma) {
            yy = __fmul2_rn(yy, g[i]);
          }
          am = fmaxf(am, fmaxf(fabsf(yy.x), fabsf(yy.y)));
          y[c][i] = yy;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) y[c][i] = make_float2(0.0f, 0.0f);
      }
    }
    // non-negative floats order like their bit patterns: integer max reduce
    const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(am));
    if (lane == 0) atomicMax(&smax[s_cur], wmax);
    if (t == 0 && row + 2 * G < M) ok = ok && row_landed(bar_base, b_nn, p_nn);
    if (__syncthreads_or(!ok)) {  // X
      aborted = true;
      break;
    }
    // ---- phase 2: row it's step and codes; row it + 1's scalars
    if (t == 0) {
      smax[s_cur == 0 ? 2 : s_cur - 1] = 0u;  // the slot of row it + 2
      issued = refill_row(smem_base, bar_base, buf_stride, row_bytes, nbuf, it, b_cur, row, G, M,
                          xb, row_pitch, issued);
    }
    const float amax = __uint_as_float(smax[s_cur]);
    int8_t* qrow = q + row * static_cast<int64_t>(K);
    if constexpr (kF8) {
      float step = __fdiv_rn(amax, 448.0f);
      if (!(step >= FLT_MIN)) step = 0.0f;
      const float inv = step > 0.0f ? __frcp_rn(step) : 0.0f;
      if (t == 0) scale[row] = step;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int ch = t + c * T;
        if (!kFull && ch >= nchunks) continue;
        const uint2 code = step > 0.0f ? codes8_f8(y[c], inv) : make_uint2(0u, 0u);
        *reinterpret_cast<uint2*>(qrow + ch * kChunk) = code;
      }
    } else {
      const float step = div127(amax);
      const bool exact_only = step < FLT_MIN;  // zero or subnormal step: no reciprocal
      float rhi = 0.0f, rlo = 0.0f;
      if (!exact_only) bracket_of(step, rhi, rlo);
      if (t == 0) scale[row] = step;
      // all of this thread's codes by bracketing, stored at once; then one
      // branch: any value the two roundings disagreed on (or a step without a
      // reciprocal) sends the thread's chunks of the row to the exact
      // division, whose codes overwrite them
      uint32_t diff = exact_only ? 1u : 0u;
      const float2 rh = make_float2(rhi, rhi), rl = make_float2(rlo, rlo);
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int ch = t + c * T;
        const uint2 code = bracket8(y[c], rh, rl, diff);
        if (kFull || ch < nchunks) *reinterpret_cast<uint2*>(qrow + ch * kChunk) = code;
      }
      if (diff != 0u) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int ch = t + c * T;
          if (kFull || ch < nchunks)
            *reinterpret_cast<uint2*>(qrow + ch * kChunk) = exact8(y[c], step);
        }
      }
    }
    if (++pub_warp == nwarps) pub_warp = 0;  // (it + 1) mod nwarps
    if (has_next && warp == pub_warp)
      publish_scalars<NORMK>(dscr + nslot * 16, nwarps, scal + 2 * nslot, sbar, invK, Kd, eps,
                             lane);
    b_cur = b_nxt;
    b_nxt = b_nn;
    if (++b_nn == nbuf) {
      b_nn = 0;
      p_nn ^= 1u;
    }
    s_cur = s_cur == 2 ? 0 : s_cur + 1;
  }
  if (aborted && t == 0) {
    record_device_error(error_word, SQ_ERR_PIPELINE_TIMEOUT);
    // let every bulk copy still in flight land before the CTA exits (the
    // latest copy into buffer b is the one of row number s = b mod nbuf,
    // s < issued, which completes phase s / nbuf of the buffer's barrier)
    for (int b = 0; b < nbuf && b < issued; ++b) {
      const int s_last = b + (issued - 1 - b) / nbuf * nbuf;
      const uint32_t par = static_cast<uint32_t>((s_last / nbuf) & 1);
      const long long c0 = clock64();
      while (!mbar_try_wait(bar_base + 8u * b, par) && clock64() - c0 < kWaitBudgetCycles) {
      }
    }
  }
}

struct RowsShape {
  int ch, threads, nbuf;
  size_t smem;
};

// row buffers, nbuf + 1 barriers, 32 doubles of sums, 4 floats of scalars, 3 absmax slots
size_t rows_smem(size_t stride, int nbuf) { return nbuf * stride + 8 * (nbuf + 1) + 32 * 8 + 32; }

// Rows up to kRows4 chunks (8 elements each) run 4 chunks a thread, wider
// ones 8 (at most 256 threads either way).
constexpr int kRows4 = 4 * 128;

bool rows_shape(int K, bool bf16, RowsShape* rs) {
  const int nchunks = K / kChunk;
  const int ch = nchunks <= kRows4 ? 4 : (nchunks <= 8 * 256 ? 8 : 0);
  if (!ch || nchunks < 1) return false;
  int threads = (nchunks + ch - 1) / ch;
  threads = (threads + 31) / 32 * 32;
  const size_t stride = (static_cast<size_t>(K) * (bf16 ? 2 : 4) + 127) / 128 * 128;
  // about 200 KB of row buffers per SM over the CTAs that fit it (their
  // registers decide: four of 128 threads, three of 256): two rows of each
  // CTA in use and the rest in flight
  const int ctas = (threads <= 128) ? 4 : 3;
  int nbuf = static_cast<int>((200u << 10) / ctas / stride);
  if (nbuf < 3) nbuf = 3;
  if (nbuf > 8) nbuf = 8;
  if (nbuf * stride > (200u << 10)) return false;
  rs->ch = ch;
  rs->threads = threads;
  rs->nbuf = nbuf;
  rs->smem = rows_smem(stride, nbuf);
  return true;
}

template <bool kBF16, int NORMK, int CH, bool kG, bool kB, bool kF, bool kF8, int TF = 0>
cudaError_t launch_rows_k(const RowArgs& a, RowsShape rs, cudaStream_t st) {
  auto kern = norm_quant_rows_kernel<kBF16, NORMK, CH, kG, kB, kF, kF8, TF>;
  const void* key = reinterpret_cast<const void*>(kern);
  LaunchCache& lc = launch_cache();
  const size_t stride = (static_cast<size_t>(a.K) * (kBF16 ? 2 : 4) + 127) / 128 * 128;
  int per_sm = 0;
  // fewer row buffers when each CTA sees only a few rows: more CTAs fit an SM
  for (;;) {
    const cudaError_t e = lc.ensure_smem(key, rs.smem);
    if (e != cudaSuccess) return e;
    per_sm = lc.blocks_per_sm(key, rs.threads, rs.smem);
    const int64_t ctas = static_cast<int64_t>(per_sm) * lc.sms();
    const int64_t rows_per_cta = (a.M + ctas - 1) / ctas;
    if (rs.nbuf <= 3 || rows_per_cta >= rs.nbuf) break;
    rs.nbuf = rows_per_cta < 3 ? 3 : static_cast<int>(rows_per_cta);
    rs.smem = rows_smem(stride, rs.nbuf);
  }
  int64_t grid = static_cast<int64_t>(per_sm) * lc.sms();
  if (grid > a.M) grid = a.M;
  const double invK = 1.0 / static_cast<double>(a.K);
  cudaLaunchConfig_t cfg = pdl_config(static_cast<unsigned>(grid), rs.threads, rs.smem, st);
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, a.x, a.ldx, a.M, a.K, invK, a.gamma,
                                            a.beta, a.eps, a.q, a.scale, rs.nbuf, a.err);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

template <bool kBF16, int NORMK, int CH, bool kG, bool kB, bool kF8>
cudaError_t launch_rows_f(const RowArgs& a, const RowsShape& rs, cudaStream_t st) {
  // bf16 rows whose chunks split evenly over the threads skip the bounds
  // checks; the common widths also fix the thread count at compile time
  // (4096: 128 x 4 chunks, 8192: 128 x 8, 16384: 256 x 8)
  if constexpr (kBF16) {
    if (rs.threads * rs.ch == a.K / kChunk) {
      if (rs.threads == 128) return launch_rows_k<kBF16, NORMK, CH, kG, kB, true, kF8, 128>(a, rs, st);
      if (rs.threads == 256) return launch_rows_k<kBF16, NORMK, CH, kG, kB, true, kF8, 256>(a, rs, st);
      return launch_rows_k<kBF16, NORMK, CH, kG, kB, true, kF8>(a, rs, st);
    }
  }
  return launch_rows_k<kBF16, NORMK, CH, kG, kB, false, kF8>(a, rs, st);
}

template <bool kBF16, int NORMK, int CH, bool kF8>
cudaError_t launch_rows_g(const RowArgs& a, const RowsShape& rs, cudaStream_t st) {
  const bool hb = NORMK == 2 && a.beta != nullptr;
  if (a.gamma) {
    if (hb) return launch_rows_f<kBF16, NORMK, CH, true, NORMK == 2, kF8>(a, rs, st);
    return launch_rows_f<kBF16, NORMK, CH, true, false, kF8>(a, rs, st);
  }
  if (hb) return launch_rows_f<kBF16, NORMK, CH, false, NORMK == 2, kF8>(a, rs, st);
  return launch_rows_f<kBF16, NORMK, CH, false, false, kF8>(a, rs, st);
}

template <bool kBF16, int NORMK, bool kF8>
cudaError_t launch_rows_c(const RowArgs& a, const RowsShape& rs, cudaStream_t st) {
  if (rs.ch == 4) return launch_rows_g<kBF16, NORMK, 4, kF8>(a, rs, st);
  return launch_rows_g<kBF16, NORMK, 8, kF8>(a, rs, st);
}

// Per-token quantisation with a norm through norm_quant_rows_kernel; false
// when the shape is not one it takes.
template <bool kF8>
bool launch_norm_rows(const RowArgs& a, bool bf16, int norm, cudaStream_t st, cudaError_t* e) {
  RowsShape rs;
  if ((norm != SQ_NORM_RMS && norm != SQ_NORM_LAYER) || !rows_shape(a.K, bf16, &rs)) return false;
  if (bf16)
    *e = norm == SQ_NORM_RMS ? launch_rows_c<true, 1, kF8>(a, rs, st)
                             : launch_rows_c<true, 2, kF8>(a, rs, st);
  else
    *e = norm == SQ_NORM_RMS ? launch_rows_c<false, 1, kF8>(a, rs, st)
                             : launch_rows_c<false, 2, kF8>(a, rs, st);
  return true;
}

}  // namespace

bool norm_quant_pipe_supported(int K, bool bf16) {
  PipeShape ps;
  return pipe_shape(K, bf16, false, &ps);
}

bool calibrate_pipe_supported(int K, bool bf16) {
  PipeShape ps;
  return pipe_shape(K, bf16, true, &ps) && ps.ch == 4;
}

cudaError_t launch_norm_quant_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                   int norm, const float* gamma, const float* beta, float eps,
                                   int8_t* q, float* scale, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const RowArgs a{x, M, K, ldx, gamma, beta, eps, q, scale, nullptr, err};
  cudaError_t e = cudaSuccess;
  if (launch_norm_rows<false>(a, bf16, norm, st, &e)) return e;
  return launch_rows<kModeRowQuant>(a, bf16, norm, st);
}

cudaError_t launch_calibrate_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                  int norm, const float* gamma, const float* beta, float eps,
                                  float* act_max, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const RowArgs a{x, M, K, ldx, gamma, beta, eps, nullptr, nullptr, act_max, err};
  return launch_rows<kModeColMax>(a, bf16, norm, st);
}

cudaError_t launch_tensor_absmax_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                      int norm, const float* gamma, const float* beta, float eps,
                                      float* absmax, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const RowArgs a{x, M, K, ldx, gamma, beta, eps, nullptr, nullptr, absmax, err};
  return launch_rows<kModeTensorMax>(a, bf16, norm, st);
}

cudaError_t launch_quant_fixed_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                    int norm, const float* gamma, const float* beta, float eps,
                                    const float* absmax, int8_t* q, float* scale, int* err,
                                    cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const RowArgs a{x, M, K, ldx, gamma, beta, eps, q, scale, const_cast<float*>(absmax), err};
  return launch_rows<kModeFixedQuant>(a, bf16, norm, st);
}

cudaError_t launch_quant_given_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                    const float* row_absmax, int8_t* q, float* scale, int* err,
                                    cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  PipeShape ps;
  if (!pipe_shape(K, bf16, false, &ps)) return cudaErrorInvalidValue;
  const RowArgs a{x, M, K, ldx, nullptr, nullptr, 0.0f, q, scale,
                  const_cast<float*>(row_absmax), err};
  if (bf16) return launch_pipe_n<true, 0, kModeGivenQuant>(a, ps, st);
  return launch_pipe_n<false, 0, kModeGivenQuant>(a, ps, st);
}

cudaError_t launch_row_absmax_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                   float* row_absmax, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  PipeShape ps;
  if (!pipe_shape(K, bf16, false, &ps)) return cudaErrorInvalidValue;
  const RowArgs a{x, M, K, ldx, nullptr, nullptr, 0.0f, nullptr, nullptr, row_absmax, err};
  if (bf16) return launch_pipe_n<true, 0, kModeRowAbsmax>(a, ps, st);
  return launch_pipe_n<false, 0, kModeRowAbsmax>(a, ps, st);
}

bool silu_mul_pipe_supported(int I) {
  PipeShape ps;
  return pipe_shape(I, true, false, &ps, 2);
}

cudaError_t launch_silu_mul_quant_pipe(const void* gu, int64_t M, int I, int64_t ldgu,
                                       int8_t* q, float* scale, void* h_out, int64_t ldh,
                                       int* err, cudaStream_t st, bool fp8) {
  if (M == 0) return cudaSuccess;
  PipeShape ps;
  if (!pipe_shape(I, true, false, &ps, 2)) return cudaErrorInvalidValue;
  RowArgs a{gu, M, I, ldgu, nullptr, nullptr, 0.0f, q, scale, nullptr, err};
  a.h_out = static_cast<__nv_bfloat16*>(h_out);
  a.ldh = ldh;
  if (fp8) return launch_pipe_t<true, 0, 4, false, false, kModeSiluMulF8>(a, ps, st);
  return launch_pipe_t<true, 0, 4, false, false, kModeSiluMul>(a, ps, st);
}

cudaError_t launch_norm_quant_fp8_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                       int norm, const float* gamma, const float* beta,
                                       float eps, uint8_t* q, float* scale, int* err,
                                       cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const RowArgs a{x, M, K, ldx, gamma, beta, eps, reinterpret_cast<int8_t*>(q), scale, nullptr,
                  err};
  cudaError_t e = cudaSuccess;
  if (launch_norm_rows<true>(a, bf16, norm, st, &e)) return e;
  return launch_rows<kModeRowQuantF8>(a, bf16, norm, st);
}

}  // namespace sq
