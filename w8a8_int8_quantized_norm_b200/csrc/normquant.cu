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
//   * the quantiser avoids a division per element: with r = fl32(1/step) the
//     product t = fl32(y r) is within 3 * 2^-24 relative of y/step, so
//     rne(fl32(y/step)) = rne(t) unless y/step lies within 1e-4 of a
//     half-integer; a chunk of 8 values holding such a quotient is redone
//     with the exact division (branch-free otherwise).  Rounding to the
//     nearest integer (ties to even) is the float add of 1.5 * 2^23, whose low
//     8 mantissa bits are then the two's-complement INT8 code.
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
// within 3 * 2^-24 relative of v / step and |P| < 127.5, so the code equals
// the exact one -- no clamp needed -- unless v / step lies within 1e-4 of a
// half-integer.  The residual P - n (one more fused multiply-add) flags that
// case; a chunk holding such a value, or a step without a finite reciprocal,
// is recomputed from the exact quotient.
__device__ __forceinline__ uint2 codes8(const float2 (&v)[4], float rstep, float step,
                                        bool exact_only) {
  uint32_t m[8];
  float dmax = 0.0f;
  const float2 rs = make_float2(rstep, rstep);
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // paired fp32 instructions: each component rounds exactly like the scalar op
    const float2 mf = __ffma2_rn(v[i], rs, mg);
    const float2 n = __fadd2_rn(mf, make_float2(-kMagic, -kMagic));
    const float2 d = __ffma2_rn(v[i], rs, make_float2(-n.x, -n.y));
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
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

// NORMK: 0 = no norm (optional per-channel multiplier), 1 = RMSNorm, 2 = LayerNorm.
template <int CH>
struct PipeBounds {
  static constexpr int kMaxThreads = CH <= 4 ? 512 : 640;
  // 4-chunk CTAs keep to 64 registers a thread so four 256-thread CTAs fit an SM
  static constexpr int kMinBlocks = CH <= 4 ? 2 : 1;
};

// kFull: every thread owns all CH of its chunks (T * CH == K / 8): no bounds checks.
template <bool kBF16, int NORMK, int CH, bool kGamma, bool kBeta, bool kFull>
__global__ void __launch_bounds__(PipeBounds<CH>::kMaxThreads, PipeBounds<CH>::kMinBlocks)
    norm_quant_pipe_kernel(
    const void* __restrict__ x, int64_t ldx, int64_t M, int K, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int8_t* __restrict__ q, float* __restrict__ scale,
    int nbuf, int* error_word) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kEsz = kBF16 ? 2 : 4;
  const uint32_t row_bytes = static_cast<uint32_t>(K) * kEsz;
  const uint32_t buf_stride = (row_bytes + 127u) & ~127u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + nbuf * buf_stride);
  double* dscr = reinterpret_cast<double*>(bars + nbuf);      // [64]: sum x^2, sum x per warp
  float* fscr = reinterpret_cast<float*>(dscr + 64);           // [2]: r, mu of the row
  unsigned int* smax = reinterpret_cast<unsigned int*>(fscr + 2);  // [2]: row absmax bits
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);

  const int t = threadIdx.x, T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nchunks = K / kChunk;
  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;
  const uint8_t* xb = static_cast<const uint8_t*>(x);
  const int64_t row_pitch = ldx * kEsz;

  if (t == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(bar_base + 8u * b, 1);
    smax[0] = 0u;
    smax[1] = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  int last_phase[8];  // thread 0: phase of the latest copy issued into each buffer (-1: none)
#pragma unroll
  for (int b = 0; b < 8; ++b) last_phase[b] = (b < nbuf && first + b * G < M) ? 0 : -1;
  if (t == 0) {
    for (int b = 0; b < nbuf; ++b) {
      const int64_t row = first + b * G;
      if (row < M) {
        mbar_arrive_expect_tx(bar_base + 8u * b, row_bytes);
        bulk_load(smem_base + b * buf_stride, xb + row * row_pitch, row_bytes, bar_base + 8u * b);
      }
    }
  }

  int it = 0;
  bool aborted = false;
  for (int64_t row = first; row < M; row += G, ++it) {
    const int b = it % nbuf;
    const int slot = it & 1;
    // one thread watches the row's barrier; the others sleep in the CTA barrier
    bool ok = true;
    if (t == 0) {
      const uint32_t parity = static_cast<uint32_t>((it / nbuf) & 1);
      ok = mbar_try_wait(bar_base + 8u * b, parity);
      if (!ok) {
        const long long c0 = clock64();
        for (uint32_t i = 0; !ok; ++i) {
          ok = mbar_try_wait(bar_base + 8u * b, parity);
          if (!ok && (i & 63u) == 63u && clock64() - c0 > kWaitBudgetCycles) break;
        }
      }
    }
    if (__syncthreads_or(!ok)) {
      if (t == 0) record_device_error(error_word, SQ_ERR_PIPELINE_TIMEOUT);
      aborted = true;
      break;
    }
    // all threads are past the previous row: refill its buffer
    if (t == 0 && it > 0) {
      const int pb = (it - 1) % nbuf;
      const int64_t nrow = row - G + static_cast<int64_t>(nbuf) * G;
      if (nrow < M) {
        mbar_arrive_expect_tx(bar_base + 8u * pb, row_bytes);
        bulk_load(smem_base + pb * buf_stride, xb + nrow * row_pitch, row_bytes,
                  bar_base + 8u * pb);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k == pb) ++last_phase[k];
      }
    }
    const uint8_t* rowp = smem + b * buf_stride;

    // ---- load this thread's chunks of the row from shared memory
    float2 v[CH][4];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (kFull || ch < nchunks) {
        smem_chunk<kBF16>(rowp, ch, v[c]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[c][i] = make_float2(0.0f, 0.0f);
      }
    }
    // ---- row statistics in fp64 (two accumulators per sum for ILP)
    float mu = 0.0f, r = 1.0f;
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
      __syncthreads();
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
      __syncthreads();
      r = fscr[0];
      mu = fscr[1];
    }
    // ---- the norm output and its absmax (paired fp32 ops, same roundings;
    // a multiply followed by an add uses the scalar intrinsics, which are
    // never contracted into a fused multiply-add)
    float am = 0.0f;
    const float2 r2 = make_float2(r, r), nmu2 = make_float2(-mu, -mu);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
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
        v[c][i] = y;
        am = fmaxf(am, fmaxf(fabsf(y.x), fabsf(y.y)));
      }
    }
    // non-negative floats order like their bit patterns: integer max reduce
    const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(am));
    if (lane == 0) atomicMax(&smax[slot], wmax);
    __syncthreads();
    am = __uint_as_float(smax[slot]);
    if (t == 0) smax[slot ^ 1] = 0u;  // the next row's slot starts from zero

    // ---- per-token INT8 quantisation
    const float step = __fdiv_rn(am, 127.0f);
    const bool exact_only = step < FLT_MIN;  // zero or subnormal step: no reciprocal
    const float rstep = exact_only ? 0.0f : __fdiv_rn(1.0f, step);
    if (t == 0) scale[row] = step;
    int8_t* qrow = q + row * static_cast<int64_t>(K);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (!kFull && ch >= nchunks) continue;
      *reinterpret_cast<uint2*>(qrow + ch * kChunk) = codes8(v[c], rstep, step, exact_only);
    }
  }
  if (aborted && t == 0) {
    // let every bulk copy still in flight land before the CTA exits
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (last_phase[b] < 0) continue;
      const uint32_t par = static_cast<uint32_t>(last_phase[b] & 1);
      const long long c0 = clock64();
      while (!mbar_try_wait(bar_base + 8u * b, par) && clock64() - c0 < kWaitBudgetCycles) {
      }
    }
  }
}

struct PipeShape {
  int ch, threads, nbuf;
  size_t smem;
};

bool pipe_shape(int K, bool bf16, PipeShape* ps) {
  const int nchunks = K / kChunk;
  // chunks per thread and threads per CTA within the variant's register budget
  int ch = nchunks <= 4 * PipeBounds<4>::kMaxThreads ? 4
           : (nchunks <= 8 * PipeBounds<8>::kMaxThreads ? 8 : 0);
  if (!ch) return false;
  int threads = (nchunks + ch - 1) / ch;
  threads = (threads + 31) / 32 * 32;
  if (threads < 32) threads = 32;
  const size_t row_bytes = static_cast<size_t>(K) * (bf16 ? 2 : 4);
  const size_t stride = (row_bytes + 127) / 128 * 128;
  int nbuf = static_cast<int>((48u << 10) / stride);
  if (nbuf < 3) nbuf = 3;
  if (nbuf > 8) nbuf = 8;
  while (nbuf > 2 && nbuf * stride > (150u << 10)) --nbuf;
  if (nbuf * stride > (200u << 10)) return false;
  ps->ch = ch;
  ps->threads = threads;
  ps->nbuf = nbuf;
  ps->smem = nbuf * stride + 8 * nbuf + 64 * 8 + 4 * 4;
  return true;
}

template <bool kBF16, int NORMK, int CH, bool kG, bool kB, bool kF>
cudaError_t launch_pipe_k(const void* x, int64_t M, int K, int64_t ldx, const float* gamma,
                          const float* beta, float eps, int8_t* q, float* scale,
                          const PipeShape& ps, int* err, cudaStream_t st) {
  auto kern = norm_quant_pipe_kernel<kBF16, NORMK, CH, kG, kB, kF>;
  LaunchCache& lc = launch_cache();
  const cudaError_t e = lc.ensure_smem(reinterpret_cast<const void*>(kern), ps.smem);
  if (e != cudaSuccess) return e;
  const int per_sm = lc.blocks_per_sm(reinterpret_cast<const void*>(kern), ps.threads, ps.smem);
  int64_t grid = static_cast<int64_t>(per_sm) * lc.sms();
  if (grid > M) grid = M;
  kern<<<static_cast<unsigned>(grid), ps.threads, ps.smem, st>>>(x, ldx, M, K, gamma, beta, eps,
                                                                   q, scale, ps.nbuf, err);
  return cudaGetLastError();
}

template <bool kBF16, int NORMK, int CH, bool kG, bool kB>
cudaError_t launch_pipe_t(const void* x, int64_t M, int K, int64_t ldx, const float* gamma,
                          const float* beta, float eps, int8_t* q, float* scale,
                          const PipeShape& ps, int* err, cudaStream_t st) {
  // bf16 rows whose chunks split evenly over the threads skip the bounds checks
  if constexpr (kBF16) {
    if (ps.threads * ps.ch == K / kChunk)
      return launch_pipe_k<kBF16, NORMK, CH, kG, kB, true>(x, M, K, ldx, gamma, beta, eps, q,
                                                           scale, ps, err, st);
  }
  return launch_pipe_k<kBF16, NORMK, CH, kG, kB, false>(x, M, K, ldx, gamma, beta, eps, q, scale,
                                                        ps, err, st);
}

template <bool kBF16, int NORMK, int CH>
cudaError_t launch_pipe_c(const void* x, int64_t M, int K, int64_t ldx, const float* gamma,
                          const float* beta, float eps, int8_t* q, float* scale,
                          const PipeShape& ps, int* err, cudaStream_t st) {
  // beta only matters for LayerNorm
  const bool hb = NORMK == 2 && beta != nullptr;
  if (gamma) {
    if (hb) return launch_pipe_t<kBF16, NORMK, CH, true, NORMK == 2>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
    return launch_pipe_t<kBF16, NORMK, CH, true, false>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  }
  if (hb) return launch_pipe_t<kBF16, NORMK, CH, false, NORMK == 2>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  return launch_pipe_t<kBF16, NORMK, CH, false, false>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
}

template <bool kBF16, int NORMK>
cudaError_t launch_pipe_n(const void* x, int64_t M, int K, int64_t ldx, const float* gamma,
                          const float* beta, float eps, int8_t* q, float* scale,
                          const PipeShape& ps, int* err, cudaStream_t st) {
  if (ps.ch == 4)
    return launch_pipe_c<kBF16, NORMK, 4>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  return launch_pipe_c<kBF16, NORMK, 8>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
}

}  // namespace

bool norm_quant_pipe_supported(int K, bool bf16) {
  PipeShape ps;
  return pipe_shape(K, bf16, &ps);
}

cudaError_t launch_norm_quant_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                   int norm, const float* gamma, const float* beta, float eps,
                                   int8_t* q, float* scale, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  PipeShape ps;
  if (!pipe_shape(K, bf16, &ps)) return cudaErrorInvalidValue;
  if (bf16) {
    if (norm == SQ_NORM_RMS)
      return launch_pipe_n<true, 1>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
    if (norm == SQ_NORM_LAYER)
      return launch_pipe_n<true, 2>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
    return launch_pipe_n<true, 0>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  }
  if (norm == SQ_NORM_RMS)
    return launch_pipe_n<false, 1>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  if (norm == SQ_NORM_LAYER)
    return launch_pipe_n<false, 2>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
  return launch_pipe_n<false, 0>(x, M, K, ldx, gamma, beta, eps, q, scale, ps, err, st);
}

}  // namespace sq
