// rows.cu -- the row-wise kernels of the SmoothQuant W8A8 path on sm_100a:
//   * fused norm (carrying the folded 1/s) + per-token absmax INT8 quantise
//     (also used, in multiplier mode, to smooth and quantise weight rows);
//   * calibration: running per-channel absmax of the norm output;
//   * weight column absmax and the smoothing-factor / fold finalisation.
//
// Source pages (by title and section):
//   "SmoothQuant, in depth" -- "Where the scales go in a decoder block" (fold
//   1/s into gamma/beta), "The calibration data flow" (running max, the eps
//   clamps), "Granularity" (per-token activation and per-channel weight
//   scales); "LLM.int8() and SmoothQuant" -- "going deeper" (s_j formula,
//   W-hat = diag(s) W), "Try it" (step = max / 127).
//
// Memory layout: one CTA per row, 128-bit coalesced loads: thread t owns the
// 8-element chunks t, t + T, t + 2T, ... of its row and keeps them in
// registers through the three passes (statistics, normalise + absmax,
// quantise), so every input byte is read from HBM once and every code
// written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_launch.h"

namespace sq {
namespace {

constexpr int kChunk = 8;  // elements per 128-bit (bf16) chunk

template <bool kBF16>
__device__ __forceinline__ void load_chunk(const void* base, int64_t elem, float (&v)[kChunk]) {
  if constexpr (kBF16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void load_param8(const float* p, int64_t elem, float (&v)[kChunk]) {
  const float4* q = reinterpret_cast<const float4*>(p + elem);
  const float4 a = __ldg(q), b = __ldg(q + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T* scratch /* >= 32 */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  __syncthreads();  // scratch may still be read by a previous reduction
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = scratch[0];
  for (int w = 1; w < nwarps; ++w) r = op(r, scratch[w]);
  return r;
}

struct AddD {
  __device__ double operator()(double a, double b) const { return __dadd_rn(a, b); }
};
struct MaxF {
  __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

// Loads this thread's chunks of row `row` and replaces them by the norm
// output y.  Every fp operation is an explicit round-to-nearest intrinsic so
// the compiler cannot contract or reorder it.
template <bool kBF16, int CH>
__device__ __forceinline__ void norm_row(const void* x, int64_t row_off, int nchunks, int K,
                                         int norm, const float* gamma, const float* beta,
                                         float eps, float (&v)[CH][kChunk], double* dscratch) {
  const int t = threadIdx.x, T = blockDim.x;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = t + c * T;
    if (ch < nchunks) {
      load_chunk<kBF16>(x, row_off + (int64_t)ch * kChunk, v[c]);
    } else {
#pragma unroll
      for (int i = 0; i < kChunk; ++i) v[c][i] = 0.0f;
    }
  }
  float mu = 0.0f, r = 1.0f;
  if (norm != SQ_NORM_NONE) {
    double s1 = 0.0, s2 = 0.0;
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        const double d = static_cast<double>(v[c][i]);
        s1 = __dadd_rn(s1, d);
        s2 = __fma_rn(d, d, s2);  // d*d is exact in binary64
      }
    const double S1 = block_reduce(s1, AddD(), dscratch);
    const double S2 = block_reduce(s2, AddD(), dscratch);
    const double ms = __ddiv_rn(S2, static_cast<double>(K));
    double var;
    if (norm == SQ_NORM_RMS) {
      var = ms;
    } else {
      const double mu64 = __ddiv_rn(S1, static_cast<double>(K));
      var = __dsub_rn(ms, __dmul_rn(mu64, mu64));
      if (var < 0.0) var = 0.0;
      mu = __double2float_rn(mu64);
    }
    const double rs = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps))));
    r = __double2float_rn(rs);
  }
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = t + c * T;
    if (ch >= nchunks) continue;
    float g[kChunk], b[kChunk];
    if (gamma) load_param8(gamma, (int64_t)ch * kChunk, g);
    if (beta && norm == SQ_NORM_LAYER) load_param8(beta, (int64_t)ch * kChunk, b);
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      float y = v[c][i];
      if (norm == SQ_NORM_RMS) {
        y = __fmul_rn(y, r);
        if (gamma) y = __fmul_rn(y, g[i]);
      } else if (norm == SQ_NORM_LAYER) {
        y = __fmul_rn(__fsub_rn(y, mu), r);
        if (gamma) y = __fmul_rn(y, g[i]);
        if (beta) y = __fadd_rn(y, b[i]);
      } else if (gamma) {
        y = __fmul_rn(y, g[i]);
      }
      v[c][i] = y;
    }
  }
}

// One CTA per row: y = norm(x) (or x * multiplier), scale = fl32(absmax/127),
// q = clamp(rne(fl32(y/scale)), +-127).
// Threads per CTA are capped so that CH chunks of fp32 values fit in registers.
template <int CH>
struct RowBounds {
  static constexpr int kMaxThreads = CH <= 4 ? 1024 : 640;
};

template <bool kBF16, int CH>
__global__ void __launch_bounds__(RowBounds<CH>::kMaxThreads) norm_quant_kernel(const void* __restrict__ x, int64_t ldx,
                                                          int K, int norm,
                                                          const float* __restrict__ gamma,
                                                          const float* __restrict__ beta, float eps,
                                                          int8_t* __restrict__ q,
                                                          float* __restrict__ scale) {
  __shared__ double dscratch[32];
  __shared__ float fscratch[32];
  const int64_t row = blockIdx.x;
  const int nchunks = K / kChunk;
  float v[CH][kChunk];
  norm_row<kBF16, CH>(x, row * ldx, nchunks, K, norm, gamma, beta, eps, v, dscratch);
  float am = 0.0f;
#pragma unroll
  for (int c = 0; c < CH; ++c)
#pragma unroll
    for (int i = 0; i < kChunk; ++i) am = fmaxf(am, fabsf(v[c][i]));
  am = block_reduce(am, MaxF(), fscratch);
  const float step = __fdiv_rn(am, 127.0f);
  if (threadIdx.x == 0) scale[row] = step;
  const int t = threadIdx.x, T = blockDim.x;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = t + c * T;
    if (ch >= nchunks) continue;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      const uint32_t b = static_cast<uint32_t>(quant_code(v[c][i], step)) & 0xffu;
      w[i >> 2] |= b << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(q + row * (int64_t)K + (int64_t)ch * kChunk) = make_uint2(w[0], w[1]);
  }
}

// Calibration: `rows_per_cta` rows per CTA; the per-channel max of |y| is
// kept in shared memory (each thread updates only its own channels) and merged
// into act_max with an atomic max on the bit pattern (non-negative binary32
// values order like their unsigned bit patterns).
template <bool kBF16, int CH>
__global__ void __launch_bounds__(RowBounds<CH>::kMaxThreads) calib_kernel(
    const void* __restrict__ x, int64_t ldx, int64_t M, int K, int rows_per_cta, int norm,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
    float* __restrict__ act_max) {
  __shared__ double dscratch[32];
  extern __shared__ float colmax[];  // [K]
  const int nchunks = K / kChunk;
  const int t = threadIdx.x, T = blockDim.x;
  for (int j = t; j < K; j += T) colmax[j] = 0.0f;
  const int64_t r0 = (int64_t)blockIdx.x * rows_per_cta;
  const int64_t r1 = min(M, r0 + rows_per_cta);
  for (int64_t row = r0; row < r1; ++row) {
    float v[CH][kChunk];
    norm_row<kBF16, CH>(x, row * ldx, nchunks, K, norm, gamma, beta, eps, v, dscratch);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = t + c * T;
      if (ch >= nchunks) continue;
#pragma unroll
      for (int i = 0; i < kChunk; ++i)
        colmax[ch * kChunk + i] = fmaxf(colmax[ch * kChunk + i], fabsf(v[c][i]));
    }
  }
  for (int ch = t; ch < nchunks; ch += T)
#pragma unroll
    for (int i = 0; i < kChunk; ++i)
      atomicMax(reinterpret_cast<unsigned int*>(act_max) + (int64_t)ch * kChunk + i,
                __float_as_uint(colmax[ch * kChunk + i]));
}

// Column absmax of a weight [N, K].  A CTA owns a slab of 256 columns (one
// 8-column chunk per lane, so every warp reads 512 contiguous bytes of a bf16
// row) and a run of rows, split over its 8 warps with 8 independent 16-byte
// loads in flight per thread; the warps' maxima meet in shared memory, and
// each column is merged into wmax with an atomic max on the bit pattern --
// issued only where this CTA's value beats the one already there.
template <bool kBF16>
__global__ void __launch_bounds__(256) weight_colmax_kernel(const void* __restrict__ W, int64_t N,
                                                            int K, int64_t rows_per_cta,
                                                            float* __restrict__ wmax) {
  __shared__ __align__(16) float red[8][kChunk * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = K / kChunk;
  const int ch = blockIdx.x * 32 + lane;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r1 = r0 + rows_per_cta < N ? r0 + rows_per_cta : N;
  float m[kChunk];
#pragma unroll
  for (int i = 0; i < kChunk; ++i) m[i] = 0.0f;
  if (ch < nchunks) {
    constexpr int U = 8;
    int64_t n = r0 + warp;
    for (; n + 8 * (U - 1) < r1; n += 8 * U) {
      float v[U][kChunk];
#pragma unroll
      for (int u = 0; u < U; ++u)
        load_chunk<kBF16>(W, (n + 8 * u) * static_cast<int64_t>(K) + static_cast<int64_t>(ch) * kChunk,
                          v[u]);
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int i = 0; i < kChunk; ++i) m[i] = fmaxf(m[i], fabsf(v[u][i]));
    }
    for (; n < r1; n += 8) {
      float v[kChunk];
      load_chunk<kBF16>(W, n * static_cast<int64_t>(K) + static_cast<int64_t>(ch) * kChunk, v);
#pragma unroll
      for (int i = 0; i < kChunk; ++i) m[i] = fmaxf(m[i], fabsf(v[i]));
    }
  }
  float4* dst = reinterpret_cast<float4*>(&red[warp][lane * kChunk]);
  dst[0] = make_float4(m[0], m[1], m[2], m[3]);
  dst[1] = make_float4(m[4], m[5], m[6], m[7]);
  __syncthreads();
  // column of the slab, rotated by the CTA's row run so that concurrent CTAs
  // of one slab merge into different L2 lines
  const int j = static_cast<int>((threadIdx.x + blockIdx.y * 37u) % (kChunk * 32));
  float v = red[0][j];
#pragma unroll
  for (int w = 1; w < 8; ++w) v = fmaxf(v, red[w][j]);
  const int64_t col = static_cast<int64_t>(blockIdx.x) * (kChunk * 32) + j;
  if (col < K) {
    unsigned int* p = reinterpret_cast<unsigned int*>(wmax) + col;
    const unsigned int bits = __float_as_uint(v);
    if (bits > __ldcg(p)) atomicMax(p, bits);
  }
}

// s_j = max(max(a,eps)^alpha / max(w,eps)^(1-alpha), eps) in binary64, stored
// as binary32; gamma' = gamma / s, beta' = beta / s.  w = wmax[j]; `s` may be
// `wmax` itself (each thread reads its channel before writing it).
__global__ void smooth_finalize_kernel(const float* __restrict__ act_max, const float* wmax,
                                       float* s, int K,
                                       double alpha, float clamp_eps,
                                       const float* __restrict__ gamma,
                                       const float* __restrict__ beta, float* __restrict__ gf,
                                       float* __restrict__ bfo) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double eps = static_cast<double>(clamp_eps);
  const double a = fmax(static_cast<double>(act_max[j]), eps);
  const double w = fmax(static_cast<double>(wmax[j]), eps);
  double sj = __ddiv_rn(pow(a, alpha), pow(w, __dsub_rn(1.0, alpha)));
  if (sj < eps) sj = eps;
  const float s32 = __double2float_rn(sj);
  s[j] = s32;
  gf[j] = __fdiv_rn(gamma ? gamma[j] : 1.0f, s32);
  if (beta && bfo) bfo[j] = __fdiv_rn(beta[j], s32);
}

// elements-per-thread choice: CH chunks of 8 per thread within the CTA cap
int pick_ch(int K) {
  const int nchunks = K / kChunk;
  if (nchunks <= 4 * RowBounds<4>::kMaxThreads) return 4;
  if (nchunks <= 8 * RowBounds<8>::kMaxThreads) return 8;
  return 0;
}

int threads_for(int K, int ch) {
  const int nchunks = K / kChunk;
  int t = (nchunks + ch - 1) / ch;
  t = (t + 31) / 32 * 32;
  return t < 32 ? 32 : t;
}

}  // namespace

cudaError_t launch_norm_quant(const void* x, bool bf16, int64_t M, int K, int64_t ldx, int norm,
                              const float* gamma, const float* beta, float eps, int8_t* q,
                              float* scale, int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  // rows that fit the shared-memory ring take the pipelined kernel; very wide
  // rows keep everything in registers instead
  if (norm_quant_pipe_supported(K, bf16))
    return launch_norm_quant_pipe(x, bf16, M, K, ldx, norm, gamma, beta, eps, q, scale, err, st);
  const int ch = pick_ch(K);
  const int threads = threads_for(K, ch);
  const dim3 grid(static_cast<unsigned>(M));
  if (bf16) {
    if (ch == 4)
      norm_quant_kernel<true, 4><<<grid, threads, 0, st>>>(x, ldx, K, norm, gamma, beta, eps, q, scale);
    else
      norm_quant_kernel<true, 8><<<grid, threads, 0, st>>>(x, ldx, K, norm, gamma, beta, eps, q, scale);
  } else {
    if (ch == 4)
      norm_quant_kernel<false, 4><<<grid, threads, 0, st>>>(x, ldx, K, norm, gamma, beta, eps, q, scale);
    else
      norm_quant_kernel<false, 8><<<grid, threads, 0, st>>>(x, ldx, K, norm, gamma, beta, eps, q, scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_calibrate(const void* x, bool bf16, int64_t M, int K, int64_t ldx, int norm,
                             const float* gamma, const float* beta, float eps, float* act_max,
                             int* err, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  // rows that fit the shared-memory ring (and a 4-chunk thread layout) take
  // the pipelined kernel; wider rows keep a column max in shared memory
  if (calibrate_pipe_supported(K, bf16))
    return launch_calibrate_pipe(x, bf16, M, K, ldx, norm, gamma, beta, eps, act_max, err, st);
  const int ch = pick_ch(K);
  const int threads = threads_for(K, ch);
  // about two CTAs per SM: enough parallelism, few atomics per channel
  const int64_t target = 2 * static_cast<int64_t>(launch_cache().sms());
  const int rows_per_cta = static_cast<int>((M + target - 1) / target);
  const dim3 grid(static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
  const size_t smem = static_cast<size_t>(K) * sizeof(float);
  auto go = [&](auto kernel) {
    cudaError_t e = launch_cache().ensure_smem(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, threads, smem, st>>>(x, ldx, M, K, rows_per_cta, norm, gamma, beta, eps, act_max);
    return cudaGetLastError();
  };
  if (bf16) return ch == 4 ? go(calib_kernel<true, 4>) : go(calib_kernel<true, 8>);
  return ch == 4 ? go(calib_kernel<false, 4>) : go(calib_kernel<false, 8>);
}

cudaError_t launch_weight_colmax(const void* W, bool bf16, int64_t N, int K, float* wmax,
                                 cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  const int nchunks = K / kChunk;
  const int slabs = (nchunks + 31) / 32;
  // about four CTAs per SM (what fits at once: one wave of long-lived CTAs),
  // at least 64 rows (8 per warp) each, and no more row runs than gridDim.y
  // allows; fewer runs also mean fewer atomics (runs x K)
  const int64_t target = 4 * static_cast<int64_t>(launch_cache().sms());
  int64_t runs = target / slabs;
  if (runs < 1) runs = 1;
  int64_t rows = (N + runs - 1) / runs;
  if (rows < 64) rows = 64;
  const int64_t min_rows = (N + 65534) / 65535;
  if (rows < min_rows) rows = min_rows;
  rows = (rows + 7) / 8 * 8;
  const dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>((N + rows - 1) / rows));
  if (bf16)
    weight_colmax_kernel<true><<<grid, 256, 0, st>>>(W, N, K, rows, wmax);
  else
    weight_colmax_kernel<false><<<grid, 256, 0, st>>>(W, N, K, rows, wmax);
  return cudaGetLastError();
}

cudaError_t launch_smooth_finalize(const float* act_max, const float* wmax, float* s, int K,
                                   double alpha, float clamp_eps, const float* gamma,
                                   const float* beta, float* gf, float* bfo, cudaStream_t st) {
  const int threads = 256;
  smooth_finalize_kernel<<<(K + threads - 1) / threads, threads, 0, st>>>(
      act_max, wmax, s, K, alpha, clamp_eps, gamma, beta, gf, bfo);
  return cudaGetLastError();
}

bool rows_supported(int K) { return K % kChunk == 0 && pick_ch(K) != 0; }

}  // namespace sq
