// llmint8.cu -- LLM.int8()'s mixed-precision decomposition, as a comparator
// of the SmoothQuant path on the same inputs.
//
// Source page (by title and section): "LLM.int8() and SmoothQuant" -- "Fix 1:
// give the outliers their own lane (LLM.int8())" and "going deeper -- LLM.int8()
// decomposition": the outlier channels O = { j : max_t |X[t, j]| >= tau }
// (tau = 6) are multiplied in 16-bit, the others in INT8 with one scale per
// token row and one per output channel, and the two results are added.  The
// pages also give its cost: a gather, a second (16-bit) product and a merge.
//
// The layer runs as five calls of the library:
//   sq_weight_column_max on x      -> col_absmax[j] = max_t |x[t, j]|
//   sq_llmint8_outliers            -> mask (0 on O, 1 elsewhere), the channels of O
//   sq_norm_smooth_quant_per_token (no norm, multiplier = mask): per-token codes
//                                     of the other channels (O's codes are 0)
//   sq_w8a8_gemm_dequant (SQ_EPI_I32_RAW): the INT8 lane's accumulator
//   sq_llmint8_combine             -> the INT8 lane's epilogue, the 16-bit lane,
//                                     their sum, bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_launch.h"

namespace sq {
namespace {

constexpr int kOutThreads = 1024;

// One CTA: thread t owns channels [t * seg, (t + 1) * seg); the outlier
// counts of the segments are prefix-summed across the CTA, so idx lists O in
// ascending channel order (the same order on every call).
__global__ void __launch_bounds__(kOutThreads)
    llmint8_outliers_kernel(const float* __restrict__ col_absmax, int K, float tau,
                            float* __restrict__ mask, int32_t* __restrict__ idx,
                            int32_t* __restrict__ count) {
  __shared__ int warp_tot[kOutThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int seg = (K + kOutThreads - 1) / kOutThreads;
  const int j0 = t * seg, j1 = min(K, j0 + seg);
  int mine = 0;
  for (int j = j0; j < j1; ++j) mine += col_absmax[j] >= tau ? 1 : 0;
  // exclusive prefix sum of `mine` over the CTA
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kOutThreads / 32 ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < kOutThreads / 32) warp_tot[lane] = wi - w;  // exclusive, per warp
    if (lane == 31) *count = wi;
  }
  __syncthreads();
  int pos = warp_tot[warp] + incl - mine;
  for (int j = j0; j < j1; ++j) {
    const bool out = col_absmax[j] >= tau;
    mask[j] = out ? 0.0f : 1.0f;
    if (out) idx[pos++] = j;
  }
}

constexpr int kCombRows = 32;   // output rows per CTA
constexpr int kCombCols = 256;  // output columns per pass (one per thread)
constexpr int kLaneCache = 32;  // outlier channels held in shared memory / registers

// Element i of a bf16 or fp32 array, widened (exactly) to fp64.
__device__ __forceinline__ double elem(const void* p, int64_t i, bool bf) {
  if (bf) {
    const uint16_t h = static_cast<const uint16_t*>(p)[i];
    return static_cast<double>(__uint_as_float(static_cast<uint32_t>(h) << 16));
  }
  return static_cast<double>(static_cast<const float*>(p)[i]);
}

// out[m, n] = bf16(y), y = fl32(fl32(fl32(fl32(acc) xs[m]) ws[n]) + fl32(s)),
// ReLU on y when asked, where s = sum over the outlier channels j (ascending)
// of x[m, j] w[n, j] in fp64 (each product is exact in fp64, and fma rounds
// s + x w once, as the oracle's s = s + x * w does).  A CTA owns kCombRows
// rows, whose outlier inputs it gathers once into shared memory, and walks
// the column passes blockIdx.y, blockIdx.y + gridDim.y, ...; thread = column
// of a pass, its outlier weights in registers (the first kLaneCache
// channels; the rest are read as they come).
template <bool kXBF16, bool kWBF16>
__global__ void __launch_bounds__(kCombCols)
    llmint8_combine_kernel(const int32_t* __restrict__ acc, int64_t M, int64_t N, int64_t lda,
                           const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                           const void* __restrict__ x, int64_t ldx, const void* __restrict__ W,
                           int64_t ldw, const int32_t* __restrict__ idx,
                           const int32_t* __restrict__ count, int relu,
                           __nv_bfloat16* __restrict__ out, int64_t ldo) {
  __shared__ double xo[kCombRows][kLaneCache];
  __shared__ float xsr[kCombRows];
  const int t = threadIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kCombRows;
  const int rows = M - m0 < kCombRows ? static_cast<int>(M - m0) : kCombRows;
  const int nout = *count;
  const int ncache = min(nout, kLaneCache);
  for (int i = t; i < kCombRows * ncache; i += kCombCols) {
    const int r = i / ncache, c = i - r * ncache;
    xo[r][c] = r < rows ? elem(x, (m0 + r) * ldx + idx[c], kXBF16) : 0.0;
  }
  if (t < kCombRows) xsr[t] = t < rows ? x_scale[m0 + t] : 0.0f;
  __syncthreads();
  for (int64_t n0 = static_cast<int64_t>(blockIdx.y) * kCombCols; n0 < N;
       n0 += static_cast<int64_t>(gridDim.y) * kCombCols) {
    const int64_t n = n0 + t;
    if (n >= N) continue;
    double wv[kLaneCache];
#pragma unroll
    for (int c = 0; c < kLaneCache; ++c)
      wv[c] = c < ncache ? elem(W, n * ldw + idx[c], kWBF16) : 0.0;
    const float ws = w_scale[n];
    for (int r = 0; r < rows; ++r) {
      const int64_t m = m0 + r;
      double s = 0.0;
#pragma unroll
      for (int c = 0; c < kLaneCache; ++c)
        if (c < ncache) s = __fma_rn(xo[r][c], wv[c], s);
      for (int c = kLaneCache; c < nout; ++c) {
        const int j = idx[c];
        s = __fma_rn(elem(x, m * ldx + j, kXBF16), elem(W, n * ldw + j, kWBF16), s);
      }
      const float y8 = __fmul_rn(__fmul_rn(__int2float_rn(acc[m * lda + n]), xsr[r]), ws);
      float y = __fadd_rn(y8, __double2float_rn(s));
      if (relu) y = y > 0.0f ? y : 0.0f;  // -0 becomes +0
      out[m * ldo + n] = __float2bfloat16_rn(y);
    }
  }
}

}  // namespace

cudaError_t launch_llmint8_outliers(const float* col_absmax, int64_t K, float tau, float* mask,
                                    int32_t* idx, int32_t* count, cudaStream_t st) {
  llmint8_outliers_kernel<<<1, kOutThreads, 0, st>>>(col_absmax, static_cast<int>(K), tau, mask,
                                                     idx, count);
  return cudaGetLastError();
}

cudaError_t launch_llmint8_combine(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                                   const float* x_scale, const float* w_scale, const void* x,
                                   bool x_bf16, int64_t ldx, const void* W, bool w_bf16,
                                   int64_t ldw, const int32_t* idx, const int32_t* count, int relu,
                                   void* out, int64_t ldo, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  // row blocks, and column passes split over gridDim.y only as far as needed
  // to give every SM a few CTAs (few row blocks: small M)
  const int64_t row_blocks = (M + kCombRows - 1) / kCombRows;
  const int64_t passes = (N + kCombCols - 1) / kCombCols;
  int64_t col_split = (4 * static_cast<int64_t>(num_sms_current_device()) + row_blocks - 1) /
                      row_blocks;
  if (col_split > passes) col_split = passes;
  if (col_split < 1) col_split = 1;
  if (col_split > 65535) col_split = 65535;
  const dim3 grid(static_cast<unsigned>(row_blocks), static_cast<unsigned>(col_split));
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (x_bf16 && w_bf16)
    llmint8_combine_kernel<true, true><<<grid, kCombCols, 0, st>>>(
        acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw, idx, count, relu, o, ldo);
  else if (x_bf16)
    llmint8_combine_kernel<true, false><<<grid, kCombCols, 0, st>>>(
        acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw, idx, count, relu, o, ldo);
  else if (w_bf16)
    llmint8_combine_kernel<false, true><<<grid, kCombCols, 0, st>>>(
        acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw, idx, count, relu, o, ldo);
  else
    llmint8_combine_kernel<false, false><<<grid, kCombCols, 0, st>>>(
        acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw, idx, count, relu, o, ldo);
  return cudaGetLastError();
}

}  // namespace sq
