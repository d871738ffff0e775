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

constexpr int kCombRows = 16;   // rows per tile
constexpr int kCombCols = 256;  // columns of a CTA's slab (one per thread)
constexpr int kStages = 3;      // accumulator tiles in the shared-memory ring
constexpr int kRegLane = 8;     // outlier channels whose weights sit in registers
constexpr int kLaneCache = 16;  // outlier channels staged on chip (registers + shared)
constexpr int kGather = (kCombRows * kLaneCache + kCombCols - 1) / kCombCols;  // per thread
static_assert(kRegLane % 2 == 0 && kLaneCache % 2 == 0, "xo rows are read as pairs");
// dynamic shared memory: the accumulator ring [kStages][kCombRows][kCombCols]
// (int32), xo [2][kCombRows][kLaneCache] and wo [kLaneCache - kRegLane]
// [kCombCols] (fp64), the tiles' token scales [2][kCombRows] (fp32)
constexpr size_t kCombSmem =
    static_cast<size_t>(kStages) * kCombRows * kCombCols * sizeof(int32_t) +
    (2 * static_cast<size_t>(kCombRows) * kLaneCache +
     static_cast<size_t>(kLaneCache - kRegLane) * kCombCols) *
        sizeof(double) +
    2 * kCombRows * sizeof(float);

// Element i of a bf16 or fp32 array, widened (exactly) to fp64.
__device__ __forceinline__ double elem(const void* p, int64_t i, bool bf) {
  if (bf) {
    const uint16_t h = static_cast<const uint16_t*>(p)[i];
    return static_cast<double>(__uint_as_float(static_cast<uint32_t>(h) << 16));
  }
  return static_cast<double>(static_cast<const float*>(p)[i]);
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src))
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Starts the copies of a tile's accumulators (column n of its rows) into
// ring slot `slot`, as one commit group (empty past the last tile).
__device__ __forceinline__ void issue_tile(uint32_t ring, int slot, const int32_t* acc,
                                           int64_t lda, int64_t tile, int64_t tiles, int64_t M,
                                           int64_t n, bool col, int t) {
  if (col && tile < tiles) {
    const int64_t m0 = tile * kCombRows;
    const int rows = M - m0 < kCombRows ? static_cast<int>(M - m0) : kCombRows;
    const uint32_t dst = ring + static_cast<uint32_t>((slot * kCombRows * kCombCols + t) * 4);
    for (int g = 0; g < rows; ++g)
      cp_async4(dst + static_cast<uint32_t>(g * kCombCols * 4), acc + (m0 + g) * lda + n);
  }
  cp_async_commit();
}

// This thread's share of a tile's outlier inputs (entry i = r * kLaneCache + c
// of xo, zero past the rows or the count) and token scales.
struct TileInputs {
  double xg[kGather];
  float xs;
};

template <bool kXBF16>
__device__ __forceinline__ void load_inputs(TileInputs& L, int64_t m0, int rows,
                                            const float* __restrict__ x_scale, const void* x,
                                            int64_t ldx, const int32_t* __restrict__ idx,
                                            int ncache, int t) {
#pragma unroll
  for (int k = 0; k < kGather; ++k) {
    const int i = t + k * kCombCols;
    const int r = i / kLaneCache, c = i - r * kLaneCache;
    L.xg[k] = i < kCombRows * kLaneCache && r < rows && c < ncache
                  ? elem(x, (m0 + r) * ldx + idx[c], kXBF16)
                  : 0.0;
  }
  L.xs = t < rows ? x_scale[m0 + t] : 0.0f;
}

__device__ __forceinline__ void stage_inputs(const TileInputs& L, double* xo, float* xsr, int t) {
#pragma unroll
  for (int k = 0; k < kGather; ++k) {
    const int i = t + k * kCombCols;
    if (i < kCombRows * kLaneCache) xo[i] = L.xg[k];
  }
  if (t < kCombRows) xsr[t] = L.xs;
}

// out[m, n] = bf16(y), y = fl32(fl32(fl32(fl32(acc) xs[m]) ws[n]) + fl32(s)),
// ReLU on y when asked, where s = sum over the outlier channels j (ascending)
// of x[m, j] w[n, j] in fp64 (each product is exact in fp64, and fma rounds
// s + x w once, as the oracle's s = s + x * w does).
//
// A CTA owns the column slab blockIdx.x (thread = column) and walks the row
// tiles blockIdx.y, blockIdx.y + gridDim.y, ...  Its columns' outlier weights
// are read once (one scattered load per channel): the first kRegLane into
// registers (zero past the count), the next ones into the thread's own column
// of wo; channels past kLaneCache are read per row from global memory.  Each
// thread copies its own column of the accumulator tiles into a ring of
// kStages slots with cp.async, kStages - 1 tiles ahead (it reads back only
// what it copied, so the ring needs no barrier); the next tile's outlier
// inputs are loaded into registers before the current tile is computed and
// stored to the other xo buffer after it.  The register lane runs all
// kRegLane fused multiply-adds: a padded term adds 0 * 0 to s, which leaves s
// unchanged (s starts at +0 and a rounded sum is never -0).
template <bool kXBF16, bool kWBF16>
__global__ void __launch_bounds__(kCombCols, 3)
    llmint8_combine_kernel(const int32_t* __restrict__ acc, int64_t M, int64_t N, int64_t lda,
                           const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                           const void* __restrict__ x, int64_t ldx, const void* __restrict__ W,
                           int64_t ldw, const int32_t* __restrict__ idx,
                           const int32_t* __restrict__ count, int relu,
                           __nv_bfloat16* __restrict__ out, int64_t ldo) {
  extern __shared__ __align__(16) unsigned char comb_smem[];
  const int32_t* accs = reinterpret_cast<const int32_t*>(comb_smem);  // [slot][r][t]
  double* xo = reinterpret_cast<double*>(comb_smem + static_cast<size_t>(kStages) * kCombRows *
                                                         kCombCols * 4);  // [2][r][c]
  double* wo = xo + 2 * kCombRows * kLaneCache;  // [c - kRegLane][t]: thread t's own
  float* xsr = reinterpret_cast<float*>(wo + (kLaneCache - kRegLane) * kCombCols);  // [2][r]
  const uint32_t ring = smem_u32(comb_smem);
  const int t = threadIdx.x;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kCombCols + t;
  const bool col = n < N;
  const int nout = *count;
  const int ncache = min(nout, kLaneCache);
  const int64_t tiles = (M + kCombRows - 1) / kCombRows;
  const int64_t G = gridDim.y;
  int64_t tile = blockIdx.y;
  if (tile >= tiles) return;

#pragma unroll
  for (int k = 0; k < kStages - 1; ++k)
    issue_tile(ring, k, acc, lda, tile + k * G, tiles, M, n, col, t);
  double wr[kRegLane];
#pragma unroll
  for (int c = 0; c < kRegLane; ++c)
    wr[c] = col && c < ncache ? elem(W, n * ldw + idx[c], kWBF16) : 0.0;
  if (col)
    for (int c = kRegLane; c < ncache; ++c)
      wo[(c - kRegLane) * kCombCols + t] = elem(W, n * ldw + idx[c], kWBF16);
  const float ws = col ? w_scale[n] : 0.0f;

  auto rows_of = [&](int64_t tl) {
    const int64_t left = M - tl * kCombRows;
    return left < kCombRows ? static_cast<int>(left) : kCombRows;
  };
  TileInputs in;
  load_inputs<kXBF16>(in, tile * kCombRows, rows_of(tile), x_scale, x, ldx, idx, ncache, t);
  stage_inputs(in, xo, xsr, t);
  __syncthreads();
  int buf = 0, slot = 0;
  for (;;) {
    const int64_t next = tile + G;
    const bool has_next = next < tiles;
    // the slot read in the previous iteration takes the tile kStages - 1 ahead
    issue_tile(ring, slot == 0 ? kStages - 1 : slot - 1, acc, lda, tile + (kStages - 1) * G,
               tiles, M, n, col, t);
    if (has_next)
      load_inputs<kXBF16>(in, next * kCombRows, rows_of(next), x_scale, x, ldx, idx, ncache, t);
    cp_async_wait<kStages - 1>();  // this thread's copies of the current tile have landed
    const int64_t m0 = tile * kCombRows;
    const int rows = rows_of(tile);
    const double* xb = xo + buf * kCombRows * kLaneCache;
    const float* sb = xsr + buf * kCombRows;
    const int32_t* ab = accs + slot * kCombRows * kCombCols + t;
    if (col) {
      __nv_bfloat16* op = out + m0 * ldo + n;
      for (int g = 0; g < rows; ++g, op += ldo) {
        const double2* xr = reinterpret_cast<const double2*>(xb + g * kLaneCache);
        double s = 0.0;
#pragma unroll
        for (int c = 0; c < kRegLane; c += 2) {
          const double2 v = xr[c / 2];
          s = __fma_rn(v.x, wr[c], s);
          s = __fma_rn(v.y, wr[c + 1], s);
        }
        for (int c = kRegLane; c < ncache; ++c)
          s = __fma_rn(xb[g * kLaneCache + c], wo[(c - kRegLane) * kCombCols + t], s);
        for (int c = kLaneCache; c < nout; ++c) {
          const int j = idx[c];
          s = __fma_rn(elem(x, (m0 + g) * ldx + j, kXBF16), elem(W, n * ldw + j, kWBF16), s);
        }
        const float y8 = __fmul_rn(__fmul_rn(__int2float_rn(ab[g * kCombCols]), sb[g]), ws);
        float y = __fadd_rn(y8, __double2float_rn(s));
        if (relu) y = y > 0.0f ? y : 0.0f;  // -0 becomes +0
        *op = __float2bfloat16_rn(y);
      }
    }
    if (!has_next) break;
    // the other buffer was last read before the previous iteration's barrier
    stage_inputs(in, xo + (buf ^ 1) * kCombRows * kLaneCache, xsr + (buf ^ 1) * kCombRows, t);
    __syncthreads();
    buf ^= 1;
    slot = slot == kStages - 1 ? 0 : slot + 1;
    tile = next;
  }
  cp_async_wait<0>();  // no copy outlives the CTA
}

template <bool kXBF16, bool kWBF16>
cudaError_t launch_combine(dim3 grid, cudaStream_t st, const int32_t* acc, int64_t M, int64_t N,
                           int64_t lda, const float* x_scale, const float* w_scale, const void* x,
                           int64_t ldx, const void* W, int64_t ldw, const int32_t* idx,
                           const int32_t* count, int relu, __nv_bfloat16* out, int64_t ldo) {
  cudaError_t e = cudaFuncSetAttribute(llmint8_combine_kernel<kXBF16, kWBF16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kCombSmem));
  if (e != cudaSuccess) return e;
  llmint8_combine_kernel<kXBF16, kWBF16><<<grid, kCombCols, kCombSmem, st>>>(
      acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw, idx, count, relu, out, ldo);
  return cudaGetLastError();
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
  // one CTA per column slab and row-tile stream; the streams per slab fill
  // three CTAs per SM (one wave) when the slabs alone do not
  const int64_t slabs = (N + kCombCols - 1) / kCombCols;
  const int64_t tiles = (M + kCombRows - 1) / kCombRows;
  int64_t streams = 3 * static_cast<int64_t>(num_sms_current_device()) / slabs;
  if (streams > tiles) streams = tiles;
  if (streams < 1) streams = 1;
  if (streams > 65535) streams = 65535;
  if (slabs > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>(streams));
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (x_bf16 && w_bf16)
    return launch_combine<true, true>(grid, st, acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw,
                                      idx, count, relu, o, ldo);
  if (x_bf16)
    return launch_combine<true, false>(grid, st, acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw,
                                       idx, count, relu, o, ldo);
  if (w_bf16)
    return launch_combine<false, true>(grid, st, acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw,
                                       idx, count, relu, o, ldo);
  return launch_combine<false, false>(grid, st, acc, M, N, lda, x_scale, w_scale, x, ldx, W, ldw,
                                      idx, count, relu, o, ldo);
}

}  // namespace sq
