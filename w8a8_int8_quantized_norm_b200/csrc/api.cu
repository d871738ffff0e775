// api.cu -- the extern "C" entry points declared in include/sq.h: argument
// validation on the host (nothing is launched for a rejected call), the
// device error word, and the launches.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/sq.h"
#include "sq_launch.h"

namespace sq {
namespace {

// First device-side error recorded since the host last read it (0 = none);
// one copy per device.
__device__ int g_sq_device_error = 0;

std::atomic<int64_t> g_wait_polls{0};

constexpr int kMaxDevices = 64;

int* device_error_word() {
  static int* words[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!words[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sq_device_error) != cudaSuccess) return nullptr;
    words[dev] = static_cast<int*>(p);
  }
  return words[dev];
}

int sms_cached() {
  static int sms[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (!sms[dev]) sms[dev] = num_sms_current_device();
  return sms[dev];
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_dtype(int d) { return d == SQ_F32 || d == SQ_BF16; }
inline bool valid_norm(int n) { return n == SQ_NORM_NONE || n == SQ_NORM_RMS || n == SQ_NORM_LAYER; }
inline int64_t dsize(int d) { return d == SQ_BF16 ? 2 : 4; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline sq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

// Checks shared by every row-wise call on an activation / weight matrix.
sq_status check_rows(const void* x, int dtype, int64_t M, int64_t K, int64_t ld) {
  if (!valid_dtype(dtype) || M < 0 || K <= 0 || ld < K) return SQ_ERR_INVALID_ARG;
  if (M > 0 && !x) return SQ_ERR_INVALID_ARG;
  if (M > 0x7fffffff || K > 0x7fffffff) return SQ_ERR_UNSUPPORTED;
  if (K % 16 != 0 || (ld * dsize(dtype)) % 16 != 0 || !aligned16(x)) return SQ_ERR_ALIGNMENT;
  if (!rows_supported(static_cast<int>(K))) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}

sq_status check_vec(const float* p, bool required) {
  if (!p) return required ? SQ_ERR_INVALID_ARG : SQ_OK;
  return aligned16(p) ? SQ_OK : SQ_ERR_ALIGNMENT;
}

sq_status check_gemm(const int8_t* Xq, const int8_t* Wq, const float* x_scale,
                     const float* w_scale, int64_t M, int64_t N, int64_t K, int epi,
                     const void* out, int64_t ldo, int path_hint, int split_k) {
  if (M < 0 || N < 0 || K <= 0 || split_k < 0) return SQ_ERR_INVALID_ARG;
  if (epi != SQ_EPI_BF16 && epi != SQ_EPI_BF16_RELU && epi != SQ_EPI_I32_RAW)
    return SQ_ERR_INVALID_ARG;
  if (path_hint < 0 || path_hint > 3) return SQ_ERR_INVALID_ARG;
  if (ldo < N) return SQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SQ_OK;
  if (!Xq || !Wq || !out) return SQ_ERR_INVALID_ARG;
  if (epi != SQ_EPI_I32_RAW && (!x_scale || !w_scale)) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_OVERFLOW_RISK;
  if (M > 0x7fffffff || N > 0x7fffffff) return SQ_ERR_UNSUPPORTED;
  if (path_hint == 2 && M > 256) return SQ_ERR_UNSUPPORTED;
  const uintptr_t esz = epi == SQ_EPI_I32_RAW ? 4 : 2;
  if (K % 16 != 0 || !aligned16(Xq) || !aligned16(Wq) ||
      (reinterpret_cast<uintptr_t>(out) % esz) != 0)
    return SQ_ERR_ALIGNMENT;
  if ((x_scale && !aligned16(x_scale)) || (w_scale && !aligned16(w_scale))) return SQ_ERR_ALIGNMENT;
  return SQ_OK;
}

}  // namespace

LaunchCache& launch_cache() {
  static LaunchCache cache;
  return cache;
}

}  // namespace sq

using namespace sq;

extern "C" {

const char* sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG: invalid argument";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED: dtype or shape not supported";
    case SQ_ERR_ALIGNMENT: return "SQ_ERR_ALIGNMENT: pointer or row stride not 16-byte aligned";
    case SQ_ERR_OVERFLOW_RISK: return "SQ_ERR_OVERFLOW_RISK: K too large for exact INT32 accumulation";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA: CUDA runtime error";
    case SQ_ERR_PIPELINE_TIMEOUT: return "SQ_ERR_PIPELINE_TIMEOUT: a device pipeline wait gave up";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown sq_status";
}

void sq_set_wait_limit(int64_t polls) { g_wait_polls.store(polls < 0 ? 0 : polls); }

sq_status sq_get_device_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_sq_device_error, sizeof(int)) != cudaSuccess) return SQ_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_sq_device_error, &zero, sizeof(int)) != cudaSuccess) return SQ_ERR_CUDA;
  }
  return static_cast<sq_status>(v);
}

sq_status sq_calibrate_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                              sq_norm norm, const float* gamma, const float* beta, float eps,
                              float* act_max, void* stream) {
  if (!valid_norm(norm) || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_rows(x, dtype, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(act_max, true)) != SQ_OK) return st;
  if ((st = check_vec(gamma, false)) != SQ_OK) return st;
  if ((st = check_vec(beta, false)) != SQ_OK) return st;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_calibrate(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx, norm, gamma,
                                    beta, eps, act_max, err, as_stream(stream)));
}

sq_status sq_weight_column_max(const void* const* W, const int64_t* N, int num_w, sq_dtype dtype,
                               int64_t K, float* w_max, void* stream) {
  if (!W || !N || num_w < 1 || !valid_dtype(dtype) || K <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st;
  if ((st = check_vec(w_max, true)) != SQ_OK) return st;
  for (int l = 0; l < num_w; ++l) {
    if ((st = check_rows(W[l], dtype, N[l], K, K)) != SQ_OK) return st;
  }
  cudaStream_t cs = as_stream(stream);
  // the maxima accumulate as bit patterns (non-negative floats order like them)
  cudaError_t e = cudaMemsetAsync(w_max, 0, static_cast<size_t>(K) * sizeof(float), cs);
  for (int l = 0; l < num_w && e == cudaSuccess; ++l)
    e = launch_weight_colmax(W[l], dtype == SQ_BF16, N[l], static_cast<int>(K), w_max, cs);
  return from_cuda(e);
}

sq_status sq_smooth_scales_from_maxima(const float* act_max, const float* w_max, int64_t K,
                                       double alpha, float clamp_eps, const float* gamma,
                                       const float* beta, float* s, float* gamma_folded,
                                       float* beta_folded, void* stream) {
  if (K <= 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0 && alpha <= 1.0) || !(clamp_eps > 0.0f) || isinf(clamp_eps))
    return SQ_ERR_INVALID_ARG;
  sq_status st;
  if ((st = check_vec(act_max, true)) != SQ_OK) return st;
  if ((st = check_vec(w_max, true)) != SQ_OK) return st;
  if ((st = check_vec(s, true)) != SQ_OK) return st;
  if ((st = check_vec(gamma_folded, true)) != SQ_OK) return st;
  if ((st = check_vec(gamma, false)) != SQ_OK) return st;
  if ((st = check_vec(beta, false)) != SQ_OK) return st;
  if ((st = check_vec(beta_folded, false)) != SQ_OK) return st;
  return from_cuda(launch_smooth_finalize(act_max, w_max, s, static_cast<int>(K), alpha,
                                          clamp_eps, gamma, beta, gamma_folded, beta_folded,
                                          as_stream(stream)));
}

sq_status sq_compute_smooth_scales(const float* act_max, const void* const* W, const int64_t* N,
                                   int num_w, sq_dtype dtype, int64_t K, double alpha,
                                   float clamp_eps, const float* gamma, const float* beta,
                                   float* s, float* gamma_folded, float* beta_folded,
                                   void* stream) {
  if (!W || !N || num_w < 1 || !valid_dtype(dtype) || K <= 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0 && alpha <= 1.0) || !(clamp_eps > 0.0f) || isinf(clamp_eps))
    return SQ_ERR_INVALID_ARG;
  sq_status st;
  if ((st = check_vec(act_max, true)) != SQ_OK) return st;
  if ((st = check_vec(s, true)) != SQ_OK) return st;
  if ((st = check_vec(gamma_folded, true)) != SQ_OK) return st;
  if ((st = check_vec(gamma, false)) != SQ_OK) return st;
  if ((st = check_vec(beta, false)) != SQ_OK) return st;
  if ((st = check_vec(beta_folded, false)) != SQ_OK) return st;
  for (int l = 0; l < num_w; ++l) {
    if ((st = check_rows(W[l], dtype, N[l], K, K)) != SQ_OK) return st;
  }
  // s first holds the weight column maxima, then the smoothing factors
  st = sq_weight_column_max(W, N, num_w, dtype, K, s, stream);
  if (st != SQ_OK) return st;
  return sq_smooth_scales_from_maxima(act_max, s, K, alpha, clamp_eps, gamma, beta, s,
                                      gamma_folded, beta_folded, stream);
}

sq_status sq_smooth_quantize_weights(const void* W, sq_dtype dtype, int64_t N, int64_t K,
                                     int64_t ldw, const float* s, int8_t* Wq, float* w_scale,
                                     void* stream) {
  sq_status st = check_rows(W, dtype, N, K, ldw);
  if (st != SQ_OK) return st;
  if ((st = check_vec(s, false)) != SQ_OK) return st;
  if (N > 0) {
    if (!Wq) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Wq)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(w_scale, true)) != SQ_OK) return st;
  }
  // a weight row smoothed by s is the no-norm row path with s as multiplier
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_norm_quant(W, dtype == SQ_BF16, N, static_cast<int>(K), ldw,
                                     SQ_NORM_NONE, s, nullptr, 0.0f, Wq, w_scale, err,
                                     as_stream(stream)));
}

sq_status sq_norm_smooth_quant_per_token(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                         int64_t ldx, sq_norm norm, const float* gamma_folded,
                                         const float* beta_folded, float eps, int8_t* Xq,
                                         float* x_scale, void* stream) {
  if (!valid_norm(norm) || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_rows(x, dtype, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(gamma_folded, false)) != SQ_OK) return st;
  if ((st = check_vec(beta_folded, false)) != SQ_OK) return st;
  if (M > 0) {
    if (!Xq) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Xq)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(x_scale, true)) != SQ_OK) return st;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_norm_quant(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx, norm,
                                     gamma_folded, beta_folded, eps, Xq, x_scale, err,
                                     as_stream(stream)));
}

namespace {

// Shared checks of the per-tensor row calls.
sq_status check_tensor_rows(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                            sq_norm norm, const float* gamma, const float* beta, float eps) {
  if (!valid_norm(norm) || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_rows(x, dtype, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(gamma, false)) != SQ_OK) return st;
  if ((st = check_vec(beta, false)) != SQ_OK) return st;
  if (!norm_quant_pipe_supported(static_cast<int>(K), dtype == SQ_BF16)) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}

}  // namespace

sq_status sq_norm_smooth_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                                sq_norm norm, const float* gamma_folded,
                                const float* beta_folded, float eps, float* absmax,
                                void* stream) {
  sq_status st = check_tensor_rows(x, dtype, M, K, ldx, norm, gamma_folded, beta_folded, eps);
  if (st != SQ_OK) return st;
  if (!absmax) return SQ_ERR_INVALID_ARG;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_tensor_absmax_pipe(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx,
                                             norm, gamma_folded, beta_folded, eps, absmax, err,
                                             as_stream(stream)));
}

sq_status sq_norm_smooth_quant_per_tensor(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                          int64_t ldx, sq_norm norm, const float* gamma_folded,
                                          const float* beta_folded, float eps,
                                          const float* absmax, int8_t* Xq, float* x_scale,
                                          void* stream) {
  sq_status st = check_tensor_rows(x, dtype, M, K, ldx, norm, gamma_folded, beta_folded, eps);
  if (st != SQ_OK) return st;
  if (!absmax) return SQ_ERR_INVALID_ARG;
  if (M > 0) {
    if (!Xq) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Xq)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(x_scale, true)) != SQ_OK) return st;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_quant_fixed_pipe(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx, norm,
                                           gamma_folded, beta_folded, eps, absmax, Xq, x_scale,
                                           err, as_stream(stream)));
}

sq_status sq_quant_per_token_given_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                          int64_t ldx, const float* row_absmax, int8_t* Xq,
                                          float* x_scale, void* stream) {
  sq_status st = check_tensor_rows(x, dtype, M, K, ldx, SQ_NORM_NONE, nullptr, nullptr, 0.0f);
  if (st != SQ_OK) return st;
  if (M > 0) {
    if (!Xq) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Xq)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(x_scale, true)) != SQ_OK) return st;
    if ((st = check_vec(row_absmax, true)) != SQ_OK) return st;
  }
  if (M == 0) return SQ_OK;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_quant_given_pipe(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx,
                                           row_absmax, Xq, x_scale, err, as_stream(stream)));
}

sq_status sq_row_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                        float* row_absmax, void* stream) {
  sq_status st = check_tensor_rows(x, dtype, M, K, ldx, SQ_NORM_NONE, nullptr, nullptr, 0.0f);
  if (st != SQ_OK) return st;
  if (M == 0) return SQ_OK;
  if ((st = check_vec(row_absmax, true)) != SQ_OK) return st;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_row_absmax_pipe(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx,
                                          row_absmax, err, as_stream(stream)));
}

sq_status sq_dequant_i32(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                         const float* x_scale, const float* w_scale, sq_epilogue epi, void* out,
                         int64_t ldo, void* stream) {
  if (M < 0 || N < 0 || lda < N || ldo < N) return SQ_ERR_INVALID_ARG;
  if (epi != SQ_EPI_BF16 && epi != SQ_EPI_BF16_RELU) return SQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SQ_OK;
  if (!acc || !out || !x_scale || !w_scale) return SQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(acc) & 3u) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return SQ_ERR_ALIGNMENT;
  return from_cuda(launch_dequant_i32(acc, M, N, lda, x_scale, w_scale, epi, out, ldo,
                                      as_stream(stream)));
}

sq_status sq_llmint8_outliers(const float* col_absmax, int64_t K, float tau, float* mask,
                              int32_t* idx, int32_t* count, void* stream) {
  if (K <= 0 || K > SQ_LLMINT8_MAX_K || !(tau >= 0.0f)) return SQ_ERR_INVALID_ARG;
  if (!col_absmax || !mask || !idx || !count) return SQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(col_absmax) | reinterpret_cast<uintptr_t>(mask) |
       reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(count)) & 3u)
    return SQ_ERR_ALIGNMENT;
  return from_cuda(launch_llmint8_outliers(col_absmax, K, tau, mask, idx, count,
                                           as_stream(stream)));
}

sq_status sq_llmint8_combine(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                             const float* x_scale, const float* w_scale, const void* x,
                             sq_dtype x_dtype, int64_t ldx, const void* W, sq_dtype w_dtype,
                             int64_t ldw, int64_t K, const int32_t* idx, const int32_t* count,
                             sq_epilogue epi, void* out, int64_t ldo, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || lda < N || ldo < N || ldx < K || ldw < K)
    return SQ_ERR_INVALID_ARG;
  if (!valid_dtype(x_dtype) || !valid_dtype(w_dtype)) return SQ_ERR_INVALID_ARG;
  if (epi != SQ_EPI_BF16 && epi != SQ_EPI_BF16_RELU) return SQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return SQ_OK;
  if (!acc || !x_scale || !w_scale || !x || !W || !idx || !count || !out)
    return SQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(acc) & 3u) || (reinterpret_cast<uintptr_t>(out) & 1u) ||
      (reinterpret_cast<uintptr_t>(x) % dsize(x_dtype)) ||
      (reinterpret_cast<uintptr_t>(W) % dsize(w_dtype)))
    return SQ_ERR_ALIGNMENT;
  return from_cuda(launch_llmint8_combine(acc, M, N, lda, x_scale, w_scale, x, x_dtype == SQ_BF16,
                                          ldx, W, w_dtype == SQ_BF16, ldw, idx, count,
                                          epi == SQ_EPI_BF16_RELU ? 1 : 0, out, ldo,
                                          as_stream(stream)));
}

sq_status sq_norm_smooth_quant_per_token_fp8(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                             int64_t ldx, sq_norm norm,
                                             const float* gamma_folded, const float* beta_folded,
                                             float eps, uint8_t* Xq8, float* x_scale,
                                             void* stream) {
  sq_status st = check_tensor_rows(x, dtype, M, K, ldx, norm, gamma_folded, beta_folded, eps);
  if (st != SQ_OK) return st;
  if (M > 0) {
    if (!Xq8) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Xq8)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(x_scale, true)) != SQ_OK) return st;
  }
  if (M == 0) return SQ_OK;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_norm_quant_fp8_pipe(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx,
                                              norm, gamma_folded, beta_folded, eps, Xq8, x_scale,
                                              err, as_stream(stream)));
}

sq_status sq_smooth_quantize_weights_fp8(const void* W, sq_dtype dtype, int64_t N, int64_t K,
                                         int64_t ldw, const float* s, uint8_t* Wq8,
                                         float* w_scale, void* stream) {
  // a weight row smoothed by s is the no-norm row path with s as multiplier
  return sq_norm_smooth_quant_per_token_fp8(W, dtype, N, K, ldw, SQ_NORM_NONE, s, nullptr, 0.0f,
                                            Wq8, w_scale, stream);
}

sq_status sq_fp8_gemm_dequant(const uint8_t* Xq8, const uint8_t* Wq8, const float* x_scale,
                              const float* w_scale, int64_t M, int64_t N, int64_t K,
                              sq_epilogue epi, void* out, int64_t ldo, void* workspace,
                              size_t ws_bytes, int path_hint, void* stream) {
  if (epi != SQ_EPI_BF16 && epi != SQ_EPI_BF16_RELU && epi != SQ_EPI_F32_RAW)
    return SQ_ERR_INVALID_ARG;
  // the shape, alignment and scale checks of the INT8 call (a raw fp32
  // accumulator has the raw INT32 output's size and needs no scales)
  const sq_epilogue e = epi == SQ_EPI_F32_RAW ? SQ_EPI_I32_RAW : epi;
  sq_status st = check_gemm(reinterpret_cast<const int8_t*>(Xq8),
                            reinterpret_cast<const int8_t*>(Wq8), x_scale, w_scale, M, N, K, e,
                            out, ldo, path_hint, 0);
  if (st != SQ_OK) return st;
  if (M == 0 || N == 0) return SQ_OK;
  const int sms = sms_cached();
  // decode tiles run stream-K (fp32 partial sums added in a fixed order) when
  // a workspace is given; without one every tile runs its whole K
  GemmPlan plan = plan_gemm(M, N, K, path_hint, workspace ? 0 : 1, sms);
  if (plan.workspace_bytes > 0) {
    if (ws_bytes < plan.workspace_bytes) return SQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SQ_ERR_ALIGNMENT;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_gemm(plan, reinterpret_cast<const int8_t*>(Xq8),
                               reinterpret_cast<const int8_t*>(Wq8), x_scale, w_scale, M, N, K,
                               epi, out, ldo, workspace, sms, g_wait_polls.load(), err,
                               as_stream(stream), nullptr, true));
}

static sq_status silu_mul_quant(const void* gate_up, sq_dtype dtype, int64_t M, int64_t I,
                                int64_t ld_gu, void* Xq, float* x_scale, void* h_out,
                                int64_t ld_h, void* stream, bool fp8) {
  if (!valid_dtype(dtype) || M < 0 || I <= 0 || ld_gu < 2 * I) return SQ_ERR_INVALID_ARG;
  if (h_out && ld_h < I) return SQ_ERR_INVALID_ARG;
  if (dtype != SQ_BF16) return SQ_ERR_UNSUPPORTED;
  if (M > 0x7fffffff || I > 0x7fffffff) return SQ_ERR_UNSUPPORTED;
  if (M > 0 && (!gate_up || !Xq)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_vec(x_scale, M > 0);
  if (st != SQ_OK) return st;
  if (I % 16 != 0 || (ld_gu * 2) % 16 != 0 || !aligned16(gate_up) || !aligned16(Xq))
    return SQ_ERR_ALIGNMENT;
  if (h_out && (!aligned16(h_out) || (ld_h * 2) % 16 != 0)) return SQ_ERR_ALIGNMENT;
  if (!silu_mul_pipe_supported(static_cast<int>(I))) return SQ_ERR_UNSUPPORTED;
  if (M == 0) return SQ_OK;
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_silu_mul_quant_pipe(gate_up, M, static_cast<int>(I), ld_gu,
                                              static_cast<int8_t*>(Xq), x_scale, h_out, ld_h,
                                              err, as_stream(stream), fp8));
}

sq_status sq_silu_mul_quant_per_token(const void* gate_up, sq_dtype dtype, int64_t M, int64_t I,
                                      int64_t ld_gu, int8_t* Xq, float* x_scale, void* h_out,
                                      int64_t ld_h, void* stream) {
  return silu_mul_quant(gate_up, dtype, M, I, ld_gu, Xq, x_scale, h_out, ld_h, stream, false);
}

sq_status sq_silu_mul_quant_per_token_fp8(const void* gate_up, sq_dtype dtype, int64_t M,
                                          int64_t I, int64_t ld_gu, uint8_t* Xq8,
                                          float* x_scale, void* h_out, int64_t ld_h,
                                          void* stream) {
  return silu_mul_quant(gate_up, dtype, M, I, ld_gu, Xq8, x_scale, h_out, ld_h, stream, true);
}

sq_status sq_smooth_quantize_weights_per_tensor(const void* W, sq_dtype dtype, int64_t N,
                                                int64_t K, int64_t ldw, const float* s,
                                                int8_t* Wq, float* w_scale, float* w_absmax,
                                                void* stream) {
  sq_status st = check_tensor_rows(W, dtype, N, K, ldw, SQ_NORM_NONE, s, nullptr, 0.0f);
  if (st != SQ_OK) return st;
  if (!w_absmax) return SQ_ERR_INVALID_ARG;
  if (N > 0) {
    if (!Wq) return SQ_ERR_INVALID_ARG;
    if (!aligned16(Wq)) return SQ_ERR_ALIGNMENT;
    if ((st = check_vec(w_scale, true)) != SQ_OK) return st;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  cudaStream_t cs = as_stream(stream);
  // a weight row smoothed by s is the no-norm row path with s as multiplier
  cudaError_t e = cudaMemsetAsync(w_absmax, 0, sizeof(float), cs);
  if (e == cudaSuccess)
    e = launch_tensor_absmax_pipe(W, dtype == SQ_BF16, N, static_cast<int>(K), ldw, SQ_NORM_NONE,
                                  s, nullptr, 0.0f, w_absmax, err, cs);
  if (e == cudaSuccess)
    e = launch_quant_fixed_pipe(W, dtype == SQ_BF16, N, static_cast<int>(K), ldw, SQ_NORM_NONE, s,
                                nullptr, 0.0f, w_absmax, Wq, w_scale, err, cs);
  return from_cuda(e);
}

size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int split_k) {
  if (M <= 0 || N <= 0 || K <= 0 || split_k < 0) return 0;
  const int sms = sms_cached();
  size_t need = plan_gemm(M, N, K, 0, split_k, sms).workspace_bytes;
  if (M <= 256) {
    const size_t dec = plan_gemm(M, N, K, 2, split_k, sms).workspace_bytes;
    if (dec > need) need = dec;
  }
  return need;
}

sq_status sq_w8a8_gemm_plan(int64_t M, int64_t N, int64_t K, int path_hint, int split_k,
                            sq_gemm_plan_info* info) {
  if (!info || M < 0 || N < 0 || K <= 0 || split_k < 0 || path_hint < 0 || path_hint > 3)
    return SQ_ERR_INVALID_ARG;
  const int sms = sms_cached();
  const GemmPlan plan = plan_gemm(M, N, K, path_hint, split_k, sms);
  if (!plan.swap && split_k > 1) return SQ_ERR_UNSUPPORTED;
  sq_gemm_plan_info r{};
  r.kernel = plan.swap ? 2 : (plan.pair ? 1 : 0);
  r.tile_m = plan.pair ? 256 : 128;
  r.tile_n = plan.bn;
  r.split_k = plan.splits;
  r.stream_k = plan.streamk;
  const int64_t p_rows = plan.swap ? N : M, q_rows = plan.swap ? M : N;
  const int64_t tiles = ((p_rows + r.tile_m - 1) / r.tile_m) * ((q_rows + r.tile_n - 1) / r.tile_n);
  int64_t ctas = plan.streamk ? plan.grid : tiles * plan.splits;
  const int64_t sm_count = sms > 0 ? sms : 148;  // the planner's own default
  const int64_t cap = plan.pair ? (sm_count / 2) * 2 : sm_count;
  if (plan.pair) ctas *= 2;
  if (ctas > cap) ctas = cap;
  r.ctas = static_cast<int>(M == 0 || N == 0 ? 0 : ctas);
  r.launches = (M == 0 || N == 0) ? 0 : 1 + (plan.workspace_bytes > 0 ? 1 : 0);
  r.workspace_bytes = plan.workspace_bytes;
  *info = r;
  return SQ_OK;
}

sq_status sq_w8a8_gemm_dequant(const int8_t* Xq, const int8_t* Wq, const float* x_scale,
                               const float* w_scale, int64_t M, int64_t N, int64_t K,
                               sq_epilogue epi, void* out, int64_t ldo, void* workspace,
                               size_t ws_bytes, int path_hint, int split_k, void* stream) {
  sq_status st = check_gemm(Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, path_hint, split_k);
  if (st != SQ_OK) return st;
  if (M == 0 || N == 0) return SQ_OK;
  const int sms = sms_cached();
  const GemmPlan plan = plan_gemm(M, N, K, path_hint, split_k, sms);
  if (!plan.swap && split_k > 1) return SQ_ERR_UNSUPPORTED;
  if (plan.workspace_bytes > 0) {
    if (!workspace || ws_bytes < plan.workspace_bytes) return SQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SQ_ERR_ALIGNMENT;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_gemm(plan, Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, workspace,
                               sms, g_wait_polls.load(), err, as_stream(stream)));
}

sq_status sq_w8a8_gemm_dequant_rowmax(const int8_t* Xq, const int8_t* Wq, const float* x_scale,
                                      const float* w_scale, int64_t M, int64_t N, int64_t K,
                                      sq_epilogue epi, void* out, int64_t ldo, float* row_absmax,
                                      int path_hint, void* stream) {
  if (epi != SQ_EPI_BF16 && epi != SQ_EPI_BF16_RELU) return SQ_ERR_INVALID_ARG;
  if (path_hint == 2) return SQ_ERR_INVALID_ARG;
  sq_status st = check_gemm(Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, path_hint, 1);
  if (st != SQ_OK) return st;
  if (M == 0) return SQ_OK;
  if ((st = check_vec(row_absmax, true)) != SQ_OK) return st;
  cudaStream_t cs = as_stream(stream);
  // the running maxima start from zero (every output is >= 0 in magnitude)
  cudaError_t e = cudaMemsetAsync(row_absmax, 0, static_cast<size_t>(M) * sizeof(float), cs);
  if (e != cudaSuccess || N == 0) return from_cuda(e);
  const int sms = sms_cached();
  const GemmPlan plan = plan_gemm(M, N, K, path_hint == 0 ? 1 : path_hint, 1, sms);
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  return from_cuda(launch_gemm(plan, Xq, Wq, x_scale, w_scale, M, N, K, epi, out, ldo, nullptr,
                               sms, g_wait_polls.load(), err, cs, row_absmax));
}

sq_status sq_linear_w8a8(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                         sq_norm norm, const float* gamma_folded, const float* beta_folded,
                         float eps, const int8_t* Wq, const float* w_scale, int64_t N,
                         sq_epilogue epi, void* out, int64_t ldo, int8_t* Xq_scratch,
                         float* xscale_scratch, void* workspace, size_t ws_bytes, void* stream) {
  // validate both halves before launching either
  if (!valid_norm(norm) || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_rows(x, dtype, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(gamma_folded, false)) != SQ_OK) return st;
  if ((st = check_vec(beta_folded, false)) != SQ_OK) return st;
  if (M > 0 && N > 0 && (!Xq_scratch || !xscale_scratch)) return SQ_ERR_INVALID_ARG;
  st = check_gemm(Xq_scratch, Wq, xscale_scratch, w_scale, M, N, K, epi, out, ldo, 0, 0);
  if (st != SQ_OK) return st;
  if (M == 0 || N == 0) return SQ_OK;
  const int sms = sms_cached();
  const GemmPlan plan = plan_gemm(M, N, K, 0, 0, sms);
  if (plan.workspace_bytes > 0) {
    if (!workspace || ws_bytes < plan.workspace_bytes) return SQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SQ_ERR_ALIGNMENT;
  }
  int* err = device_error_word();
  if (!err) return SQ_ERR_CUDA;
  cudaStream_t cs = as_stream(stream);
  cudaError_t e = launch_norm_quant(x, dtype == SQ_BF16, M, static_cast<int>(K), ldx, norm,
                                    gamma_folded, beta_folded, eps, Xq_scratch, xscale_scratch,
                                    err, cs);
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  return from_cuda(launch_gemm(plan, Xq_scratch, Wq, xscale_scratch, w_scale, M, N, K, epi, out,
                               ldo, workspace, sms, g_wait_polls.load(), err, cs));
}

}  // extern "C"
