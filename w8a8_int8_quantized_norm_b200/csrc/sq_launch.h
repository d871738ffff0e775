// sq_launch.h -- host-side launchers of the library's kernels (internal; the
// public surface is include/sq.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <tuple>

namespace sq {

// Host-side launch queries (function attributes, occupancy, SM counts) are
// answered once per device and shape and remembered: they cost microseconds,
// comparable to the small kernels they launch.
class LaunchCache {
 public:
  // Makes sure `kernel` may use `smem` bytes of dynamic shared memory on the
  // current device; returns the CUDA error of the attribute call, if made.
  cudaError_t ensure_smem(const void* kernel, size_t smem) {
    const int dev = device();
    std::lock_guard<std::mutex> lock(mu_);
    size_t& have = smem_[std::make_pair(dev, kernel)];
    if (smem <= have) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e == cudaSuccess) have = smem;
    return e;
  }
  // Resident CTAs per SM of `kernel` for (threads, smem) on the current device.
  int blocks_per_sm(const void* kernel, int threads, size_t smem) {
    const int dev = device();
    std::lock_guard<std::mutex> lock(mu_);
    auto key = std::make_tuple(dev, kernel, threads, smem);
    auto it = occ_.find(key);
    if (it != occ_.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
      n = 1;
    if (n < 1) n = 1;
    occ_[key] = n;
    return n;
  }
  int sms() {
    const int dev = device();
    std::lock_guard<std::mutex> lock(mu_);
    auto it = sms_.find(dev);
    if (it != sms_.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    sms_[dev] = n;
    return n;
  }
  static int device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
  }

 private:
  std::mutex mu_;
  std::map<std::pair<int, const void*>, size_t> smem_;
  std::map<std::tuple<int, const void*, int, size_t>, int> occ_;
  std::map<int, int> sms_;
};

LaunchCache& launch_cache();

// rows.cu
bool rows_supported(int K);
cudaError_t launch_norm_quant(const void* x, bool bf16, int64_t M, int K, int64_t ldx, int norm,
                              const float* gamma, const float* beta, float eps, int8_t* q,
                              float* scale, int* err, cudaStream_t st);

// normquant.cu
bool norm_quant_pipe_supported(int K, bool bf16);
cudaError_t launch_norm_quant_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                   int norm, const float* gamma, const float* beta, float eps,
                                   int8_t* q, float* scale, int* err, cudaStream_t st);
bool calibrate_pipe_supported(int K, bool bf16);
cudaError_t launch_calibrate_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                  int norm, const float* gamma, const float* beta, float eps,
                                  float* act_max, int* err, cudaStream_t st);
// Per-tensor variants (rows the shared-memory ring holds: norm_quant_pipe_supported).
cudaError_t launch_tensor_absmax_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                      int norm, const float* gamma, const float* beta, float eps,
                                      float* absmax, int* err, cudaStream_t st);
cudaError_t launch_quant_fixed_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                    int norm, const float* gamma, const float* beta, float eps,
                                    const float* absmax, int8_t* q, float* scale, int* err,
                                    cudaStream_t st);
// Each row's max |x| (no norm) into row_absmax[M].
cudaError_t launch_row_absmax_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                   float* row_absmax, int* err, cudaStream_t st);
// Per-row codes from given row maxima (no norm): row i's step is
// fl32(row_absmax[i] / 127); codes clamp to +-127.
cudaError_t launch_quant_given_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                    const float* row_absmax, int8_t* q, float* scale, int* err,
                                    cudaStream_t st);
// Per-row codes of h = SiLU(gate) * up from bf16 rows [gate (I) | up (I)],
// h rounded to bf16 first (and stored to h_out [M, I], stride ldh, if given).
// Norm + per-row FP8 (e4m3) codes: step = fl32(max |y| / 448), codes
// e4m3(fl32(y * fl32(1 / step))); rows the pipeline supports only.
cudaError_t launch_norm_quant_fp8_pipe(const void* x, bool bf16, int64_t M, int K, int64_t ldx,
                                       int norm, const float* gamma, const float* beta,
                                       float eps, uint8_t* q, float* scale, int* err,
                                       cudaStream_t st);
bool silu_mul_pipe_supported(int I);
cudaError_t launch_silu_mul_quant_pipe(const void* gu, int64_t M, int I, int64_t ldgu,
                                       int8_t* q, float* scale, void* h_out, int64_t ldh,
                                       int* err, cudaStream_t st, bool fp8 = false);
cudaError_t launch_calibrate(const void* x, bool bf16, int64_t M, int K, int64_t ldx, int norm,
                             const float* gamma, const float* beta, float eps, float* act_max,
                             int* err, cudaStream_t st);
cudaError_t launch_weight_colmax(const void* W, bool bf16, int64_t N, int K, float* wmax,
                                 cudaStream_t st);
cudaError_t launch_smooth_finalize(const float* act_max, const float* wmax, float* s, int K,
                                   double alpha, float clamp_eps, const float* gamma,
                                   const float* beta, float* gf, float* bfo, cudaStream_t st);

// llmint8.cu (the LLM.int8() comparator)
cudaError_t launch_llmint8_outliers(const float* col_absmax, int64_t K, float tau, float* mask,
                                    int32_t* idx, int32_t* count, cudaStream_t st);
cudaError_t launch_llmint8_combine(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                                   const float* x_scale, const float* w_scale, const void* x,
                                   bool x_bf16, int64_t ldx, const void* W, bool w_bf16,
                                   int64_t ldw, const int32_t* idx, const int32_t* count, int relu,
                                   void* out, int64_t ldo, cudaStream_t st);

// gemm.cu
struct GemmPlan {
  int swap;       // 0: tokens on the MMA M side (prefill); 1: weight rows (decode)
  int pair;       // prefill on CTA pairs (2-SM MMA, 256 x 256 tiles)
  int bn;         // MMA N (tile width on the Q side)
  int splits;     // K slices
  int streamk;    // decode tiles: balanced k-block ranges per CTA + a fix-up pass
  int grid;       // stream-K: CTAs
  int64_t sk_iters;  // stream-K: tiles x k-blocks
  size_t workspace_bytes;
};
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int path_hint, int split_k, int num_sms);
cudaError_t launch_gemm(const GemmPlan& plan, const int8_t* Xq, const int8_t* Wq,
                        const float* x_scale, const float* w_scale, int64_t M, int64_t N,
                        int64_t K, int epi, void* out, int64_t ldo, void* workspace,
                        int num_sms, int64_t wait_polls, int* error_word, cudaStream_t st,
                        float* row_absmax = nullptr, bool fp8 = false);
int num_sms_current_device();
// The dequantising epilogue of an INT32 accumulator matrix acc [M, N]
// (stride lda): out = bf16(fl32(fl32(fl32(acc) x_scale[m]) w_scale[n])), ReLU
// for SQ_EPI_BF16_RELU.
cudaError_t launch_dequant_i32(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                               const float* x_scale, const float* w_scale, int epi, void* out,
                               int64_t ldo, cudaStream_t st);

}  // namespace sq
