// sq_launch.h -- host-side launchers of the library's kernels (internal; the
// public surface is include/sq.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sq {

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
cudaError_t launch_calibrate(const void* x, bool bf16, int64_t M, int K, int64_t ldx, int norm,
                             const float* gamma, const float* beta, float eps, float* act_max,
                             cudaStream_t st);
cudaError_t launch_weight_colmax(const void* W, bool bf16, int64_t N, int K, float* wmax,
                                 cudaStream_t st);
cudaError_t launch_smooth_finalize(const float* act_max, float* s, int K, double alpha,
                                   float clamp_eps, const float* gamma, const float* beta,
                                   float* gf, float* bfo, cudaStream_t st);

// gemm.cu
struct GemmPlan {
  int swap;       // 0: tokens on the MMA M side (prefill); 1: weight rows (decode)
  int pair;       // prefill on CTA pairs (2-SM MMA, 256 x 256 tiles)
  int bn;         // MMA N (tile width on the Q side)
  int splits;     // K slices
  size_t workspace_bytes;
};
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int path_hint, int split_k, int num_sms);
cudaError_t launch_gemm(const GemmPlan& plan, const int8_t* Xq, const int8_t* Wq,
                        const float* x_scale, const float* w_scale, int64_t M, int64_t N,
                        int64_t K, int epi, void* out, int64_t ldo, void* workspace,
                        int num_sms, int64_t wait_polls, int* error_word, cudaStream_t st);
int num_sms_current_device();

}  // namespace sq
